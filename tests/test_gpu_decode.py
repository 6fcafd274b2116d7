"""GPU parity of the decode step (cca_decode through the C ABI) against the float64 oracle.

Two checks per case:
  * one step against the oracle's decode step given the same state (the GPU prefill's bf16 KV
    cache and conv state, read back): y_t, the new cache row, the advanced conv state, at the
    block's standard tolerance; cache rows other than t must not change;
  * prefill(S0) + decode steps against the oracle's prefill of all S0 + n tokens, row by row: the
    step reads the cache in the block's storage type, so its tolerance (DECODE_TOL) is the one
    derived for that rounding.
"""
import numpy as np
import pytest
import torch

import compressed_latent_space_cca_b200 as cca
import oracle
import workloads
from parity import TOL, assert_close, row_errors, to_device

pytestmark = pytest.mark.gpu

# bf16: the decode attends over the bf16 cache (the prefill's attention reads fp16 copies); with
# only the cache, o and y roundings an fp64 simulation gives a mean row error of about 2e-3
DECODE_TOL = {"f32": (1e-4, None), "bf16": (2e-2, 3e-3)}


def shape(**kw):
    base = dict(name="decode", batch=1, seq_len=300, hidden=2048, n_q_heads=4, n_kv_heads=2, head_dim=128,
                conv_kernel=4, dtype="bf16", seed=21)
    base.update(kw)
    return workloads.BlockShape(**base)


def oracle_inputs(sh, inp):
    if sh.conv_kernel == 0:
        one, oi = workloads.plain_as_identity(sh, inp)
        return one, workloads.as_float64(oi)
    return sh, workloads.as_float64(inp)


def weights(inp):
    return {k: v for k, v in inp.items() if k != "x"}


def setup_state(sh, dev, S0, rows):
    """GPU prefill of the first S0 tokens; caches widened to `rows` rows per sequence (NaN beyond
    the prefill, so a read of a row the step must not touch shows up), conv state zero when S0 = 0."""
    B, nkv, d = sh.batch, sh.n_kv_heads, sh.head_dim
    dt = workloads.torch_dtype(sh.dtype)
    kc = torch.full((B, rows, nkv, d), float("nan"), dtype=dt, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    K = sh.conv_kernel
    cs = None
    if K > 0:
        cs = torch.zeros((B, (K - 1) * (sh.latent_q + sh.latent_kv) + sh.latent_kv), dtype=dt, device="cuda")
    if S0 > 0:
        pre = sh.replace(seq_len=S0)
        pin = dict(dev)
        pin["x"] = dev["x"][:, :S0].contiguous()
        res = cca.prefill(cca.config_from_shape(pre), pin, conv_state=K > 0)
        kc[:, :S0] = res["k_cache"]
        vc[:, :S0] = res["v_cache"]
        if K > 0:
            cs.copy_(res["conv_state"])
    return kc, vc, cs


def run_steps(sh, dev, kc, vc, cs, S0, n, out_dtype=None):
    ys = []
    ws = None
    for i in range(n):
        t = S0 + i
        cfg = cca.config_from_shape(sh.replace(seq_len=t + 1), out_dtype)
        if ws is None:
            ws = torch.empty(cca.decode_workspace_size(cfg), dtype=torch.uint8, device="cuda")
        ys.append(cca.decode(cfg, dev["x"][:, t].contiguous(), weights(dev), kc, vc, cs, workspace=ws))
    assert cca.poll_device_status() == cca.CCA_OK
    return torch.stack(ys, dim=1)


def np64(t):
    return t.double().cpu().numpy()


def check_one_step(sh, S0, rows=None):
    """One step against the oracle's step from the same (GPU-made) state."""
    inp = workloads.make_inputs(sh)
    dev = to_device(inp)
    rows = rows or S0 + 3
    kc, vc, cs = setup_state(sh, dev, S0, rows)
    k0, v0 = np64(kc), np64(vc)
    c0 = np64(cs) if cs is not None else None
    y = np64(run_steps(sh, dev, kc, vc, cs, S0, 1)[:, 0])
    k1, v1 = np64(kc), np64(vc)
    osh, oi = oracle_inputs(sh, inp)
    dt = sh.dtype
    for b in range(sh.batch):
        state = c0[b] if c0 is not None else np.zeros(osh.latent_kv)
        ref = oracle.decode_step(oi, oi["x"][b, S0], k0[b], v0[b], state, S0, sh.n_q_heads, sh.n_kv_heads,
                                 sh.head_dim, qk_mean_mode=sh.qk_mean_mode, use_value_shift=bool(sh.value_shift),
                                 use_rope=bool(sh.use_rope), rope_base=sh.rope_base,
                                 softmax_scale=sh.softmax_scale)
        assert_close(f"y[{b}]", y[b][None], ref["y"][None], dt)
        assert_close(f"k row t[{b}]", k1[b, S0].reshape(1, -1), ref["k"].reshape(1, -1), dt)
        assert_close(f"v row t[{b}]", v1[b, S0].reshape(1, -1), ref["v"].reshape(1, -1), dt)
        if c0 is not None:
            c1 = np64(cs)[b]
            assert_close(f"conv_state[{b}]", c1[None], ref["conv_state"][None], dt)
            K, lq, lkv = sh.conv_kernel, sh.latent_q, sh.latent_kv
            # the rows that only move are copied exactly
            np.testing.assert_array_equal(c1[:(K - 2) * lq], c0[b][lq:(K - 1) * lq])
            kq = (K - 1) * lq
            np.testing.assert_array_equal(c1[kq:kq + (K - 2) * lkv], c0[b][kq + lkv:kq + (K - 1) * lkv])
    # rows other than t are untouched (NaN beyond stays NaN)
    np.testing.assert_array_equal(k1[:, :S0], k0[:, :S0])
    np.testing.assert_array_equal(v1[:, :S0], v0[:, :S0])
    assert np.isnan(k1[:, S0 + 1:]).all() and np.isnan(v1[:, S0 + 1:]).all()


def check_end_to_end(sh, S0, n, out_dtype=None):
    """prefill(S0) + n decode steps against the oracle's prefill of S0 + n tokens."""
    inp = workloads.make_inputs(sh.replace(seq_len=S0 + n))
    full = sh.replace(seq_len=S0 + n)
    dev = to_device(inp)
    kc, vc, cs = setup_state(full, dev, S0, S0 + n + 5)
    y = np64(run_steps(full, dev, kc, vc, cs, S0, n, out_dtype))
    osh, oi = oracle_inputs(full, inp)
    ref = oracle.cca_block(oi, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, qk_mean_mode=sh.qk_mean_mode,
                           use_value_shift=bool(sh.value_shift), use_rope=bool(sh.use_rope),
                           rope_base=sh.rope_base, softmax_scale=sh.softmax_scale,
                           rows=list(range(S0, S0 + n)))
    mx_lim, mean_lim = DECODE_TOL[sh.dtype]
    mx, mean = row_errors(y, ref["y"])
    assert mx <= mx_lim and (mean_lim is None or mean <= mean_lim), (mx, mean)
    # the cache rows the steps wrote and the final conv state
    T = S0 + n
    assert_close("k rows", np64(kc)[:, S0:T], ref["k_cache"][:, S0:T], sh.dtype)
    assert_close("v rows", np64(vc)[:, S0:T], ref["v_cache"][:, S0:T], sh.dtype)
    if cs is not None:
        st = np.concatenate([ref["conv_state_q"].reshape(sh.batch, -1), ref["conv_state_k"].reshape(sh.batch, -1),
                             ref["conv_state_v"].reshape(sh.batch, -1)], axis=1)
        assert_close("conv_state", np64(cs), st, sh.dtype)
    return mx, mean


# ------------------------------------------------------------------------- one step, strict --
STEP_CASES = [
    dict(),                                                           # CCGQA E=2048, 2 chunks
    dict(seq_len=5000),                                               # 74 chunks per group, merged
    dict(batch=3, seq_len=700, n_q_heads=8, n_kv_heads=2, hidden=1024),        # G = 4
    dict(seq_len=400, n_q_heads=6, n_kv_heads=2, head_dim=64, hidden=768),     # G = 3 (heads padded to 4)
    dict(seq_len=257, n_q_heads=4, n_kv_heads=4, head_dim=32, hidden=512),     # G = 1, d = 32
    dict(seq_len=150, n_q_heads=2, n_kv_heads=1, hidden=512, qk_mean_mode=1),  # n_kv = 1: shift inside the head
    dict(batch=10, seq_len=90, n_q_heads=4, n_kv_heads=2, head_dim=64, hidden=512),  # two GEMV batches
    dict(seq_len=200, conv_kernel=1, qk_mean_mode=2, use_rope=0),
    dict(seq_len=120, conv_kernel=7, value_shift=0, n_q_heads=8, n_kv_heads=1, hidden=1024),  # G = 8
]


@pytest.mark.parametrize("case", range(len(STEP_CASES)))
def test_step_matches_oracle_step(case):
    sh = shape(**STEP_CASES[case])
    check_one_step(sh, sh.seq_len - 1)


def test_step_fp32():
    sh = shape(dtype="f32", batch=2, seq_len=130, n_q_heads=4, n_kv_heads=2, head_dim=32, hidden=256)
    check_one_step(sh, 129)


def test_first_token():
    """t = 0: empty cache, zero conv state (the state a sequence starts from)."""
    sh = shape(batch=2)
    check_one_step(sh, 0, rows=4)


# ------------------------------------------------------------------ prefill + decode, end to end --
E2E_CASES = [
    (dict(), 299, 3),
    (dict(batch=2, n_q_heads=8, n_kv_heads=2, hidden=1024), 1000, 2),
    (dict(seq_len=1, batch=2), 0, 4),                  # from the first token on
    (dict(dtype="f32", head_dim=64, hidden=512), 200, 3),
]


@pytest.mark.parametrize("case", range(len(E2E_CASES)))
def test_prefill_then_decode(case):
    kw, S0, n = E2E_CASES[case]
    check_end_to_end(shape(**kw), S0, n)


def test_prefill_then_decode_f32_out():
    check_end_to_end(shape(batch=2), 150, 2, out_dtype="f32")


# --------------------------------------------------------------------------- plain blocks --
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_plain_block_decode(dtype):
    sh = shape(conv_kernel=0, qk_mean_mode=0, value_shift=0, dtype=dtype, seq_len=260, n_q_heads=4,
               n_kv_heads=4, head_dim=64, hidden=256)
    check_one_step(sh, 259)
    check_end_to_end(sh, 255, 3)


def test_repeated_two_step_decode_finite():
    """The two-step end-to-end case of two sequences, repeated 200 times: every output finite.
    (Before every thread of an attention chunk fenced its partial rows ahead of the finished-chunk
    count, about one run in twenty of this case had the merging chunk read a partial row that had
    not landed, from a fresh workspace, and produce a non-finite row.)"""
    sh = shape(batch=2)
    S0, n = 150, 2
    full = sh.replace(seq_len=S0 + n)
    inp = workloads.make_inputs(full)
    dev = to_device(inp)
    for _ in range(200):
        kc, vc, cs = setup_state(full, dev, S0, S0 + n + 5)
        y = run_steps(full, dev, kc, vc, cs, S0, n, "f32")
        assert torch.isfinite(y).all()
