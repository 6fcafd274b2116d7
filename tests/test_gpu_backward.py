"""GPU parity of the block's backward pass (cca_backward through the C ABI) against the float64
oracle's cca_block_backward, which is pinned by finite differences of the pinned forward.

Metric per gradient tensor: max |gpu - oracle| / rms(oracle) and the mean of the same ratio. Limits
are the forward's: fp32 blocks max <= 1e-4; bf16 blocks max <= 2e-2, mean <= 2e-3. Where the
forward keeps its intermediates in fp16 (bf16 blocks) every gradient inherits their 2^-11 rounding;
the backward's own arithmetic is fp32 and its token sums average those roundings, so the forward's
limits hold for the gradients too.
"""
import numpy as np
import pytest
import torch

import compressed_latent_space_cca_b200 as cca
import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = {"f32": (1e-4, None), "bf16": (2e-2, 2e-3)}


def _err(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite gradient"
    rms = np.sqrt(np.mean(ref * ref))
    rms = rms if rms > 0 else 1.0
    e = np.abs(gpu - ref) / rms
    return float(e.max()), float(e.mean())


def _run(shape, kv_split=None, out_dtype=None):
    inp = workloads.make_inputs(shape)
    dy = workloads.make_dy(shape)
    if out_dtype == "f32":
        dy = dy.float()
    cfg = cca.config_from_shape(shape, out_dtype)
    vfrom = None
    if kv_split is not None:  # one rank's share of a block twice as wide in KV groups
        rank, world = kv_split
        full_cfg = cfg
        cfg, dev_inp = cca.kv_group_shard(full_cfg, {k: v.cuda() for k, v in inp.items()}, rank, world)
        vfrom = cfg.kv_total_channels // 2 - cfg.kv_channel_offset
        inp = {k: v.cpu() for k, v in dev_inp.items()}
        shape = shape.replace(n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads)
    d_in = {k: v.cuda() for k, v in inp.items()}
    g = cca.backward(cfg, d_in, dy.cuda())
    assert cca.poll_device_status() == cca.CCA_OK
    ref = oracle.cca_block_backward(workloads.as_float64(inp), dy.double().numpy(), shape.n_q_heads,
                                    shape.n_kv_heads, shape.head_dim, qk_mean_mode=shape.qk_mean_mode,
                                    use_value_shift=bool(shape.value_shift), use_rope=bool(shape.use_rope),
                                    rope_base=shape.rope_base, softmax_scale=shape.softmax_scale,
                                    value_shift_from=vfrom)
    return {k: v.cpu().numpy() for k, v in g.items()}, ref


def _check(shape, got, ref):
    mx_lim, mean_lim = TOL[shape.dtype]
    report = {}
    for name in cca.GRAD_NAMES:
        mx, mean = _err(got[name], ref[name])
        report[name] = (mx, mean)
    bad = {k: v for k, v in report.items() if v[0] > mx_lim or (mean_lim is not None and v[1] > mean_lim)}
    assert not bad, f"{shape.name}: gradients out of tolerance {bad} (all: {report})"


def S_(name, B, S, E, nq, nkv, d, K, dtype="f32", **kw):
    return workloads.BlockShape(name, B, S, E, nq, nkv, d, K, dtype, 11, **kw)


FP32_CASES = [
    S_("ragged_gqa", 2, 100, 64, 4, 2, 16, 4),
    S_("mode_pre_norope", 1, 130, 128, 2, 2, 32, 3, qk_mean_mode=1, use_rope=0),
    S_("k1_g4_noshift", 1, 64, 64, 4, 1, 16, 1, qk_mean_mode=0, value_shift=0),
    S_("post_only_k2", 2, 37, 128, 8, 2, 16, 2, qk_mean_mode=2),
    S_("one_token", 1, 1, 64, 2, 1, 16, 4),
    S_("d128", 1, 70, 256, 2, 1, 128, 4),
    S_("d64_k8", 1, 150, 128, 2, 2, 64, 8, softmax_scale=0.2),
]


@pytest.mark.parametrize("shape", FP32_CASES, ids=[s.name for s in FP32_CASES])
def test_backward_fp32_matches_oracle(shape):
    got, ref = _run(shape)
    _check(shape, got, ref)


BF16_CASES = [
    S_("bf16_ccgqa", 1, 200, 1024, 4, 2, 128, 4, "bf16"),       # tcgen05 preprocessing in the forward
    S_("bf16_pre_mean", 2, 96, 256, 2, 2, 128, 4, "bf16", qk_mean_mode=1),  # mma.sync preprocessing
    S_("bf16_simt_d64", 1, 130, 128, 2, 1, 64, 3, "bf16"),     # SIMT forward
    S_("bf16_1k", 1, 1024, 1024, 4, 2, 128, 4, "bf16"),
    S_("bf16_g4_split", 1, 1600, 1024, 8, 2, 128, 4, "bf16"),   # key tiles split over CTAs, ragged
    S_("bf16_b2_mha", 2, 333, 512, 4, 4, 128, 3, "bf16"),       # G = 1, two sequences, ragged
]


@pytest.mark.parametrize("shape", BF16_CASES, ids=[s.name for s in BF16_CASES])
def test_backward_bf16_matches_oracle(shape):
    got, ref = _run(shape)
    _check(shape, got, ref)


def test_backward_bf16_block_fp32_output():
    """A bf16 block whose y (so dy) is fp32: the GEMM operands are converted to bf16 first."""
    shape = BF16_CASES[0]
    got, ref = _run(shape, out_dtype="f32")
    _check(shape, got, ref)


@pytest.mark.parametrize("rank", [0, 1])
def test_backward_kv_group_share(rank):
    """A share of the KV groups: the value shift's boundary is the whole block's."""
    shape = S_("share", 1, 80, 128, 4, 2, 16, 4)
    got, ref = _run(shape, kv_split=(rank, 2))
    _check(shape, got, ref)


PLAIN_CASES = [
    S_("plain_mha_bf16", 1, 300, 512, 4, 4, 128, 0, "bf16", qk_mean_mode=0, value_shift=0),
    S_("plain_gqa_fp32", 2, 90, 128, 4, 2, 32, 0, qk_mean_mode=0, value_shift=0),
]


@pytest.mark.parametrize("shape", PLAIN_CASES, ids=[s.name for s in PLAIN_CASES])
def test_backward_plain_block(shape):
    """A plain block (no convolutions, QK-mean or value shift: multi-head or grouped attention on the
    projections) against the oracle's backward of the same block written with one seq-conv tap of 1
    and identity channel mixes; the gradients of x and the projections must agree."""
    import numpy as np
    inp = workloads.make_inputs(shape)
    dy = workloads.make_dy(shape)
    cfg = cca.config_from_shape(shape)
    g = cca.backward(cfg, {k: v.cuda() for k, v in inp.items()}, dy.cuda())
    assert cca.poll_device_status() == cca.CCA_OK
    assert set(g) == {"x", "W_q", "W_k", "W_v", "W_o"}
    nq, nkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    ref_in = workloads.as_float64(inp)
    ref_in.update(convq_seq=np.ones((nq * d, 1)), convk_seq=np.ones((nkv * d, 1)),
                  convq_chan=np.broadcast_to(np.eye(d), (nq, d, d)).copy(),
                  convk_chan=np.broadcast_to(np.eye(d), (nkv, d, d)).copy())
    ref = oracle.cca_block_backward(ref_in, dy.double().numpy(), nq, nkv, d, qk_mean_mode=0,
                                    use_value_shift=False, use_rope=bool(shape.use_rope))
    mx_lim, mean_lim = TOL[shape.dtype]
    for name in g:
        mx, mean = _err(g[name].cpu().numpy(), ref[name])
        assert mx <= mx_lim and (mean_lim is None or mean <= mean_lim), (name, mx, mean)


def test_backward_overwrites_outputs():
    """Every gradient is written in full: outputs that start as NaN come back finite and equal to a
    second call's."""
    shape = FP32_CASES[0]
    inp = {k: v.cuda() for k, v in workloads.make_inputs(shape).items()}
    dy = workloads.make_dy(shape).cuda()
    cfg = cca.config_from_shape(shape)
    sh = {k: tuple(v.shape) for k, v in inp.items()}
    grads = {n: torch.full(sh[n], float("nan"), device="cuda") for n in cca.GRAD_NAMES}
    ws = torch.full((cca.backward_workspace_size(cfg),), 255, dtype=torch.uint8, device="cuda")
    a = cca.backward(cfg, inp, dy, grads=grads, workspace=ws)
    a = {k: v.clone() for k, v in a.items()}
    b = cca.backward(cfg, inp, dy)
    for n in cca.GRAD_NAMES:
        assert torch.isfinite(a[n]).all(), n
        torch.testing.assert_close(a[n], b[n], rtol=1e-5, atol=1e-6)


def test_backward_rejects_bad_arguments():
    shape = FP32_CASES[0]
    inp = {k: v.cuda() for k, v in workloads.make_inputs(shape).items()}
    cfg = cca.config_from_shape(shape)
    lib = cca.library()
    import ctypes
    n = cca.backward_workspace_size(cfg)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ptrs = [inp[k].data_ptr() for k in cca.INPUT_NAMES]
    g = [torch.empty(inp[k].shape, device="cuda").data_ptr() for k in cca.GRAD_NAMES]
    dy = workloads.make_dy(shape).cuda()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.cca_backward(ctypes.byref(cfg), *ptrs, None, *g, ws.data_ptr(), n, s)
    assert st == cca.CCA_ERR_INVALID_ARG
    st = lib.cca_backward(ctypes.byref(cfg), *ptrs, dy.data_ptr(), *g, ws.data_ptr(), n - 256, s)
    assert st == cca.CCA_ERR_WORKSPACE
    too_long = cca.config_from_shape(shape.replace(conv_kernel=9))
    assert cca.backward_workspace_size(too_long) == 0
    torch.cuda.synchronize()


@pytest.mark.parametrize("shape", [BF16_CASES[0], BF16_CASES[1], PLAIN_CASES[0]], ids=["ccgqa", "pre_mean", "plain_mha"])
def test_backward_from_saved_forward(shape):
    """prefill_train + backward(saved=True) gives prefill's outputs exactly and cca_backward's gradients
    up to the order of fp32 atomic sums (dK / dV across key-tile chunks, K-split GEMM slices, dW_c
    across row blocks), which can move a bf16 hi / lo split by one unit of the hi part (about 2^-16
    of a value): the same kernels run on the same values, only the forward is not recomputed. A
    saved path that read a wrong activation would differ by O(1)."""
    inp = {k: v.cuda() for k, v in workloads.make_inputs(shape).items()}
    dy = workloads.make_dy(shape).cuda()
    cfg = cca.config_from_shape(shape)
    ref_fwd = cca.prefill(cfg, inp)
    ref = cca.backward(cfg, inp, dy)
    fwd = cca.prefill_train(cfg, inp)
    for k in ("y", "k_cache", "v_cache"):
        assert torch.equal(fwd[k], ref_fwd[k]), k
    got = cca.backward(cfg, inp, dy, workspace=fwd["workspace"], saved=True)
    assert cca.poll_device_status() == cca.CCA_OK
    for n in got:
        a, b = got[n].double(), ref[n].double()
        rms = b.pow(2).mean().sqrt().clamp_min(1e-30)
        assert ((a - b).abs().max() / rms).item() <= 1e-3, n


def test_saved_forward_unsupported_for_fp32():
    shape = FP32_CASES[0]
    inp = {k: v.cuda() for k, v in workloads.make_inputs(shape).items()}
    cfg = cca.config_from_shape(shape)
    with pytest.raises(cca.CcaError) as e:
        cca.prefill_train(cfg, inp)
    assert e.value.status == cca.CCA_ERR_UNSUPPORTED
