"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs, element by element, per row-normalised error."""
import numpy as np
import pytest
import torch

import compressed_latent_space_cca_b200 as cca
import workloads
from parity import assert_close, run_gpu, run_oracle, sample_rows

pytestmark = pytest.mark.gpu

SIMT, AUTO, TENSOR = cca.CCA_PATH_SIMT, cca.CCA_PATH_AUTO, cca.CCA_PATH_TENSOR
# every stage on its tensor-core kernel, the preprocessing on the warp-specialised tcgen05 kernel
WS = cca.CCA_PATH_TENSOR_MASK(1 | 2 | 4 | 16)
# the same with the value shift fused into the down-projection's epilogue (no v~ in the workspace)
WSV = cca.CCA_PATH_TENSOR_MASK(1 | 2 | 4 | 16 | 32)
PATHS = [SIMT, AUTO, TENSOR, WS, WSV]
PATH_IDS = ["simt", "auto", "tensor", "tcgen05pre", "vfused"]


def shape(**kw):
    base = dict(name="case", batch=1, seq_len=300, hidden=512, n_q_heads=4, n_kv_heads=2, head_dim=128,
                conv_kernel=4, dtype="bf16", seed=11)
    base.update(kw)
    return workloads.BlockShape(**base)


def check_all(sh, gpu, ref, stages=True):
    dt = sh.dtype
    assert_close("k_cache", gpu["k_cache"], ref["k_cache"], dt)
    assert_close("v_cache", gpu["v_cache"], ref["v_cache"], dt)
    if stages:
        T = sh.seq_len
        lq, lkv = sh.latent_q, sh.latent_kv
        lat = gpu["qkv_lat"]
        assert_close("q_lat", lat[..., :lq], ref["q_lat"], dt)
        assert_close("k_lat", lat[..., lq:lq + lkv], ref["k_lat"], dt)
        if not gpu.get("_v_fused"):  # the fused value shift leaves no v~ in the workspace
            assert_close("v_lat", lat[..., lq + lkv:], ref["v_lat"], dt)
        assert_close("q", gpu["q"], ref["q"], dt)
        if "k_att" in gpu:
            assert_close("k_att", gpu["k_att"], ref["k_cache"].reshape(gpu["k_att"].shape), dt)
            assert_close("v_att", gpu["v_att"], ref["v_cache"].reshape(gpu["v_att"].shape), dt)
        assert_close("o", gpu["o"], ref["o"], dt)
    return assert_close("y", gpu["y"], ref["y"], dt)


# --------------------------------------------------------------- fp32 tiny --
def test_tiny_fp32_block():
    sh = workloads.WORKLOADS["tiny_cca_fp32"]
    inp = workloads.make_inputs(sh)
    check_all(sh, run_gpu(sh, inp), run_oracle(sh, inp))


@pytest.mark.parametrize("S,nq,nkv,d,K", [(1, 2, 2, 16, 4), (65, 4, 1, 32, 4), (130, 4, 2, 64, 1),
                                          (97, 6, 3, 8, 7)])
def test_fp32_shapes(S, nq, nkv, d, K):
    sh = shape(dtype="f32", seq_len=S, n_q_heads=nq, n_kv_heads=nkv, head_dim=d, hidden=2 * nq * d,
               conv_kernel=K, batch=2)
    inp = workloads.make_inputs(sh)
    check_all(sh, run_gpu(sh, inp), run_oracle(sh, inp))


# ------------------------------------------------------------ bf16, small --
BF16_CASES = [
    dict(seq_len=300, n_q_heads=4, n_kv_heads=2, hidden=512),             # CCGQA, ragged tail
    dict(seq_len=256, n_q_heads=4, n_kv_heads=4, hidden=1024, batch=2),   # CCA, C=2
    dict(seq_len=1, n_q_heads=4, n_kv_heads=2, hidden=512),               # one token
    dict(seq_len=129, n_q_heads=8, n_kv_heads=2, hidden=1024, batch=3),   # G=4
    dict(seq_len=200, n_q_heads=2, n_kv_heads=1, hidden=512),             # n_kv=1: shift within the head
    dict(seq_len=383, n_q_heads=2, n_kv_heads=2, hidden=256),             # C=1
    dict(seq_len=300, n_q_heads=3, n_kv_heads=1, hidden=384),             # G=3; GEMM widths 640 and 384 end mid-tile
]


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("case", range(len(BF16_CASES)))
def test_bf16_small(path, case):
    sh = shape(**BF16_CASES[case])
    inp = workloads.make_inputs(sh)
    check_all(sh, run_gpu(sh, inp, path=path), run_oracle(sh, inp))


# The tensor-core attention runs the longest (query tile pair, KV group) items as two halves of
# their key range on different CTAs and merges the halves' partial rows. With 16 or fewer items the
# grid has one CTA per item, so the longest items are split whatever the GPU; every row is compared.
SPLIT_CASES = [
    dict(seq_len=1024, n_q_heads=4, n_kv_heads=2, hidden=512),  # G=2: two heads per item
    dict(seq_len=1000, n_q_heads=2, n_kv_heads=2, hidden=512),  # G=1: consecutive query tiles, ragged
]


@pytest.mark.parametrize("case", range(len(SPLIT_CASES)))
def test_bf16_split_key_ranges(case):
    sh = shape(**SPLIT_CASES[case])
    inp = workloads.make_inputs(sh)
    check_all(sh, run_gpu(sh, inp, path=TENSOR), run_oracle(sh, inp))


# Plain attention blocks (conv_kernel 0): the uncompressed baseline the method is compared
# against. The oracle computes each as the CCA block it equals, with one seq-conv tap of 1 and
# identity channel mixes (QK-mean and value shift off in both).
PLAIN_CASES = [
    dict(seq_len=300, n_q_heads=4, n_kv_heads=4, hidden=512),               # MHA, C = 1, ragged tail
    dict(seq_len=520, n_q_heads=4, n_kv_heads=2, hidden=512, batch=2),      # GQA, C = 1
    dict(seq_len=200, n_q_heads=2, n_kv_heads=2, hidden=1024, use_rope=0),  # C = 4, no RoPE
]


@pytest.mark.parametrize("path", [SIMT, AUTO], ids=["simt", "auto"])
@pytest.mark.parametrize("case", range(len(PLAIN_CASES)))
def test_plain_blocks(path, case):
    sh = shape(conv_kernel=0, qk_mean_mode=0, value_shift=0, **PLAIN_CASES[case])
    inp = workloads.make_inputs(sh)
    assert not any(n.startswith("conv") for n in inp)  # passed to the library as NULL
    one, oi = workloads.plain_as_identity(sh, inp)
    check_all(sh, run_gpu(sh, inp, path=path), run_oracle(one, oi))


def test_plain_block_fp32():
    sh = shape(dtype="f32", conv_kernel=0, qk_mean_mode=0, value_shift=0, seq_len=97, n_q_heads=4,
               n_kv_heads=2, head_dim=32, hidden=128, batch=2)
    inp = workloads.make_inputs(sh)
    one, oi = workloads.plain_as_identity(sh, inp)
    check_all(sh, run_gpu(sh, inp), run_oracle(one, oi))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
@pytest.mark.parametrize("mode,vshift,rope", [(0, 0, 0), (1, 0, 1), (2, 1, 0), (3, 1, 1), (0, 1, 1)])
def test_bf16_modes(path, mode, vshift, rope):
    sh = shape(seq_len=257, qk_mean_mode=mode, value_shift=vshift, use_rope=rope, batch=2)
    inp = workloads.make_inputs(sh)
    if path in (WS, WSV) and not mode & 2:
        # the tcgen05 preprocessing folds the after-conv mean into its MMAs: without it, it declines
        with pytest.raises(cca.CcaError) as ei:
            run_gpu(sh, inp, path=path)
        assert ei.value.status == cca.CCA_ERR_UNSUPPORTED
        return
    check_all(sh, run_gpu(sh, inp, path=path), run_oracle(sh, inp))


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_fp32_output_and_conv_state(path):
    sh = shape(seq_len=190, batch=2)
    inp = workloads.make_inputs(sh)
    gpu = run_gpu(sh, inp, path=path, conv_state=True, out_dtype="f32")
    ref = run_oracle(sh, inp)
    check_all(sh, gpu, ref, stages=False)
    K = sh.conv_kernel
    lq, lkv = sh.latent_q, sh.latent_kv
    cs = gpu["conv_state"]
    nq_part = (K - 1) * lq
    np.testing.assert_allclose(cs[:, :nq_part].reshape(2, K - 1, lq), ref["conv_state_q"], rtol=1e-2, atol=1e-2)
    np.testing.assert_allclose(cs[:, nq_part:nq_part + (K - 1) * lkv].reshape(2, K - 1, lkv), ref["conv_state_k"],
                               rtol=1e-2, atol=1e-2)
    np.testing.assert_allclose(cs[:, nq_part + (K - 1) * lkv:].reshape(2, 1, lkv), ref["conv_state_v"],
                               rtol=1e-2, atol=1e-2)
    # the conv state is the workspace latents converted to the block dtype: exact
    lat = torch.from_numpy(gpu["qkv_lat"][:, -(K - 1):, :lq]).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(cs[:, :nq_part].reshape(2, K - 1, lq), lat)


@pytest.mark.parametrize("path", PATHS, ids=PATH_IDS)
def test_deterministic_and_causal(path):
    """Three runs are bit-identical; perturbing x[t0] leaves every output row
    before t0 bit-identical (nothing reads the future)."""
    sh = shape(seq_len=520, batch=2)
    inp = workloads.make_inputs(sh)
    a = run_gpu(sh, inp, path=path)
    for _ in range(2):
        b = run_gpu(sh, inp, path=path)
        for k in ("y", "k_cache", "v_cache", "q", "o"):
            assert np.array_equal(a[k], b[k]), k
    t0 = 300
    inp2 = dict(inp)
    x = inp["x"].clone()
    x[1, t0] += 1.0
    inp2["x"] = x
    c = run_gpu(sh, inp2, path=path)
    for k in ("y", "k_cache", "v_cache"):
        assert np.array_equal(c[k][1, :t0], a[k][1, :t0]), k
        assert np.array_equal(c[k][0], a[k][0]), k
        assert not np.array_equal(c[k][1, t0], a[k][1, t0]), k


@pytest.mark.parametrize("path", [AUTO, TENSOR, WS, WSV], ids=["auto", "tensor", "tcgen05pre", "vfused"])
def test_bf16_long_ragged(path):
    """S = 4097: 33 query tiles whose last holds one row, two sequences, the split
    schedule of a long sequence; caches in full, y and O on sampled rows."""
    sh = shape(seq_len=4097, batch=2)
    inp = workloads.make_inputs(sh)
    rows = sample_rows(sh.seq_len, 40, seed=5)
    gpu = run_gpu(sh, inp, path=path, rows=rows, stages=False)
    ref = run_oracle(sh, inp, rows=rows)
    assert_close("k_cache", gpu["k_cache"], ref["k_cache"], "bf16")
    assert_close("v_cache", gpu["v_cache"], ref["v_cache"], "bf16")
    assert_close("o", gpu["o"], ref["o"], "bf16")
    assert_close("y", gpu["y"], ref["y"], "bf16")


# ------------------------------------------------- the five named workloads --
@pytest.mark.parametrize("path", [AUTO, TENSOR, WSV], ids=["auto", "tensor", "vfused"])
@pytest.mark.parametrize("name", ["cca_dense_bf16", "ccgqa_16k_bf16", "ccgqa_8x_bf16", "ccgqa_64k_bf16"])
def test_named_workload_full_size(name, path):
    """Full-size run in the bench's launch configuration (auto path) and with the tcgen05
    preprocessing; the KV cache is compared in full, y and the attention output on sampled rows
    the oracle computes one by one."""
    sh = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(sh)
    rows = sample_rows(sh.seq_len, 40, seed=sh.seed)
    gpu = run_gpu(sh, inp, rows=rows, stages=False, path=path)
    ref = run_oracle(sh, inp, rows=rows)
    assert_close("k_cache", gpu["k_cache"], ref["k_cache"], "bf16")
    assert_close("v_cache", gpu["v_cache"], ref["v_cache"], "bf16")
    assert_close("o", gpu["o"], ref["o"], "bf16")
    assert_close("y", gpu["y"], ref["y"], "bf16")
    del gpu
    torch.cuda.empty_cache()


# ----------------------------------------------- KV groups split over GPUs, on one GPU --
# One sequence's heads split in two shares of KV groups (es 2.C, 2.B item 2): each share is a block
# of its own, given the whole block's V-channel offset and width so that its value shift splits the
# whole block's V channels (es 2.B item 3); the shares' outputs summed are the whole block's y, and
# each share's KV cache is the whole cache's slice of its heads. Both shares run here, one after the
# other, through the C ABI (on several GPUs, one per GPU and one all-reduce of y).
SPLIT_PATHS = [AUTO, TENSOR, SIMT, WSV]


@pytest.mark.parametrize("path", SPLIT_PATHS, ids=["auto", "tensor", "simt", "vfused"])
@pytest.mark.parametrize("nq,nkv", [(4, 2), (8, 4)])
def test_kv_group_split_shares_sum_to_the_block(path, nq, nkv):
    sh = shape(seq_len=300, batch=2, n_q_heads=nq, n_kv_heads=nkv, hidden=nq * 128 * 2)
    inp = workloads.make_inputs(sh)
    cfg = cca.config_from_shape(sh, "f32")
    dev = {k: v.cuda() for k, v in inp.items()}
    ref = run_oracle(sh, inp)
    y = None
    for rank in range(2):
        cfg_r, inp_r = cca.kv_group_shard(cfg, dev, rank, 2)
        res = cca.prefill(cfg_r, inp_r, path=path)
        assert cca.poll_device_status() == cca.CCA_OK
        y = res["y"].double() if y is None else y + res["y"].double()
        gk = nkv // 2
        assert_close(f"k_cache[{rank}]", res["k_cache"].double().cpu().numpy(),
                     ref["k_cache"][:, :, rank * gk:(rank + 1) * gk], "bf16")
        assert_close(f"v_cache[{rank}]", res["v_cache"].double().cpu().numpy(),
                     ref["v_cache"][:, :, rank * gk:(rank + 1) * gk], "bf16")
    assert_close("y", y.cpu().numpy(), ref["y"], "bf16")


def test_kv_group_split_fp32():
    sh = shape(dtype="f32", seq_len=70, batch=2, n_q_heads=4, n_kv_heads=4, head_dim=16, hidden=128)
    inp = workloads.make_inputs(sh)
    cfg = cca.config_from_shape(sh)
    dev = {k: v.cuda() for k, v in inp.items()}
    ref = run_oracle(sh, inp)
    y = 0
    for rank in range(2):
        cfg_r, inp_r = cca.kv_group_shard(cfg, dev, rank, 2)
        res = cca.prefill(cfg_r, inp_r)
        assert cca.poll_device_status() == cca.CCA_OK
        y = y + res["y"].double()
        assert_close(f"v_cache[{rank}]", res["v_cache"].double().cpu().numpy(),
                     ref["v_cache"][:, :, rank * 2:(rank + 1) * 2], "f32")
    assert_close("y", y.cpu().numpy(), ref["y"], "f32")
