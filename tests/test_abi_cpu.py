"""Host-side checks of the C ABI: the library loads, exports every function
declared in include/cca.h, and validates configurations. No kernel runs."""
import ctypes
import os
import re

import pytest

import compressed_latent_space_cca_b200 as cca
from compressed_latent_space_cca_b200 import _capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "cca.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(cca_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_function():
    lib = _capi.load()
    names = declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(lib, n), n
        assert n in _capi.SIGNATURES, f"{n} has no ctypes signature"
    assert lib.cca_version() == 1


def test_struct_layouts():
    assert ctypes.sizeof(cca.CcaConfig) == 17 * 4
    assert ctypes.sizeof(cca.CcaWorkspaceLayout) == 2 * 8 + 2 * 4 + 8 * 8


def good(**kw):
    base = dict(batch=1, seq_len=16384, hidden=2048, n_q_heads=4, n_kv_heads=2, head_dim=128, dtype="bf16")
    base.update(kw)
    return cca.make_config(**base)


def test_valid_configs_and_workspace():
    assert cca.validate(good()) == cca.CCA_OK
    cfg = good()
    T, Lq, Lkv = 16384, 512, 256
    lay = cca.workspace_layout(cfg)
    assert lay.elem_bytes == 2 and lay.lat_dtype == cca.CCA_F16
    assert lay.q_offset >= T * (Lq + 2 * Lkv) * 2
    assert lay.k_att_offset - lay.q_offset >= T * Lq * 2
    assert lay.v_att_offset - lay.k_att_offset >= T * Lkv * 2
    assert lay.o_offset - lay.v_att_offset >= T * Lkv * 2
    assert lay.wo_offset - lay.o_offset >= T * Lq * 2
    assert lay.wc_offset - lay.wo_offset >= 2048 * Lq * 2
    assert lay.sched_offset - lay.wc_offset >= (4 + 2) * 128 * 128 * 2
    assert cca.workspace_size(cfg) == lay.total_bytes
    for off in (lay.qkv_lat_offset, lay.q_offset, lay.k_att_offset, lay.v_att_offset, lay.o_offset,
                lay.wo_offset, lay.wc_offset, lay.sched_offset, lay.total_bytes):
        assert off % 256 == 0
    tiny = cca.make_config(batch=1, seq_len=64, hidden=128, n_q_heads=2, n_kv_heads=2, head_dim=16, dtype="f32")
    assert cca.validate(tiny) == cca.CCA_OK
    lt = cca.workspace_layout(tiny)
    assert lt.elem_bytes == 4 and lt.lat_dtype == cca.CCA_F32
    assert lt.k_att_offset == lt.v_att_offset == lt.o_offset  # fp32 blocks read the cache directly


@pytest.mark.parametrize("bad,code", [
    (dict(batch=0), cca.CCA_ERR_INVALID_ARG),
    (dict(seq_len=0), cca.CCA_ERR_INVALID_ARG),
    (dict(n_kv_heads=3), cca.CCA_ERR_INVALID_ARG),
    (dict(head_dim=127, hidden=4 * 127), cca.CCA_ERR_INVALID_ARG),
    (dict(C=3), cca.CCA_ERR_INVALID_ARG),
    (dict(conv_kernel=0), cca.CCA_ERR_INVALID_ARG),
    (dict(qk_mean_mode=4), cca.CCA_ERR_INVALID_ARG),
    (dict(value_shift=2), cca.CCA_ERR_INVALID_ARG),
    (dict(rope_base=0.5), cca.CCA_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), cca.CCA_ERR_INVALID_ARG),
    (dict(head_dim=256, hidden=4096), cca.CCA_ERR_UNSUPPORTED),
])
def test_invalid_configs_rejected(bad, code):
    cfg = good(**bad)
    assert cca.validate(cfg) == code
    assert cca.workspace_size(cfg) == 0
    assert cca.library().cca_last_error_message().decode()


def test_bad_dtype_and_null_config():
    cfg = good()
    cfg.dtype = 7
    assert cca.validate(cfg) == cca.CCA_ERR_INVALID_ARG
    cfg.dtype = cca.CCA_F16  # fp16 is only an intermediate type
    assert cca.validate(cfg) == cca.CCA_ERR_INVALID_ARG
    lib = cca.library()
    assert lib.cca_validate(None) == cca.CCA_ERR_INVALID_ARG
    assert lib.cca_workspace_size(None) == 0
    assert lib.cca_status_string(cca.CCA_ERR_DEVICE_TIMEOUT) == b"device-side wait timed out"


def test_prefill_without_device_fails_cleanly():
    """No GPU here: the call must return an error status, never fall back."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = good(seq_len=128)
    lib = cca.library()
    null = [ctypes.c_void_p(16)] * 9
    outs = [ctypes.c_void_p(16)] * 3
    st = lib.cca_prefill(ctypes.byref(cfg), *null, *outs, None, ctypes.c_void_p(256), 1 << 40, None)
    assert st in (cca.CCA_ERR_CUDA, cca.CCA_ERR_UNSUPPORTED)
    st = lib.cca_prefill(ctypes.byref(cfg), *null, *outs, None, None, 0, None)
    assert st != cca.CCA_OK


def test_plain_block_configs():
    """conv_kernel 0 is a plain attention block: no convolutions, so QK-mean and the value shift
    must be off; its workspace has no channel-conv weight region."""
    plain = good(conv_kernel=0, qk_mean_mode=0, value_shift=0)
    assert cca.validate(plain) == cca.CCA_OK
    for kw in (dict(qk_mean_mode=3), dict(qk_mean_mode=1), dict(value_shift=1)):
        bad = good(conv_kernel=0, **{**dict(qk_mean_mode=0, value_shift=0), **kw})
        assert cca.validate(bad) == cca.CCA_ERR_INVALID_ARG
        assert "plain block" in cca.library().cca_last_error_message().decode()
    lay = cca.workspace_layout(plain)
    assert lay.sched_offset == lay.wc_offset
    assert cca.validate(good(conv_kernel=-1)) == cca.CCA_ERR_INVALID_ARG


def test_decode_workspace_and_shapes():
    """The decode workspace depends on the batch and head layout, not on the position; shapes the
    decode kernels do not take report 0."""
    sizes = {cca.decode_workspace_size(good(seq_len=s)) for s in (1, 100, 16384, 100000)}
    assert len(sizes) == 1 and sizes.pop() > 0
    assert cca.decode_workspace_size(good(batch=8)) > cca.decode_workspace_size(good(batch=1))
    assert cca.decode_workspace_size(good(n_q_heads=32, n_kv_heads=2, hidden=32 * 128)) == 0  # G = 16
    assert cca.decode_workspace_size(good(head_dim=16, hidden=4 * 16)) == 0
    assert cca.decode_workspace_size(good(head_dim=64, hidden=4 * 64)) > 0
    assert cca.decode_workspace_size(good(batch=0)) == 0


def test_decode_argument_checks():
    """Every argument error is reported before any launch (no GPU here)."""
    lib = cca.library()
    cfg = good(seq_len=10)
    p = ctypes.c_void_p(256)
    ws, nws = ctypes.c_void_p(1 << 20), cca.decode_workspace_size(cfg)

    def call(rows=16, ptrs=None, state=p, w=ws, n=nws, c=cfg):
        args = ptrs if ptrs is not None else [p] * 10
        return lib.cca_decode(ctypes.byref(c), rows, *args[:9], args[9], p, p, state, w, n, None)
    assert call(rows=9) == cca.CCA_ERR_INVALID_ARG
    assert "cache_rows" in lib.cca_last_error_message().decode()
    assert call(ptrs=[None] + [p] * 9) == cca.CCA_ERR_INVALID_ARG
    assert call(ptrs=[ctypes.c_void_p(258)] + [p] * 9) == cca.CCA_ERR_INVALID_ARG
    assert call(state=None) == cca.CCA_ERR_INVALID_ARG
    assert call(w=None) == cca.CCA_ERR_WORKSPACE
    assert call(w=ctypes.c_void_p(256 + 16)) == cca.CCA_ERR_WORKSPACE
    assert call(n=nws - 1) == cca.CCA_ERR_WORKSPACE
    plain = good(seq_len=10, conv_kernel=0, qk_mean_mode=0, value_shift=0)
    assert call(c=plain) == cca.CCA_ERR_INVALID_ARG  # a plain block has no conv state
    assert "plain block" in lib.cca_last_error_message().decode()
    assert call(c=good(seq_len=10, head_dim=16, hidden=64)) == cca.CCA_ERR_UNSUPPORTED


def test_backward_workspace_and_argument_checks():
    """The backward's workspace holds the forward's and its own fp32 buffers; shapes it does not take
    report 0; every argument error is reported before any launch (no GPU here)."""
    cfg = good(seq_len=100)
    n = cca.backward_workspace_size(cfg)
    assert n > cca.workspace_size(cfg)
    assert cca.backward_workspace_size(good(seq_len=200)) > n
    assert cca.backward_workspace_size(good(conv_kernel=0, qk_mean_mode=0, value_shift=0)) > 0  # plain block
    assert cca.backward_workspace_size(good(conv_kernel=9)) == 0
    assert cca.backward_workspace_size(good(batch=0)) == 0
    lib = cca.library()
    p = ctypes.c_void_p(256)

    def call(ins=None, grads=None, w=ctypes.c_void_p(1 << 20), nw=n, c=cfg):
        ins = ins if ins is not None else [p] * 9
        grads = grads if grads is not None else [p] * 10
        return lib.cca_backward(ctypes.byref(c), *ins, *grads, w, nw, None)
    assert call(ins=[None] + [p] * 8) == cca.CCA_ERR_INVALID_ARG
    assert call(ins=[p] * 8 + [ctypes.c_void_p(264)]) == cca.CCA_ERR_INVALID_ARG
    assert call(grads=[None] + [p] * 9) == cca.CCA_ERR_INVALID_ARG          # dy
    assert "dy" in lib.cca_last_error_message().decode()
    assert call(grads=[p] * 9 + [None]) == cca.CCA_ERR_INVALID_ARG          # dW_o
    assert call(w=None) == cca.CCA_ERR_WORKSPACE
    assert call(w=ctypes.c_void_p(256 + 16)) == cca.CCA_ERR_WORKSPACE
    assert call(nw=n - 1) == cca.CCA_ERR_WORKSPACE
    assert call(c=good(conv_kernel=9)) == cca.CCA_ERR_UNSUPPORTED
