"""ctypes declarations of the C ABI in include/cca.h (no logic here)."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, Structure, c_char_p, c_float, c_int, c_size_t, c_uint, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcca.so")

CCA_OK = 0
CCA_ERR_INVALID_ARG = 1
CCA_ERR_UNSUPPORTED = 2
CCA_ERR_WORKSPACE = 3
CCA_ERR_CUDA = 4
CCA_ERR_DEVICE_TIMEOUT = 5
CCA_ERR_NUMERIC_RANGE = 6

CCA_F32 = 0
CCA_BF16 = 1
CCA_F16 = 2

CCA_NOALLOC_WORKSPACE_BYTES = 64 << 20

CCA_PATH_AUTO = 0
CCA_PATH_SIMT = 1
CCA_PATH_TENSOR = 2


def CCA_PATH_TENSOR_MASK(bits: int) -> int:
    """bit0 down-projection, bit1 attention, bit2 output projection, bit3 preprocessing (mma.sync),
    bit4 preprocessing (tcgen05), bit5 value shift in the down-projection (with bits 0 and 4)."""
    return 0x100 | (bits & 63)


class CcaConfig(Structure):
    _fields_ = [
        ("batch", c_int),
        ("seq_len", c_int),
        ("hidden", c_int),
        ("C", c_int),
        ("n_q_heads", c_int),
        ("n_kv_heads", c_int),
        ("head_dim", c_int),
        ("conv_kernel", c_int),
        ("qk_mean_mode", c_int),
        ("value_shift", c_int),
        ("use_rope", c_int),
        ("rope_base", c_float),
        ("softmax_scale", c_float),
        ("dtype", c_int),
        ("out_dtype", c_int),
        ("kv_channel_offset", c_int),
        ("kv_total_channels", c_int),
    ]


class CcaPrefillOpts(Structure):
    _fields_ = [("path", c_int), ("stage_events", POINTER(c_void_p))]


class CcaWorkspaceLayout(Structure):
    _fields_ = [
        ("total_bytes", c_size_t),
        ("elem_bytes", c_size_t),
        ("lat_dtype", c_int),
        ("reserved", c_int),
        ("qkv_lat_offset", c_size_t),
        ("q_offset", c_size_t),
        ("k_att_offset", c_size_t),
        ("v_att_offset", c_size_t),
        ("o_offset", c_size_t),
        ("wo_offset", c_size_t),
        ("wc_offset", c_size_t),
        ("sched_offset", c_size_t),
    ]


class CcaPlan(Structure):
    _fields_ = [("down_proj_tensor", c_int), ("attention_tensor", c_int), ("out_proj_tensor", c_int),
                ("preproc_tensor", c_int), ("launches", c_int), ("value_shift_fused", c_int)]


_PREFILL_ARGS = [POINTER(CcaConfig)] + [c_void_p] * 9 + [c_void_p] * 4 + [c_void_p, c_size_t, c_void_p]

# name -> (restype, argtypes)
SIGNATURES = {
    "cca_validate": (c_int, [POINTER(CcaConfig)]),
    "cca_workspace_size": (c_size_t, [POINTER(CcaConfig)]),
    "cca_workspace_layout": (c_int, [POINTER(CcaConfig), POINTER(CcaWorkspaceLayout)]),
    "cca_plan": (c_int, [POINTER(CcaConfig), c_int, POINTER(CcaPlan)]),
    "cca_prefill": (c_int, _PREFILL_ARGS),
    "cca_prefill_ex": (c_int, _PREFILL_ARGS + [POINTER(CcaPrefillOpts)]),
    "cca_prefill_noalloc": (c_int, [POINTER(CcaConfig)] + [c_void_p] * 9 + [c_void_p] * 4 + [c_void_p]),
    "cca_prefill_host": (c_int, [POINTER(CcaConfig), c_void_p, c_void_p] + [c_void_p] * 8
                         + [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "cca_decode_workspace_size": (c_size_t, [POINTER(CcaConfig)]),
    "cca_decode": (c_int, [POINTER(CcaConfig), c_int] + [c_void_p] * 9 + [c_void_p] * 4
                   + [c_void_p, c_size_t, c_void_p]),
    "cca_backward_workspace_size": (c_size_t, [POINTER(CcaConfig)]),
    "cca_backward": (c_int, [POINTER(CcaConfig)] + [c_void_p] * 10 + [c_void_p] * 9
                     + [c_void_p, c_size_t, c_void_p]),
    "cca_prefill_train": (c_int, [POINTER(CcaConfig)] + [c_void_p] * 9 + [c_void_p] * 3
                          + [c_void_p, c_size_t, c_void_p]),
    "cca_backward_saved": (c_int, [POINTER(CcaConfig)] + [c_void_p] * 10 + [c_void_p] * 9
                           + [c_void_p, c_size_t, c_void_p]),
    "cca_poll_device_status": (c_int, [c_void_p]),
    "cca_selftest_wait_timeout": (c_int, [c_uint, c_void_p]),
    "cca_status_string": (c_char_p, [c_int]),
    "cca_last_error_message": (c_char_p, []),
    "cca_version": (c_int, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libcca.so once. Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m compressed_latent_space_cca_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
