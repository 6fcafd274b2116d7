"""B200 prefill of one Compressed Convolutional Attention (CCA / CCGQA) block.

Thin Python binding over the C ABI in include/cca.h (libcca.so, built in-tree
by `python -m compressed_latent_space_cca_b200.build`). This module only
marshals arguments: shapes, dtypes and pointers are checked and passed
through; every step of the block runs in the library's CUDA kernels. PyTorch
is used for device memory and streams. If libcca.so is missing, every call
raises: there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional, Sequence

import torch

from . import _capi
from ._capi import (  # noqa: F401
    CCA_BF16,
    CCA_ERR_CUDA,
    CCA_ERR_DEVICE_TIMEOUT,
    CCA_ERR_INVALID_ARG,
    CCA_ERR_NUMERIC_RANGE,
    CCA_ERR_UNSUPPORTED,
    CCA_ERR_WORKSPACE,
    CCA_F16,
    CCA_F32,
    CCA_OK,
    CCA_PATH_AUTO,
    CCA_PATH_SIMT,
    CCA_PATH_TENSOR,
    CCA_PATH_TENSOR_MASK,
    CcaConfig,
    CcaWorkspaceLayout,
)

INPUT_NAMES = ("x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan", "W_o")

_DT = {CCA_F32: torch.float32, CCA_BF16: torch.bfloat16, CCA_F16: torch.float16}
_DT_CODE = {torch.float32: CCA_F32, torch.bfloat16: CCA_BF16, "f32": CCA_F32, "bf16": CCA_BF16}


class CcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _capi.load()
        msg = lib.cca_last_error_message().decode()
        super().__init__(f"{where}: {lib.cca_status_string(status).decode()} ({msg})")
        self.status = status


def library() -> ctypes.CDLL:
    return _capi.load()


def make_config(*, batch: int, seq_len: int, hidden: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                conv_kernel: int = 4, dtype="bf16", out_dtype=None, qk_mean_mode: int = 3,
                value_shift: int = 1, use_rope: int = 1, rope_base: float = 10000.0,
                softmax_scale: float = 0.0, C: Optional[int] = None, kv_channel_offset: int = 0,
                kv_total_channels: int = 0) -> CcaConfig:
    """Build a cca_config_t. C defaults to hidden / (n_q_heads * head_dim)."""
    dt = _DT_CODE[dtype]
    odt = dt if out_dtype is None else _DT_CODE[out_dtype]
    if C is None:
        C = hidden // max(1, n_q_heads * head_dim)
    return CcaConfig(batch, seq_len, hidden, C, n_q_heads, n_kv_heads, head_dim, conv_kernel, qk_mean_mode,
                     value_shift, use_rope, rope_base, softmax_scale, dt, odt, kv_channel_offset, kv_total_channels)


def kv_group_shard(cfg: CcaConfig, inputs: Dict[str, torch.Tensor], rank: int, world: int):
    """The block made of one share of the KV groups, for splitting one sequence's heads over `world`
    GPUs: share `rank` holds KV groups [rank * n, (rank + 1) * n) (n = n_kv_heads / world) and their
    query heads. Returns (cfg, inputs) of that block: the rows of W_q, W_k, W_v and the conv weights
    of its heads, the columns of W_o of its query heads, x unchanged, and the V-channel offset and
    width of the whole block so that the value shift splits the whole block's V channels. The
    block's y summed over the shares is the whole block's y; its KV cache is the whole cache's slice
    of its heads."""
    nkv, nq, d = cfg.n_kv_heads, cfg.n_q_heads, cfg.head_dim
    if world < 1 or nkv % world != 0 or not 0 <= rank < world:
        raise ValueError("n_kv_heads must be a multiple of world, 0 <= rank < world")
    G = nq // nkv
    gk = nkv // world
    k0, k1 = rank * gk * d, (rank + 1) * gk * d                # V / K channels of the share
    q0, q1 = rank * gk * G * d, (rank + 1) * gk * G * d        # Q channels of the share
    out = {"x": inputs["x"], "W_q": inputs["W_q"][q0:q1].contiguous(), "W_k": inputs["W_k"][k0:k1].contiguous(),
           "W_v": inputs["W_v"][k0:k1].contiguous(),
           "W_o": inputs["W_o"][:, q0:q1].contiguous()}
    if cfg.conv_kernel > 0:
        out["convq_seq"] = inputs["convq_seq"][q0:q1].contiguous()
        out["convk_seq"] = inputs["convk_seq"][k0:k1].contiguous()
        out["convq_chan"] = inputs["convq_chan"][rank * gk * G:(rank + 1) * gk * G].contiguous()
        out["convk_chan"] = inputs["convk_chan"][rank * gk:(rank + 1) * gk].contiguous()
    sh = CcaConfig.from_buffer_copy(cfg)
    sh.n_q_heads, sh.n_kv_heads = gk * G, gk
    sh.C = cfg.hidden // (gk * G * d)
    sh.kv_channel_offset = cfg.kv_channel_offset + k0
    sh.kv_total_channels = cfg.kv_total_channels or nkv * d
    return sh, out


def config_from_shape(shape, out_dtype=None) -> CcaConfig:
    """cca_config_t from any object with the BlockShape attributes."""
    return make_config(batch=shape.batch, seq_len=shape.seq_len, hidden=shape.hidden,
                       n_q_heads=shape.n_q_heads, n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                       conv_kernel=shape.conv_kernel, dtype=shape.dtype, out_dtype=out_dtype,
                       qk_mean_mode=shape.qk_mean_mode, value_shift=shape.value_shift,
                       use_rope=shape.use_rope, rope_base=shape.rope_base, softmax_scale=shape.softmax_scale,
                       kv_channel_offset=getattr(shape, "kv_channel_offset", 0),
                       kv_total_channels=getattr(shape, "kv_total_channels", 0))


def validate(cfg: CcaConfig) -> int:
    return library().cca_validate(ctypes.byref(cfg))


def workspace_size(cfg: CcaConfig) -> int:
    return library().cca_workspace_size(ctypes.byref(cfg))


def workspace_layout(cfg: CcaConfig) -> CcaWorkspaceLayout:
    out = CcaWorkspaceLayout()
    st = library().cca_workspace_layout(ctypes.byref(cfg), ctypes.byref(out))
    if st != CCA_OK:
        raise CcaError(st, "cca_workspace_layout")
    return out


def plan(cfg: CcaConfig, path: int = CCA_PATH_AUTO) -> dict:
    """Which kernels cca_prefill_ex would launch on the current device."""
    out = _capi.CcaPlan()
    st = library().cca_plan(ctypes.byref(cfg), path, ctypes.byref(out))
    if st != CCA_OK:
        raise CcaError(st, "cca_plan")
    return {"down_proj_tensor": bool(out.down_proj_tensor), "attention_tensor": bool(out.attention_tensor),
            "out_proj_tensor": bool(out.out_proj_tensor), "preproc_tensor": bool(out.preproc_tensor),
            "preproc_kind": {0: "simt", 1: "mma", 2: "tcgen05"}[out.preproc_tensor], "launches": out.launches,
            "value_shift_fused": bool(out.value_shift_fused)}


def _shapes(cfg: CcaConfig) -> Dict[str, tuple]:
    B, S, E = cfg.batch, cfg.seq_len, cfg.hidden
    Lq, Lkv, K = cfg.n_q_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.conv_kernel
    d = cfg.head_dim
    return {
        "x": (B, S, E), "W_q": (Lq, E), "W_k": (Lkv, E), "W_v": (Lkv, E),
        "convq_seq": (Lq, K), "convq_chan": (cfg.n_q_heads, d, d),
        "convk_seq": (Lkv, K), "convk_chan": (cfg.n_kv_heads, d, d), "W_o": (E, Lq),
        "y": (B, S, E), "k_cache": (B, S, cfg.n_kv_heads, d), "v_cache": (B, S, cfg.n_kv_heads, d),
        "conv_state": (B, (K - 1) * (Lq + cfg.n_kv_heads * d) + cfg.n_kv_heads * d),
    }


def _input_ptrs(cfg: CcaConfig, tensors: Dict[str, torch.Tensor], names, dtype, device) -> list:
    """Device pointers of the block inputs; a plain block (conv_kernel 0) may omit the conv weights,
    which are then passed as NULL."""
    sh = _shapes(cfg)
    ptrs = []
    for n in names:
        if cfg.conv_kernel == 0 and n.startswith("conv") and tensors.get(n) is None:
            ptrs.append(None)
        else:
            ptrs.append(_check(tensors[n], n, sh[n], dtype, device))
    return ptrs


def _check(t: torch.Tensor, name: str, shape: tuple, dtype: torch.dtype, device) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def alloc_outputs(cfg: CcaConfig, device, conv_state: bool = False) -> Dict[str, torch.Tensor]:
    sh = _shapes(cfg)
    dt, odt = _DT[cfg.dtype], _DT[cfg.out_dtype]
    out = {
        "y": torch.empty(sh["y"], dtype=odt, device=device),
        "k_cache": torch.empty(sh["k_cache"], dtype=dt, device=device),
        "v_cache": torch.empty(sh["v_cache"], dtype=dt, device=device),
    }
    if conv_state:
        out["conv_state"] = torch.empty(sh["conv_state"], dtype=dt, device=device)
    return out


def alloc_workspace(cfg: CcaConfig, device) -> torch.Tensor:
    n = workspace_size(cfg)
    if n == 0:
        raise CcaError(validate(cfg), "cca_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)  # caching allocator: 512-byte aligned


def prefill(cfg: CcaConfig, inputs: Dict[str, torch.Tensor], *, out: Optional[Dict[str, torch.Tensor]] = None,
            workspace: Optional[torch.Tensor] = None, conv_state: bool = False, path: int = CCA_PATH_AUTO,
            stage_events: Optional[Sequence[torch.cuda.Event]] = None,
            stream: Optional[torch.cuda.Stream] = None) -> Dict[str, torch.Tensor]:
    """Run cca_prefill_ex on `stream` (default: the current stream).

    inputs: the nine tensors of INPUT_NAMES on one CUDA device, dtype cfg.dtype.
    Returns {"y", "k_cache", "v_cache", ["conv_state"], "workspace"}.
    """
    x = inputs["x"]
    device = x.device
    if device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    sh = _shapes(cfg)
    dt = _DT[cfg.dtype]
    ptrs = _input_ptrs(cfg, inputs, INPUT_NAMES, dt, device)
    if out is None:
        out = alloc_outputs(cfg, device, conv_state)
    y = _check(out["y"], "y", sh["y"], _DT[cfg.out_dtype], device)
    kc = _check(out["k_cache"], "k_cache", sh["k_cache"], dt, device)
    vc = _check(out["v_cache"], "v_cache", sh["v_cache"], dt, device)
    cs = _check(out["conv_state"], "conv_state", sh["conv_state"], dt, device) if "conv_state" in out else None
    if workspace is None:
        workspace = alloc_workspace(cfg, device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    opts = _capi.CcaPrefillOpts()
    opts.path = path
    if stage_events is not None:
        if len(stage_events) != 5:
            raise ValueError("stage_events needs 5 events")
        for ev in stage_events:  # torch creates the CUDA event on its first record
            if ev.cuda_event == 0:
                ev.record(stream)
        arr = (ctypes.c_void_p * 5)(*[ev.cuda_event for ev in stage_events])
        opts.stage_events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    st = library().cca_prefill_ex(ctypes.byref(cfg), *ptrs, y, kc, vc, cs, workspace.data_ptr(),
                                  workspace.numel(), ctypes.c_void_p(stream.cuda_stream), ctypes.byref(opts))
    if st != CCA_OK:
        raise CcaError(st, "cca_prefill")
    res = dict(out)
    res["workspace"] = workspace
    return res


def prefill_noalloc(cfg: CcaConfig, inputs: Dict[str, torch.Tensor], *,
                    out: Optional[Dict[str, torch.Tensor]] = None, conv_state: bool = False,
                    stream: Optional[torch.cuda.Stream] = None) -> Dict[str, torch.Tensor]:
    """cca_prefill_noalloc: the block with its intermediates in the library's own
    fixed device array (no workspace argument), for callers that must not allocate
    device memory while they run. Blocks needing more than
    CCA_NOALLOC_WORKSPACE_BYTES of workspace are rejected; calls that overlap on
    the GPU share that array and must be ordered by the caller."""
    x = inputs["x"]
    device = x.device
    if device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    sh = _shapes(cfg)
    dt = _DT[cfg.dtype]
    ptrs = _input_ptrs(cfg, inputs, INPUT_NAMES, dt, device)
    if out is None:
        out = alloc_outputs(cfg, device, conv_state)
    y = _check(out["y"], "y", sh["y"], _DT[cfg.out_dtype], device)
    kc = _check(out["k_cache"], "k_cache", sh["k_cache"], dt, device)
    vc = _check(out["v_cache"], "v_cache", sh["v_cache"], dt, device)
    cs = _check(out["conv_state"], "conv_state", sh["conv_state"], dt, device) if "conv_state" in out else None
    if stream is None:
        stream = torch.cuda.current_stream(device)
    st = library().cca_prefill_noalloc(ctypes.byref(cfg), *ptrs, y, kc, vc, cs, ctypes.c_void_p(stream.cuda_stream))
    if st != CCA_OK:
        raise CcaError(st, "cca_prefill_noalloc")
    return dict(out)


def prefill_host(cfg: CcaConfig, x_host: torch.Tensor, weights: Dict[str, torch.Tensor], x_dev: torch.Tensor,
                 y_dev: torch.Tensor, y_host: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                 workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """cca_prefill_host: x from (pinned) host memory, y back to (pinned) host memory."""
    device = x_dev.device
    sh = _shapes(cfg)
    dt = _DT[cfg.dtype]
    if x_host.device.type != "cpu" or y_host.device.type != "cpu":
        raise ValueError("x_host and y_host must be host tensors")
    if tuple(x_host.shape) != sh["x"] or x_host.dtype != dt or not x_host.is_contiguous():
        raise ValueError("x_host shape/dtype mismatch")
    if tuple(y_host.shape) != sh["y"] or y_host.dtype != _DT[cfg.out_dtype] or not y_host.is_contiguous():
        raise ValueError("y_host shape/dtype mismatch")
    wp = _input_ptrs(cfg, weights, INPUT_NAMES[1:], dt, device)
    xd = _check(x_dev, "x_dev", sh["x"], dt, device)
    yd = _check(y_dev, "y_dev", sh["y"], _DT[cfg.out_dtype], device)
    kc = _check(k_cache, "k_cache", sh["k_cache"], dt, device)
    vc = _check(v_cache, "v_cache", sh["v_cache"], dt, device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    st = library().cca_prefill_host(ctypes.byref(cfg), x_host.data_ptr(), xd, *wp, yd, y_host.data_ptr(), kc, vc,
                                    None, workspace.data_ptr(), workspace.numel(),
                                    ctypes.c_void_p(stream.cuda_stream))
    if st != CCA_OK:
        raise CcaError(st, "cca_prefill_host")


def decode_workspace_size(cfg: CcaConfig) -> int:
    """Bytes of workspace cca_decode needs (0 if the shape is not supported); independent of seq_len."""
    return library().cca_decode_workspace_size(ctypes.byref(cfg))


def decode(cfg: CcaConfig, x_t: torch.Tensor, weights: Dict[str, torch.Tensor], k_cache: torch.Tensor,
           v_cache: torch.Tensor, conv_state: Optional[torch.Tensor] = None, *, y: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """cca_decode: one decode step, the token at position cfg.seq_len - 1 of every sequence.

    x_t [B, E]; weights: the eight weight tensors of INPUT_NAMES[1:]; k_cache, v_cache
    [B, rows, n_kv, d] with rows >= seq_len (rows 0..t-1 read, row t written); conv_state
    [B, (K-1)*(Lq+Lkv) + Lkv] advanced in place (None for conv_kernel 0). Returns y_t [B, E].
    """
    device = x_t.device
    if device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    sh = _shapes(cfg)
    dt = _DT[cfg.dtype]
    B, E = cfg.batch, cfg.hidden
    xp = _check(x_t, "x_t", (B, E), dt, device)
    wp = _input_ptrs(cfg, weights, INPUT_NAMES[1:], dt, device)
    if k_cache.dim() != 4:
        raise ValueError("k_cache must be [B, rows, n_kv, d]")
    rows = k_cache.shape[1]
    cshape = (B, rows, cfg.n_kv_heads, cfg.head_dim)
    kc = _check(k_cache, "k_cache", cshape, dt, device)
    vc = _check(v_cache, "v_cache", cshape, dt, device)
    cs = None if conv_state is None else _check(conv_state, "conv_state", sh["conv_state"], dt, device)
    if y is None:
        y = torch.empty((B, E), dtype=_DT[cfg.out_dtype], device=device)
    yp = _check(y, "y_t", (B, E), _DT[cfg.out_dtype], device)
    if workspace is None:
        n = decode_workspace_size(cfg)
        if n == 0:
            raise CcaError(CCA_ERR_UNSUPPORTED, "cca_decode_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    st = library().cca_decode(ctypes.byref(cfg), rows, xp, *wp, yp, kc, vc, cs, workspace.data_ptr(),
                              workspace.numel(), ctypes.c_void_p(stream.cuda_stream))
    if st != CCA_OK:
        raise CcaError(st, "cca_decode")
    return y


GRAD_NAMES = ("x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan", "W_o")


def backward_workspace_size(cfg: CcaConfig) -> int:
    """Bytes of workspace cca_backward needs (0 if the configuration is not supported)."""
    return library().cca_backward_workspace_size(ctypes.byref(cfg))


def prefill_train(cfg: CcaConfig, inputs: Dict[str, torch.Tensor], *,
                  out: Optional[Dict[str, torch.Tensor]] = None, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> Dict[str, torch.Tensor]:
    """cca_prefill_train: the forward of a training step. Returns {"y", "k_cache", "v_cache",
    "workspace"}; pass the same inputs and that workspace to backward(..., saved=True)."""
    x = inputs["x"]
    device = x.device
    if device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    sh = _shapes(cfg)
    dt = _DT[cfg.dtype]
    ptrs = _input_ptrs(cfg, inputs, INPUT_NAMES, dt, device)
    if out is None:
        out = alloc_outputs(cfg, device)
    y = _check(out["y"], "y", sh["y"], _DT[cfg.out_dtype], device)
    kc = _check(out["k_cache"], "k_cache", sh["k_cache"], dt, device)
    vc = _check(out["v_cache"], "v_cache", sh["v_cache"], dt, device)
    if workspace is None:
        n = backward_workspace_size(cfg)
        if n == 0:
            raise CcaError(CCA_ERR_UNSUPPORTED, "cca_backward_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    st = library().cca_prefill_train(ctypes.byref(cfg), *ptrs, y, kc, vc, workspace.data_ptr(), workspace.numel(),
                                     ctypes.c_void_p(stream.cuda_stream))
    if st != CCA_OK:
        raise CcaError(st, "cca_prefill_train")
    res = dict(out)
    res["workspace"] = workspace
    return res


def backward(cfg: CcaConfig, inputs: Dict[str, torch.Tensor], dy: torch.Tensor, *,
             grads: Optional[Dict[str, torch.Tensor]] = None, workspace: Optional[torch.Tensor] = None,
             saved: bool = False, stream: Optional[torch.cuda.Stream] = None) -> Dict[str, torch.Tensor]:
    """cca_backward: the gradients of x and of the eight weights for dL/dy = dy.

    inputs: the nine tensors of INPUT_NAMES (dtype cfg.dtype); dy [B, S, E] in cfg.out_dtype.
    Returns fp32 tensors named as the inputs, in their shapes (overwritten, not accumulated); a plain
    block (conv_kernel 0) has no conv weights and returns no gradients for them. With saved=True the
    workspace is the one prefill_train filled for the same inputs (cca_backward_saved: no forward
    recomputation).
    """
    x = inputs["x"]
    device = x.device
    if device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    sh = _shapes(cfg)
    ptrs = _input_ptrs(cfg, inputs, INPUT_NAMES, _DT[cfg.dtype], device)
    dyp = _check(dy, "dy", sh["y"], _DT[cfg.out_dtype], device)
    names = [n for n in GRAD_NAMES if not (cfg.conv_kernel == 0 and n.startswith("conv"))]
    if grads is None:
        grads = {n: torch.empty(sh[n], dtype=torch.float32, device=device) for n in names}
    gp = [_check(grads[n], "d" + n, sh[n], torch.float32, device) if n in names else None for n in GRAD_NAMES]
    if workspace is None:
        if saved:
            raise ValueError("saved=True needs the workspace prefill_train filled")
        n = backward_workspace_size(cfg)
        if n == 0:
            raise CcaError(CCA_ERR_UNSUPPORTED, "cca_backward_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    fn = library().cca_backward_saved if saved else library().cca_backward
    st = fn(ctypes.byref(cfg), *ptrs, dyp, *gp, workspace.data_ptr(), workspace.numel(),
            ctypes.c_void_p(stream.cuda_stream))
    if st != CCA_OK:
        raise CcaError(st, "cca_backward_saved" if saved else "cca_backward")
    return grads


def poll_device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronize and return the device status (CCA_OK or CCA_ERR_DEVICE_TIMEOUT ...)."""
    s = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    return library().cca_poll_device_status(ctypes.c_void_p(s))


def selftest_wait_timeout(timeout_us: int, stream: Optional[torch.cuda.Stream] = None) -> int:
    s = stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream
    return library().cca_selftest_wait_timeout(timeout_us, ctypes.c_void_p(s))


def workspace_view(cfg: CcaConfig, workspace: torch.Tensor) -> Dict[str, torch.Tensor]:
    """Views of the intermediates left in the workspace by the last call."""
    L = workspace_layout(cfg)
    dt = _DT[L.lat_dtype]
    T = cfg.batch * cfg.seq_len
    Lq, Lkv = cfg.n_q_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim
    eb = L.elem_bytes

    def region(off, width):
        return workspace[off:off + T * width * eb].view(dt).view(cfg.batch, cfg.seq_len, width)
    out = {
        "qkv_lat": region(L.qkv_lat_offset, Lq + 2 * Lkv),
        "q": region(L.q_offset, Lq),
        "o": region(L.o_offset, Lq),
    }
    if L.v_att_offset > L.k_att_offset:
        out["k_att"] = region(L.k_att_offset, Lkv)
        out["v_att"] = region(L.v_att_offset, Lkv)
    return out
