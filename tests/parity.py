"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the float64 oracle on the same seeded inputs, and measure the error.

Parity metric: per token row, |gpu - oracle| / rms(oracle row). The block's
outputs shrink as attention averages more tokens, so errors are judged
relative to each row's own scale. Limits: fp32 blocks max <= 1e-4; bf16
blocks max <= 2e-2 and mean <= 2e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import compressed_latent_space_cca_b200 as cca
import oracle
import workloads

TOL = {"f32": (1e-4, None), "bf16": (2e-2, 2e-3)}


def row_errors(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    W = ref.shape[-1]
    g2 = gpu.reshape(-1, W)
    r2 = ref.reshape(-1, W)
    rms = np.sqrt(np.mean(r2 * r2, axis=1, keepdims=True))
    glob = np.sqrt(np.mean(r2 * r2)) if r2.size else 1.0
    rms = np.where(rms > 0, rms, glob if glob > 0 else 1.0)
    err = np.abs(g2 - r2) / rms
    assert np.all(np.isfinite(g2)), "non-finite GPU output"
    return float(err.max()), float(err.mean())


def assert_close(name, gpu, ref, dtype):
    mx_lim, mean_lim = TOL[dtype]
    mx, mean = row_errors(gpu, ref)
    assert mx <= mx_lim, f"{name}: max row-normalised error {mx:.3e} > {mx_lim:.0e} (mean {mean:.3e})"
    if mean_lim is not None:
        assert mean <= mean_lim, f"{name}: mean row-normalised error {mean:.3e} > {mean_lim:.0e}"
    return mx, mean


def to_device(inputs, device="cuda"):
    return {k: v.to(device) for k, v in inputs.items()}


def run_gpu(shape, inputs, path=cca.CCA_PATH_AUTO, conv_state=False, out_dtype=None, rows=None,
            keep_device=False, stages=True):
    """One cca_prefill call; returns float64 numpy copies of the outputs (y only at
    `rows` if given) and of the workspace intermediates."""
    cfg = cca.config_from_shape(shape, out_dtype)
    d_in = to_device(inputs)
    res = cca.prefill(cfg, d_in, path=path, conv_state=conv_state)
    st = cca.poll_device_status()
    assert st == cca.CCA_OK, f"device status {st}"
    out = {}
    y = res["y"]
    if rows is not None:
        y = y[:, torch.as_tensor(rows, device=y.device)]
    out["y"] = y.double().cpu().numpy()
    for k in ("k_cache", "v_cache", "conv_state"):
        if k in res:
            out[k] = res[k].double().cpu().numpy()
    views = cca.workspace_view(cfg, res["workspace"])
    for k, v in views.items():
        if rows is not None and k == "o":
            v = v[:, torch.as_tensor(rows, device=v.device)]
        elif not stages:
            continue
        out[k] = v.double().cpu().numpy()
    if keep_device:
        out["_device"] = res
    out["_v_fused"] = cca.plan(cfg, path)["value_shift_fused"] and not conv_state
    return out


def run_oracle(shape, inputs, rows=None):
    return oracle.cca_block(workloads.as_float64(inputs), shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                            qk_mean_mode=shape.qk_mean_mode, use_value_shift=bool(shape.value_shift),
                            use_rope=bool(shape.use_rope), rope_base=shape.rope_base,
                            softmax_scale=shape.softmax_scale, rows=rows)


def sample_rows(S, n, seed=0):
    """Spread of query rows: the first and last tiles, tile edges, and random rows."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 2, 63, 64, 127, 128, 129, S // 2, S - 129, S - 128, S - 2, S - 1]
    rnd = rng.integers(0, S, size=max(0, n - len(fixed)))
    rows = sorted({int(r) for r in list(fixed) + list(rnd) if 0 <= r < S})
    return rows
