"""Seeded synthetic workloads for the CCA / CCGQA prefill block.

This module only names the workload shapes and draws seeded random tensors.
It holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from here without sharing any computation.

Shapes follow "Compressed Convolutional Attention: Efficient Attention in a
Compressed Latent Space" (gist.science/es/paper/2510.04476, section 2.A: the
latent width is E/C; section 2.C: K/V heads shared across query groups). The
pages train 1B dense and MoE models on Zyda2; no dataset or weights exist
here, so Gaussian tensors of the same shapes stand in for them:
x ~ N(0,1), projection weights ~ N(0,0.02), convolution weights ~ N(0,0.1).
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import torch


@dataclasses.dataclass(frozen=True)
class BlockShape:
    """One CCA / CCGQA block workload (all sizes in elements)."""

    name: str
    batch: int
    seq_len: int
    hidden: int          # E
    n_q_heads: int
    n_kv_heads: int
    head_dim: int        # d
    conv_kernel: int     # seq-conv taps K
    dtype: str           # "f32" or "bf16"
    seed: int
    qk_mean_mode: int = 3     # bit0: mean before the convs, bit1: mean after
    value_shift: int = 1
    use_rope: int = 1
    rope_base: float = 10000.0
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(head_dim)

    @property
    def latent_q(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def latent_kv(self) -> int:
        return self.n_kv_heads * self.head_dim

    @property
    def compression(self) -> int:
        """C = E / (n_q * d): the query latent is E/C wide."""
        return self.hidden // self.latent_q

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len

    def replace(self, **kw) -> "BlockShape":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 CCA block, dense CCA, and three CCGQA shapes
# (long prefill, 8x KV-cache compression with less-compressed queries, and a
# 64k context); and the MHA baseline of the long prefill.
WORKLOADS: Dict[str, BlockShape] = {
    "tiny_cca_fp32": BlockShape("tiny_cca_fp32", 1, 64, 128, 2, 2, 16, 4, "f32", 0),
    "cca_dense_bf16": BlockShape("cca_dense_bf16", 4, 4096, 2048, 4, 4, 128, 4, "bf16", 1),
    "ccgqa_16k_bf16": BlockShape("ccgqa_16k_bf16", 1, 16384, 2048, 4, 2, 128, 4, "bf16", 2),
    "ccgqa_8x_bf16": BlockShape("ccgqa_8x_bf16", 2, 8192, 2048, 8, 2, 128, 4, "bf16", 3),
    "ccgqa_64k_bf16": BlockShape("ccgqa_64k_bf16", 1, 65536, 4096, 8, 2, 128, 4, "bf16", 4),
    # the uncompressed baseline of the long prefill: plain multi-head attention (C = 1, 16 heads
    # of 128, no convolutions, QK-mean or value shift) at the same S and E
    "mha_16k_bf16": BlockShape("mha_16k_bf16", 1, 16384, 2048, 16, 16, 128, 0, "bf16", 6, qk_mean_mode=0,
                               value_shift=0),
}

# Order in which tensors are drawn from one generator; changing it changes
# every workload.
DRAW_ORDER = ("x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan",
              "convk_seq", "convk_chan", "W_o")

X_STD = 1.0
PROJ_STD = 0.02
CONV_STD = 0.1


def tensor_shapes(shape: BlockShape) -> Dict[str, tuple]:
    """Logical shape of every block input (row-major, torch Linear layout)."""
    B, S, E = shape.batch, shape.seq_len, shape.hidden
    Lq, Lkv, K = shape.latent_q, shape.latent_kv, shape.conv_kernel
    nq, nkv, d = shape.n_q_heads, shape.n_kv_heads, shape.head_dim
    return {
        "x": (B, S, E),
        "W_q": (Lq, E),
        "W_k": (Lkv, E),
        "W_v": (Lkv, E),
        "convq_seq": (Lq, K),
        "convq_chan": (nq, d, d),
        "convk_seq": (Lkv, K),
        "convk_chan": (nkv, d, d),
        "W_o": (E, Lq),
    }


def _std(name: str) -> float:
    if name == "x":
        return X_STD
    if name.startswith("conv"):
        return CONV_STD
    return PROJ_STD


def torch_dtype(dtype: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def make_inputs(shape: BlockShape, seed: int | None = None) -> Dict[str, torch.Tensor]:
    """Draw every block input on the CPU, seeded, cast to the workload dtype."""
    g = torch.Generator().manual_seed(shape.seed if seed is None else seed)
    shapes = tensor_shapes(shape)
    dt = torch_dtype(shape.dtype)
    out = {}
    for name in DRAW_ORDER:
        if shape.conv_kernel == 0 and name.startswith("conv"):
            continue  # a plain block has no convolutions
        t = torch.randn(shapes[name], generator=g, dtype=torch.float32)
        t.mul_(_std(name))
        out[name] = t.to(dt).contiguous()
    return out


def make_dy(shape: BlockShape, seed: int = 1) -> torch.Tensor:
    """A seeded gradient of the block output y [B, S, E] ~ N(0, 1) in the workload dtype (the
    upstream gradient a backward pass starts from)."""
    g = torch.Generator().manual_seed(1_000_003 * (shape.seed + 1) + seed)
    t = torch.randn((shape.batch, shape.seq_len, shape.hidden), generator=g, dtype=torch.float32)
    return t.to(torch_dtype(shape.dtype)).contiguous()


def as_float64(inputs: Dict[str, torch.Tensor]):
    """The same values as numpy float64 arrays (exact up-cast)."""
    return {k: v.to(torch.float64).numpy() for k, v in inputs.items()}


def plain_as_identity(shape: BlockShape, inputs: Dict[str, torch.Tensor]):
    """A plain block (conv_kernel 0) as the CCA block it equals: one seq-conv tap of 1, identity
    channel mixes (QK-mean and value shift are off in both)."""
    assert shape.conv_kernel == 0 and shape.qk_mean_mode == 0 and shape.value_shift == 0
    one = shape.replace(conv_kernel=1)
    return one, identity_convs(one, inputs)


def identity_convs(shape: BlockShape, inputs: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Replace the conv weights by identities (last seq tap 1, channel mix = I)."""
    out = dict(inputs)
    dt = inputs["x"].dtype
    K, d = shape.conv_kernel, shape.head_dim
    for side, L, H in (("q", shape.latent_q, shape.n_q_heads), ("k", shape.latent_kv, shape.n_kv_heads)):
        w = torch.zeros(L, K, dtype=dt)
        w[:, K - 1] = 1
        out[f"conv{side}_seq"] = w
        out[f"conv{side}_chan"] = torch.eye(d, dtype=dt).expand(H, d, d).contiguous()
    return out
