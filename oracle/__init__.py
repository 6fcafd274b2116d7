"""CPU float64 oracle of the CCA / CCGQA block.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
bench's CPU-baseline leg, never by the library.
"""
from .cca_oracle import (  # noqa: F401
    QK_MEAN_POST,
    QK_MEAN_PRE,
    attention_flops,
    block_flops,
    causal_attention,
    cca_block,
    cca_block_backward,
    channel_conv,
    decode_step,
    default_scale,
    down_project,
    qk_mean,
    qk_mean_adjoint,
    rope,
    rope_angles,
    rope_backward,
    seq_conv_backward,
    seq_conv_causal,
    value_shift,
    value_shift_backward,
)
