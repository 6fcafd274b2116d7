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
    channel_conv,
    decode_step,
    default_scale,
    down_project,
    qk_mean,
    rope,
    rope_angles,
    seq_conv_causal,
    value_shift,
)
