"""The FMA-pipe exp2 of the tensor-core attention softmax (attn_tc.cu, exp2_fma_x2), checked on
the CPU: its shipped fp32 coefficients against the fit that derives them
(csrc/fit_exp2_cubic.py), and the whole evaluation (round-to-integer by the 1.5 * 2^23 trick,
cubic in fp32 fused multiply-adds, exponent-field add) emulated in fp32 against 2^x in float64
over the range the softmax feeds it (x <= 0 after the max is subtracted, down to the -126 clamp)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "compressed_latent_space_cca_b200", "csrc", "attn_tc.cu")
# the fit's bound on [-1/2, 1/2] (1.013e-4) plus a few fp32 roundings of the evaluation
BOUND = 1.03e-4


def shipped_coefficients():
    text = open(SRC).read()
    body = text[text.index("void exp2_fma_x2"):]
    body = body[:body.index("\n}\n")]
    fmas = re.findall(r"fma2\(q0, q1, ([^;]*)\);", body)
    assert len(fmas) == 3, fmas
    nums = [[float(v.rstrip("f")) for v in re.findall(r"-?\d+\.\d+f", line)] for line in fmas]
    c3, c2 = nums[0][0], nums[0][2]   # q = c3 f + c2
    c1 = nums[1][0]                  # q = q f + c1
    assert nums[2] == [1.0, 1.0]     # q = q f + 1
    return np.float32(c1), np.float32(c2), np.float32(c3)


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_kernel(x):
    c1, c2, c3 = shipped_coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    ones = np.ones_like(f)
    q = fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    q = fma32(q, f, np.full_like(f, c1))
    q = fma32(q, f, ones)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_shipped_coefficients_are_the_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fit_exp2_cubic", os.path.join(ROOT, "compressed_latent_space_cca_b200", "csrc", "fit_exp2_cubic.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    fitted = mod.fit(iterations=200, points=4001)
    np.testing.assert_allclose(np.array(shipped_coefficients(), dtype=np.float64), fitted, atol=1e-6)
    assert mod.max_rel_error(np.array(shipped_coefficients(), dtype=np.float64)) <= 1.02e-4


def test_exp2_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-126.0, 0.0, 400001), rng.uniform(-30.0, 0.0, 200000),
                        np.arange(-126, 1) + 0.5, np.arange(-126, 1) - 0.5, np.arange(-126, 1).astype(np.float64)])
    x32 = x.astype(np.float32)
    x32 = x32[x32 >= -126.0]  # below the clamp the kernel returns 2^-126 on purpose
    got = exp2_kernel(x32).astype(np.float64)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()
    assert exp2_kernel(np.float32([0.0]))[0] == 1.0          # 2^0 exact: constant term 1
    assert exp2_kernel(np.float32([-1.0, -2.0]))[1] == 0.25  # integers land on the exponent
    assert exp2_kernel(np.float32([-500.0]))[0] == np.float32(2.0 ** -126)  # clamped, not flushed to garbage
