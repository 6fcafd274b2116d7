"""Fit of the cubic that the attention kernel uses for 2^f, |f| <= 1/2 (attn_tc.cu, exp2_fma_x2).

The softmax of the tensor-core attention evaluates a share of its exponentials on the FMA pipes:
2^x = 2^n * 2^f with n = round(x), and 2^f ~ p(f) = 1 + f (c1 + f (c2 + f c3)). The constant
term is fixed at 1 so that 2^0 is exact. The coefficients minimise the largest relative error
|p(f) / 2^f - 1| on [-1/2, 1/2] by Lawson's iteratively reweighted least squares: a weighted
least-squares fit on a dense grid, with each point's weight multiplied by its current error
until the error curve levels out (equioscillation). Run it to print the coefficients, rounded to
fp32 as the kernel stores them, and the error bound that tests/test_exp2_cubic_cpu.py checks.
"""
import numpy as np


def fit(iterations: int = 400, points: int = 20001):
    f = np.linspace(-0.5, 0.5, points)
    target = np.exp2(f)
    # p(f) - 1 = c1 f + c2 f^2 + c3 f^3; relative residual (p(f) - 2^f) / 2^f
    A = np.stack([f, f * f, f * f * f], axis=1) / target[:, None]
    b = (target - 1.0) / target
    w = np.full(points, 1.0 / points)
    c = None
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w = w / w.sum()
    return c


def max_rel_error(c, points: int = 200001) -> float:
    f = np.linspace(-0.5, 0.5, points)
    p = 1.0 + f * (c[0] + f * (c[1] + f * c[2]))
    return float(np.max(np.abs(p / np.exp2(f) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = np.asarray(c, dtype=np.float32)
    print("c1 = %.8ff  c2 = %.8ff  c3 = %.8ff" % tuple(float(v) for v in c32))
    print("max relative error on [-1/2, 1/2]: %.3e (fp32 coefficients: %.3e)"
          % (max_rel_error(c), max_rel_error(c32.astype(np.float64))))
