"""Pins of the oracle's backward pass (cca_block_backward) by central finite differences of its
forward pass: for L = <dy, y(theta)>, (L(theta + eps u) - L(theta - eps u)) / (2 eps) must equal
<dL/dtheta, u> for a random direction u of every input (x and every weight), and a few single
entries are checked one by one. The forward is pinned by the other oracle tests, so this ties the
hand-derived chain rule to something other than itself. Small float64 cases only."""
import numpy as np
import pytest

import oracle
import workloads

NAMES = ("x", "W_q", "W_k", "W_v", "convq_seq", "convq_chan", "convk_seq", "convk_chan", "W_o")


def _loss(inp, dy, nq, nkv, d, kw):
    return float((oracle.cca_block(inp, nq, nkv, d, **kw)["y"] * dy).sum())


def _case(nq, nkv, d, S, K, B=2, seed=3):
    sh = workloads.BlockShape("bwd", B, S, 2 * nq * d, nq, nkv, d, K, "f32", seed)
    inp = workloads.as_float64(workloads.make_inputs(sh))
    rng = np.random.default_rng(seed + 100)
    dy = rng.standard_normal(inp["x"].shape[:2] + (sh.hidden,))
    return inp, dy


@pytest.mark.parametrize("mode,vshift,rope_on,nq,nkv,K,vfrom", [
    (3, True, True, 4, 2, 4, None),
    (0, False, False, 2, 2, 1, None),
    (1, True, True, 3, 1, 3, None),
    (2, False, True, 4, 4, 2, None),
    (3, True, False, 4, 1, 4, None),
    (3, True, True, 4, 2, 4, 0),     # a share whose V channels all take the previous token
])
def test_backward_matches_finite_differences(mode, vshift, rope_on, nq, nkv, K, vfrom):
    d, S = 4, 9
    inp, dy = _case(nq, nkv, d, S, K)
    kw = dict(qk_mean_mode=mode, use_value_shift=vshift, use_rope=rope_on, value_shift_from=vfrom)
    grads = oracle.cca_block_backward(inp, dy, nq, nkv, d, **kw)
    rng = np.random.default_rng(7)
    eps = 1e-6
    for name in NAMES:
        assert grads[name].shape == inp[name].shape, name
        u = rng.standard_normal(inp[name].shape)
        plus = dict(inp, **{name: inp[name] + eps * u})
        minus = dict(inp, **{name: inp[name] - eps * u})
        fd = (_loss(plus, dy, nq, nkv, d, kw) - _loss(minus, dy, nq, nkv, d, kw)) / (2 * eps)
        an = float((grads[name] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_backward_single_entries():
    nq, nkv, d, S, K = 4, 2, 4, 7, 3
    inp, dy = _case(nq, nkv, d, S, K, B=1)
    grads = oracle.cca_block_backward(inp, dy, nq, nkv, d)
    eps = 1e-6
    for name, idx in (("x", (0, 3, 5)), ("W_k", (2, 1)), ("convq_chan", (1, 2, 3)), ("convk_seq", (5, 0)),
                      ("W_v", (7, 4)), ("W_o", (3, 6))):
        plus = {k: v.copy() for k, v in inp.items()}
        minus = {k: v.copy() for k, v in inp.items()}
        plus[name][idx] += eps
        minus[name][idx] -= eps
        fd = (_loss(plus, dy, nq, nkv, d, {}) - _loss(minus, dy, nq, nkv, d, {})) / (2 * eps)
        assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grads[name][idx])


def test_backward_adjoints():
    """Each hand-written transpose is the transpose of its forward step: <A z, w> = <z, A^T w>."""
    rng = np.random.default_rng(11)
    S, nq, nkv, d = 6, 6, 2, 4
    a, b = rng.standard_normal((S, nq * d)), rng.standard_normal((S, nkv * d))
    dq, dk = rng.standard_normal((S, nq * d)), rng.standard_normal((S, nkv * d))
    mq, mk = oracle.qk_mean(a, b, nq, nkv, d)
    da, db = oracle.qk_mean_adjoint(dq, dk, nq, nkv, d)
    assert abs((mq * dq).sum() + (mk * dk).sum() - (a * da).sum() - (b * db).sum()) < 1e-12
    z, w, ds = rng.standard_normal((S, 5)), rng.standard_normal((5, 3)), rng.standard_normal((S, 5))
    dz, dw = oracle.seq_conv_backward(z, w, ds)
    assert abs((oracle.seq_conv_causal(z, w) * ds).sum() - (z * dz).sum()) < 1e-12
    w2 = rng.standard_normal((5, 3))
    assert abs((oracle.seq_conv_causal(z, w2) * ds).sum() - (w2 * dw).sum()) < 1e-12  # linear in w
    v, dv = rng.standard_normal((S, 8)), rng.standard_normal((S, 8))
    for bnd in (None, 0, 3, 8):
        assert abs((oracle.value_shift(v, bnd) * dv).sum() - (v * oracle.value_shift_backward(dv, bnd)).sum()) < 1e-12
    r, dr = rng.standard_normal((S, 2 * d)), rng.standard_normal((S, 2 * d))
    assert abs((oracle.rope(r, 2, d, 10000.0) * dr).sum() - (r * oracle.rope_backward(dr, 2, d, 10000.0)).sum()) < 1e-12
