"""Pins of the float64 oracle against things other than itself.

Each test ties one oracle step to a library routine that computes the same
special case, a closed form, an invariant, or brute force on a tiny input,
chosen so that a dropped term, a wrong sign or index, or a transposed operand
fails at least one of them. Steps follow "Compressed Convolutional Attention"
(gist.science/es/paper/2510.04476, section 2).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import workloads

RNG = np.random.default_rng(1234)


def rand(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- seq conv --
@pytest.mark.parametrize("S,L,K", [(17, 6, 4), (3, 4, 4), (1, 2, 4), (9, 3, 1), (5, 2, 7)])
def test_seq_conv_equals_torch_depthwise_conv1d(S, L, K):
    """Causal depthwise conv == conv1d(groups=L, left pad K-1) cut to S (es 2.B item 1)."""
    z, w = rand(S, L), rand(L, K)
    ref = F.conv1d(torch.from_numpy(z.T[None]), torch.from_numpy(w[:, None, :]),
                   padding=K - 1, groups=L)[0, :, :S].T.numpy()
    np.testing.assert_allclose(oracle.seq_conv_causal(z, w), ref, rtol=1e-13, atol=1e-13)


def test_seq_conv_causal_and_local():
    S, L, K = 20, 5, 4
    z, w = rand(S, L), rand(L, K)
    base = oracle.seq_conv_causal(z, w)
    z2 = z.copy()
    z2[7] += 1.0
    out = oracle.seq_conv_causal(z2, w)
    assert np.array_equal(out[:7], base[:7])            # nothing before t=7 moves
    assert np.all(out[7:7 + K] != base[7:7 + K])         # taps reach K tokens ahead
    assert np.array_equal(out[7 + K:], base[7 + K:])      # and no further


def test_seq_conv_identity_and_lag():
    S, L, K = 12, 3, 4
    z = rand(S, L)
    w = np.zeros((L, K))
    w[:, K - 1] = 1.0                                      # current-token tap
    np.testing.assert_array_equal(oracle.seq_conv_causal(z, w), z)
    w = np.zeros((L, K))
    w[:, K - 3] = 2.0                                      # two steps back, x2
    expect = np.zeros_like(z)
    expect[2:] = 2.0 * z[:-2]
    np.testing.assert_array_equal(oracle.seq_conv_causal(z, w), expect)


# ------------------------------------------------------------ channel conv --
def test_channel_conv_equals_grouped_pointwise_conv1d():
    """Per-head d x d mix == conv1d(kernel 1, groups = heads) (es 2.B item 1)."""
    S, H, d = 7, 3, 4
    s, Wc = rand(S, H * d), rand(H, d, d)
    ref = F.conv1d(torch.from_numpy(s.T[None]), torch.from_numpy(Wc.reshape(H * d, d, 1)),
                   groups=H)[0].T.numpy()
    np.testing.assert_allclose(oracle.channel_conv(s, Wc, H, d), ref, rtol=1e-13, atol=1e-13)


def test_channel_conv_stays_within_head():
    S, H, d = 4, 3, 4
    s, Wc = rand(S, H * d), rand(H, d, d)
    s2 = s.copy()
    s2[:, d:2 * d] += 1.0  # touch head 1 only
    a, b = oracle.channel_conv(s, Wc, H, d), oracle.channel_conv(s2, Wc, H, d)
    assert np.array_equal(a[:, :d], b[:, :d]) and np.array_equal(a[:, 2 * d:], b[:, 2 * d:])
    eye = np.broadcast_to(np.eye(d), (H, d, d))
    np.testing.assert_array_equal(oracle.channel_conv(s, eye, H, d), s)


# ----------------------------------------------------------------- QK-mean --
def test_qk_mean_invariants_mha():
    """G=1: adding the shared mean keeps q-k and doubles q+k (es 2.B item 2)."""
    S, H, d = 5, 3, 4
    q, k = rand(S, H * d), rand(S, H * d)
    mq, mk = oracle.qk_mean(q, k, H, H, d)
    np.testing.assert_allclose((q + mq) - (k + mk), q - k, atol=1e-14)
    np.testing.assert_allclose((q + mq) + (k + mk), 2 * (q + k), atol=1e-14)


def test_qk_mean_invariants_gqa():
    """G>1: mean over a group's q heads minus k is kept; head differences scale by 3/2."""
    S, nq, nkv, d = 4, 6, 2, 3
    G = nq // nkv
    q, k = rand(S, nq * d), rand(S, nkv * d)
    mq, mk = oracle.qk_mean(q, k, nq, nkv, d)
    q2 = (q + mq).reshape(S, nkv, G, d)
    k2 = (k + mk).reshape(S, nkv, d)
    q1 = q.reshape(S, nkv, G, d)
    k1 = k.reshape(S, nkv, d)
    np.testing.assert_allclose(q2.mean(axis=2) - k2, q1.mean(axis=2) - k1, atol=1e-14)
    np.testing.assert_allclose(q2[:, :, 0] - q2[:, :, 2], 1.5 * (q1[:, :, 0] - q1[:, :, 2]), atol=1e-14)
    # query head h pairs with KV head h // G: moving k of group 1 leaves group 0 alone
    k_alt = k.copy()
    k_alt[:, d:] += 1.0
    mq_alt, _ = oracle.qk_mean(q, k_alt, nq, nkv, d)
    assert np.array_equal(mq_alt[:, :G * d], mq[:, :G * d])
    assert np.all(mq_alt[:, G * d:] != mq[:, G * d:])


# -------------------------------------------------------------------- RoPE --
def test_rope_worked_example_d2():
    """d=2: theta_0 = 1, so position t turns (1, 0) by t radians."""
    z = np.tile(np.array([[1.0, 0.0]]), (4, 1))
    out = oracle.rope(z, 1, 2, 10000.0)
    expect = np.array([[math.cos(t), math.sin(t)] for t in range(4)])
    np.testing.assert_allclose(out, expect, atol=1e-15)


def test_rope_equals_complex_rotation():
    """Rotate-half RoPE == multiply (x_i + i x_{i+d/2}) by exp(i t base^(-2i/d))."""
    S, H, d, base = 9, 2, 8, 10000.0
    z = rand(S, H * d)
    zc = z.reshape(S, H, d)
    c = zc[..., :d // 2] + 1j * zc[..., d // 2:]
    t = np.arange(S)[:, None, None]
    i = np.arange(d // 2)[None, None, :]
    rot = c * np.exp(1j * t * np.power(base, -2.0 * i / d))
    expect = np.concatenate([rot.real, rot.imag], axis=-1).reshape(S, H * d)
    np.testing.assert_allclose(oracle.rope(z, H, d, base), expect, atol=1e-12)


def test_rope_norm_relative_and_origin():
    S, d, base = 40, 16, 10000.0
    z = rand(S, d)
    out = oracle.rope(z, 1, d, base)
    half = d // 2
    np.testing.assert_allclose(out[:, :half] ** 2 + out[:, half:] ** 2,
                               z[:, :half] ** 2 + z[:, half:] ** 2, rtol=1e-12)
    np.testing.assert_array_equal(out[0], z[0])
    a, b = rand(d), rand(d)
    for m, n in ((5, 2), (31, 17), (39, 0)):
        ra = oracle.rope(a[None], 1, d, base, positions=np.array([m]))[0]
        rb = oracle.rope(b[None], 1, d, base, positions=np.array([n]))[0]
        rd = oracle.rope(a[None], 1, d, base, positions=np.array([m - n]))[0]
        assert abs(ra @ rb - rd @ b) < 1e-12


# ------------------------------------------------------------- value shift --
def test_value_shift_closed_form():
    """Half the value channels see the previous token, zero at t=0 (es 2.B item 3)."""
    S, L = 6, 8
    v = rand(S, L)
    out = oracle.value_shift(v)
    np.testing.assert_array_equal(out[:, :4], v[:, :4])
    np.testing.assert_array_equal(out[0, 4:], 0.0)
    np.testing.assert_array_equal(out[1:, 4:], v[:-1, 4:])
    assert oracle.value_shift(v[:1]).shape == (1, L)
    # a share of a wider block's V channels shifts from the wider block's half: boundary 0 shifts all,
    # L none, 3 the channels [3, L)
    np.testing.assert_array_equal(oracle.value_shift(v, 0)[1:], v[:-1])
    np.testing.assert_array_equal(oracle.value_shift(v, 0)[0], 0.0)
    np.testing.assert_array_equal(oracle.value_shift(v, L), v)
    b3 = oracle.value_shift(v, 3)
    np.testing.assert_array_equal(b3[:, :3], v[:, :3])
    np.testing.assert_array_equal(b3[1:, 3:], v[:-1, 3:])


# --------------------------------------------------------------- attention --
def _sdpa_gqa(q, k, v, nq, nkv, d, scale):
    S = q.shape[0]
    G = nq // nkv
    qt = torch.from_numpy(q.reshape(S, nq, d).transpose(1, 0, 2).copy())
    kt = torch.from_numpy(k.reshape(S, nkv, d).transpose(1, 0, 2).copy()).repeat_interleave(G, 0)
    vt = torch.from_numpy(v.reshape(S, nkv, d).transpose(1, 0, 2).copy()).repeat_interleave(G, 0)
    o = F.scaled_dot_product_attention(qt[None], kt[None], vt[None], is_causal=True, scale=scale)[0]
    return o.numpy().transpose(1, 0, 2).reshape(S, nq * d)


@pytest.mark.parametrize("S,nq,nkv,d", [(33, 2, 2, 8), (70, 4, 2, 16), (65, 8, 2, 4), (1, 2, 1, 4)])
def test_attention_equals_torch_sdpa(S, nq, nkv, d):
    """Causal MHA / GQA == torch SDPA(is_causal) with K/V heads repeated per group."""
    q, k, v = rand(S, nq * d), rand(S, nkv * d), rand(S, nkv * d)
    scale = 1.0 / math.sqrt(d)
    out = oracle.causal_attention(q, k, v, nq, nkv, d, scale, block=16)
    np.testing.assert_allclose(out, _sdpa_gqa(q, k, v, nq, nkv, d, scale), atol=1e-12)


def test_attention_brute_force_rows_and_probs():
    """Pure-Python softmax loop on a tiny case; rows sum to 1; causal zeros."""
    S, nq, nkv, d = 6, 2, 1, 3
    q, k, v = rand(S, nq * d), rand(S, nkv * d), rand(S, nkv * d)
    scale = 0.7
    out, probs = oracle.causal_attention(q, k, v, nq, nkv, d, scale, return_probs=True)
    for h in range(nq):
        for t in range(S):
            e = [math.exp(scale * sum(q[t, h * d + i] * k[s, i] for i in range(d))) for s in range(t + 1)]
            tot = sum(e)
            for i in range(d):
                ref = sum(e[s] / tot * v[s, i] for s in range(t + 1))
                assert abs(out[t, h * d + i] - ref) < 1e-12
    np.testing.assert_allclose(probs.sum(axis=2), 1.0, atol=1e-12)
    assert np.all(np.triu(probs[0], 1) == 0.0)
    sub = oracle.causal_attention(q, k, v, nq, nkv, d, scale, rows=[5, 0, 3])
    np.testing.assert_array_equal(sub, out[[5, 0, 3]])


def test_attention_flops_scale_with_compression():
    """Attention FLOPs fall by C at fixed E (es 2.A: attention cost / C)."""
    E, S, d = 2048, 16384, 128
    mha = oracle.attention_flops(1, S, E // d, d)
    for C in (1, 2, 4, 8):
        assert oracle.attention_flops(1, S, E // (C * d), d) * C == mha
    assert oracle.attention_flops(1, 16384, 4, 128) == 274877906944.0


# -------------------------------------------------------------- whole block --
def _small_shape(**kw):
    base = dict(name="t", batch=2, seq_len=21, hidden=48, n_q_heads=2, n_kv_heads=2,
                head_dim=8, conv_kernel=4, dtype="f32", seed=7)
    base.update(kw)
    return workloads.BlockShape(**base)


def _run(shape, inp, **kw):
    return oracle.cca_block(workloads.as_float64(inp), shape.n_q_heads, shape.n_kv_heads,
                            shape.head_dim, **kw)


def _rope_complex(z, H, d, base):
    S = z.shape[0]
    zc = z.reshape(S, H, d)
    c = zc[..., :d // 2] + 1j * zc[..., d // 2:]
    ang = np.arange(S)[:, None, None] * np.power(base, -2.0 * np.arange(d // 2) / d)[None, None, :]
    r = c * np.exp(1j * ang)
    return np.concatenate([r.real, r.imag], axis=-1).reshape(S, H * d)


@pytest.mark.parametrize("use_rope", [False, True])
@pytest.mark.parametrize("nq,nkv", [(4, 4), (4, 2)])
def test_block_reduces_to_plain_attention(use_rope, nq, nkv):
    """C=1, identity convs, no QK-mean, no shift: the block is plain causal MHA/GQA."""
    d = 8
    shape = _small_shape(hidden=nq * d, n_q_heads=nq, n_kv_heads=nkv, head_dim=d)
    inp = workloads.identity_convs(shape, workloads.make_inputs(shape))
    res = _run(shape, inp, qk_mean_mode=0, use_value_shift=False, use_rope=use_rope)
    f = workloads.as_float64(inp)
    for b in range(shape.batch):
        x = torch.from_numpy(f["x"][b])
        q = (x @ torch.from_numpy(f["W_q"]).T).numpy()
        k = (x @ torch.from_numpy(f["W_k"]).T).numpy()
        v = (x @ torch.from_numpy(f["W_v"]).T).numpy()
        if use_rope:
            q, k = _rope_complex(q, nq, d, 10000.0), _rope_complex(k, nkv, d, 10000.0)
        o = _sdpa_gqa(q, k, v, nq, nkv, d, 1.0 / math.sqrt(d))
        y = o @ f["W_o"].T
        np.testing.assert_allclose(res["y"][b], y, atol=1e-12)
        np.testing.assert_allclose(res["k_cache"][b].reshape(shape.seq_len, -1), k, atol=1e-12)


@pytest.mark.parametrize("mode", [0, 2])
def test_block_zero_convs_give_running_mean(mode):
    """Zero conv weights and no before-conv mean: q = k = 0, so every query attends
    uniformly and O[t] is the running mean of v over tokens 0..t."""
    shape = _small_shape(n_kv_heads=1)
    inp = workloads.make_inputs(shape)
    for name in ("convq_seq", "convk_seq"):
        inp[name] = torch.zeros_like(inp[name])
    res = _run(shape, inp, qk_mean_mode=mode)
    d = shape.head_dim
    for b in range(shape.batch):
        v = res["v_cache"][b].reshape(shape.seq_len, -1)
        run_mean = np.cumsum(v, axis=0) / np.arange(1, shape.seq_len + 1)[:, None]
        for h in range(shape.n_q_heads):
            np.testing.assert_allclose(res["o"][b][:, h * d:(h + 1) * d], run_mean, atol=1e-13)
        assert np.all(res["q"][b] == 0.0)


def test_block_pre_mean_only_with_zero_convs():
    """Zero convs, mode PRE, G=1, no RoPE: q = k = (q~ + k~)/2 exactly."""
    shape = _small_shape()
    inp = workloads.make_inputs(shape)
    for name in ("convq_seq", "convk_seq"):
        inp[name] = torch.zeros_like(inp[name])
    res = _run(shape, inp, qk_mean_mode=1, use_rope=False)
    avg = 0.5 * (res["q_lat"] + res["k_lat"])
    np.testing.assert_allclose(res["q"], avg, atol=1e-15)
    np.testing.assert_allclose(res["k_cache"].reshape(avg.shape), avg, atol=1e-15)


def test_block_identity_convs_closed_form():
    """Identity convs, PRE|POST, G=1, no RoPE: q = q~ + (q~ + k~), k = k~ + (q~ + k~)."""
    shape = _small_shape()
    inp = workloads.identity_convs(shape, workloads.make_inputs(shape))
    res = _run(shape, inp, qk_mean_mode=3, use_rope=False)
    tot = res["q_lat"] + res["k_lat"]
    np.testing.assert_allclose(res["q"], res["q_lat"] + tot, atol=1e-14)
    np.testing.assert_allclose(res["k_cache"].reshape(tot.shape), res["k_lat"] + tot, atol=1e-14)


def test_block_gqa_equals_cca_with_duplicated_kv():
    """CCGQA with QK-mean off == CCA whose K/V weights are copied per group (es 2.C)."""
    shape = _small_shape(n_q_heads=4, n_kv_heads=2, hidden=64)
    inp = workloads.make_inputs(shape)
    res = _run(shape, inp, qk_mean_mode=0)
    d, G = shape.head_dim, 2
    dup = dict(inp)
    wk = inp["W_k"].reshape(2, d, -1)
    dup["W_k"] = wk.repeat_interleave(G, 0).reshape(4 * d, -1)
    # value shift splits the latent in halves: duplicate V so the shifted half stays the shifted heads
    wv = inp["W_v"].reshape(2, d, -1)
    dup["W_v"] = wv.repeat_interleave(G, 0).reshape(4 * d, -1)
    dup["convk_seq"] = inp["convk_seq"].reshape(2, d, -1).repeat_interleave(G, 0).reshape(4 * d, -1)
    dup["convk_chan"] = inp["convk_chan"].repeat_interleave(G, 0)
    mha = oracle.cca_block(workloads.as_float64(dup), 4, 4, d, qk_mean_mode=0)
    np.testing.assert_allclose(res["y"], mha["y"], atol=1e-12)


def test_block_causality_and_value_shift_reach():
    """Perturbing x[t0] leaves every output before t0 exactly unchanged; in v only
    the current half at t0 and the shifted half at t0+1 move."""
    shape = _small_shape(n_kv_heads=2)
    inp = workloads.make_inputs(shape)
    base = _run(shape, inp)
    t0 = 9
    inp2 = dict(inp)
    x = inp["x"].clone()
    x[1, t0] += 0.5
    inp2["x"] = x
    res = _run(shape, inp2)
    for key in ("y", "k_cache", "v_cache", "q"):
        assert np.array_equal(res[key][1, :t0], base[key][1, :t0]), key
        assert np.array_equal(res[key][0], base[key][0]), key  # other sequence untouched
    v, vb = res["v_cache"][1].reshape(shape.seq_len, -1), base["v_cache"][1].reshape(shape.seq_len, -1)
    half = v.shape[1] // 2
    assert np.all(v[t0, :half] != vb[t0, :half]) and np.array_equal(v[t0, half:], vb[t0, half:])
    assert np.array_equal(v[t0 + 1, :half], vb[t0 + 1, :half]) and np.all(v[t0 + 1, half:] != vb[t0 + 1, half:])
    assert np.array_equal(v[t0 + 2:], vb[t0 + 2:])


def test_block_batch_permutation_and_rows():
    shape = _small_shape(batch=3)
    inp = workloads.make_inputs(shape)
    base = _run(shape, inp)
    perm = [2, 0, 1]
    inp2 = dict(inp)
    inp2["x"] = inp["x"][perm].contiguous()
    res = _run(shape, inp2)
    np.testing.assert_array_equal(res["y"], base["y"][perm])
    rows = [20, 0, 7]
    sub = _run(shape, inp, rows=rows)
    np.testing.assert_allclose(sub["y"], base["y"][:, rows], atol=1e-15)
    np.testing.assert_array_equal(sub["k_cache"], base["k_cache"])


def test_conv_state_is_tail_of_latents():
    shape = _small_shape(seq_len=2)
    res = _run(shape, workloads.make_inputs(shape))
    cs = res["conv_state_q"]
    assert cs.shape == (2, 3, shape.latent_q)
    np.testing.assert_array_equal(cs[:, 0], 0.0)
    np.testing.assert_array_equal(cs[:, 1:], res["q_lat"])
    np.testing.assert_array_equal(res["conv_state_v"][:, 0], res["v_lat"][:, -1])


# --------------------------------------------------------------- decode step --
@pytest.mark.parametrize("mode,vshift,rope_on,G", [(3, 1, 1, 2), (0, 0, 1, 2), (1, 1, 0, 1), (2, 0, 1, 4)])
def test_decode_step_continues_the_prefill(mode, vshift, rope_on, G):
    """A prefill of S tokens equals a prefill of S-1 tokens followed by one decode step from its
    state (KV cache and conv state): y, q, the new cache rows and the advanced conv state, at fp64."""
    nkv, d, S = 2, 8, 23
    sh = workloads.BlockShape("dec", 2, S, G * nkv * d * 2, G * nkv, nkv, d, 3, "f32", 7,
                              qk_mean_mode=mode, value_shift=vshift, use_rope=rope_on)
    inp = workloads.as_float64(workloads.make_inputs(sh))
    kw = dict(qk_mean_mode=mode, use_value_shift=bool(vshift), use_rope=bool(rope_on))
    full = oracle.cca_block(inp, G * nkv, nkv, d, **kw)
    head = dict(inp, x=inp["x"][:, :S - 1])
    pre = oracle.cca_block(head, G * nkv, nkv, d, **kw)
    K, Lq, Lkv = 3, G * nkv * d, nkv * d
    for b in range(2):
        state = np.concatenate([pre["conv_state_q"][b].reshape(-1), pre["conv_state_k"][b].reshape(-1),
                                pre["conv_state_v"][b].reshape(-1)])
        assert state.size == (K - 1) * (Lq + Lkv) + Lkv
        out = oracle.decode_step(inp, inp["x"][b, S - 1], pre["k_cache"][b], pre["v_cache"][b], state, S - 1,
                                 G * nkv, nkv, d, **kw)
        np.testing.assert_allclose(out["y"], full["y"][b, S - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(out["q"], full["q"][b, S - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(out["k"], full["k_cache"][b, S - 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(out["v"], full["v_cache"][b, S - 1], rtol=1e-11, atol=1e-12)
        full_state = np.concatenate([full["conv_state_q"][b].reshape(-1), full["conv_state_k"][b].reshape(-1),
                                     full["conv_state_v"][b].reshape(-1)])
        np.testing.assert_allclose(out["conv_state"], full_state, rtol=1e-14, atol=1e-15)  # same latents, to rounding


def test_decode_steps_chain_and_first_token():
    """Three decode steps after a prefill of S-3 tokens reproduce the last three rows of a prefill
    of S; one step from an empty cache and a zero conv state is a prefill of one token."""
    G, nkv, d, S = 2, 2, 8, 19
    sh = workloads.BlockShape("dec", 1, S, G * nkv * d * 2, G * nkv, nkv, d, 4, "f32", 8)
    inp = workloads.as_float64(workloads.make_inputs(sh))
    full = oracle.cca_block(inp, G * nkv, nkv, d)
    pre = oracle.cca_block(dict(inp, x=inp["x"][:, :S - 3]), G * nkv, nkv, d)
    kc = np.zeros((S, nkv, d))
    vc = np.zeros((S, nkv, d))
    kc[:S - 3] = pre["k_cache"][0]
    vc[:S - 3] = pre["v_cache"][0]
    state = np.concatenate([pre["conv_state_q"][0].reshape(-1), pre["conv_state_k"][0].reshape(-1),
                            pre["conv_state_v"][0].reshape(-1)])
    for t in range(S - 3, S):
        out = oracle.decode_step(inp, inp["x"][0, t], kc, vc, state, t, G * nkv, nkv, d)
        kc[t], vc[t], state = out["k"], out["v"], out["conv_state"]
        np.testing.assert_allclose(out["y"], full["y"][0, t], rtol=1e-11, atol=1e-12)
    one = oracle.cca_block(dict(inp, x=inp["x"][:, :1]), G * nkv, nkv, d)
    K, Lq, Lkv = 4, G * nkv * d, nkv * d
    out = oracle.decode_step(inp, inp["x"][0, 0], kc, vc, np.zeros((K - 1) * (Lq + Lkv) + Lkv), 0, G * nkv, nkv, d)
    np.testing.assert_allclose(out["y"], one["y"][0, 0], rtol=1e-11, atol=1e-12)


# ------------------------------------------------------ step composition --
# The pins above check each step alone; these fix how the block composes them
# (es 2.B item 1: the sequence conv, then the channel mix within the head;
# item 2: the QK-mean terms are taken on the latents before the convs and on
# the channel-mix output after them; es section 3 item 2 and 2.C: the cache
# holds k after RoPE). One sequence of 3 tokens, E = 2, one head of d = 2,
# K = 2, W_q = W_v = W_o = I, W_k = 2 I, so q~ = v~ = x and k~ = 2 x. The seq
# taps differ per channel (channel 0 reads only the previous token, channel 1
# only the current one) and the channel mixes are a shear and a swap, so that
# taking the two convs in the other order, or the mean on the seq-conv output,
# changes the result. Every expected value below is worked out by hand.
_COMP_X = [[1.0, 2.0], [3.0, 5.0], [7.0, 11.0]]
# hand-worked, seq conv first: s_q = (x[t-1,0], x[t,1]) = (0,2) (1,5) (3,11);
#   c_q = [[1,2],[0,1]] s_q = (s0 + 2 s1, s1)
_COMP_CQ = [[4.0, 2.0], [11.0, 5.0], [25.0, 11.0]]
# s_k = (2x[t-1,0], 2x[t,1]) = (0,4) (2,10) (6,22); c_k = swap(s_k)
_COMP_CK = [[4.0, 0.0], [10.0, 2.0], [22.0, 6.0]]


def _composition_inputs(S=3):
    eye = np.eye(2)
    return {
        "x": np.array([_COMP_X[:S]]),
        "W_q": eye.copy(), "W_k": 2.0 * eye, "W_v": eye.copy(), "W_o": eye.copy(),
        "convq_seq": np.array([[1.0, 0.0], [0.0, 1.0]]),      # [channel, tap]; tap 1 = current token
        "convk_seq": np.array([[1.0, 0.0], [0.0, 1.0]]),
        "convq_chan": np.array([[[1.0, 2.0], [0.0, 1.0]]]),   # out_i = sum_j W[i][j] in_j
        "convk_chan": np.array([[[0.0, 1.0], [1.0, 0.0]]]),
    }


def test_block_seq_conv_before_channel_mix():
    """No QK-mean, RoPE or shift: q and the cached k are c_q and c_k of the hand-worked
    sequence conv followed by the channel mix (the other order gives (5,2) (13,5) (29,11))."""
    res = oracle.cca_block(_composition_inputs(), 1, 1, 2, qk_mean_mode=0, use_value_shift=False,
                           use_rope=False)
    np.testing.assert_array_equal(res["q"][0], _COMP_CQ)
    np.testing.assert_array_equal(res["k_cache"][0].reshape(3, 2), _COMP_CK)


def test_block_post_mean_on_channel_mix_output():
    """POST only: q = c_q + (c_q + c_k)/2 and k = c_k + (c_q + c_k)/2, the mean taken on the
    channel-mix outputs. With the seq-conv outputs instead, q[0] would be (4, 5)."""
    res = oracle.cca_block(_composition_inputs(), 1, 1, 2, qk_mean_mode=2, use_value_shift=False,
                           use_rope=False)
    # c_q + c_k = (8,2) (21,7) (47,17)
    np.testing.assert_array_equal(res["q"][0], [[8.0, 3.0], [21.5, 8.5], [48.5, 19.5]])
    np.testing.assert_array_equal(res["k_cache"][0].reshape(3, 2), [[8.0, 1.0], [20.5, 5.5], [45.5, 14.5]])


def test_block_pre_and_post_mean_together():
    """PRE|POST: q = c_q + (q~ + k~)/2 + (c_q + c_k)/2 with q~ + k~ = 3x, the PRE term taken on
    the latents before any conv."""
    res = oracle.cca_block(_composition_inputs(), 1, 1, 2, qk_mean_mode=3, use_value_shift=False,
                           use_rope=False)
    # 1.5 x = (1.5,3) (4.5,7.5) (10.5,16.5)
    np.testing.assert_array_equal(res["q"][0], [[9.5, 6.0], [26.0, 16.0], [59.0, 36.0]])
    np.testing.assert_array_equal(res["k_cache"][0].reshape(3, 2), [[9.5, 4.0], [25.0, 13.0], [56.0, 31.0]])


def test_block_cache_holds_k_after_rope_and_shifted_v():
    """With RoPE (d = 2: theta_0 = 1, so token t turns by t radians) the cache holds the rotated
    c_k; v keeps channel 0 of token t and takes channel 1 from token t-1 (zero at t = 0); y at
    t = 0 is v[0] and at t = 1 a two-way softmax of the rotated q and k."""
    res = oracle.cca_block(_composition_inputs(), 1, 1, 2, qk_mean_mode=0, use_value_shift=True,
                           use_rope=True)

    def rot(a, b, t):
        return [a * math.cos(t) - b * math.sin(t), b * math.cos(t) + a * math.sin(t)]

    kc = res["k_cache"][0].reshape(3, 2)
    for t in range(3):
        np.testing.assert_allclose(kc[t], rot(*_COMP_CK[t], t), rtol=0, atol=1e-13)
    np.testing.assert_array_equal(res["v_cache"][0].reshape(3, 2), [[1.0, 0.0], [3.0, 2.0], [7.0, 5.0]])
    y = res["y"][0]
    np.testing.assert_allclose(y[0], [1.0, 0.0], atol=1e-15)
    q1 = rot(*_COMP_CQ[1], 1)
    k0, k1 = rot(*_COMP_CK[0], 0), rot(*_COMP_CK[1], 1)
    s0 = (q1[0] * k0[0] + q1[1] * k0[1]) / math.sqrt(2.0)
    s1 = (q1[0] * k1[0] + q1[1] * k1[1]) / math.sqrt(2.0)
    p1 = 1.0 / (1.0 + math.exp(s0 - s1))
    np.testing.assert_allclose(y[1], [(1 - p1) * 1.0 + p1 * 3.0, (1 - p1) * 0.0 + p1 * 2.0], rtol=1e-12)


@pytest.mark.parametrize("mode,expect_q,expect_k", [
    (0, [25.0, 11.0], [22.0, 6.0]),
    (2, [48.5, 19.5], [45.5, 14.5]),
    (3, [59.0, 36.0], [56.0, 31.0]),
])
def test_decode_step_composition_by_hand(mode, expect_q, expect_k):
    """The decode step of token 2 from the state of tokens 0..1 (conv state: q~[1] = (3,5),
    k~[1] = (6,10), v~[1] = (3,5)) gives the hand-worked row 2 above, without any prefill."""
    inp = _composition_inputs()
    state = np.array([3.0, 5.0, 6.0, 10.0, 3.0, 5.0])
    kc = np.array([[[4.0, 0.0]], [[10.0, 2.0]]])   # any cache rows: only y depends on them
    vc = np.array([[[1.0, 0.0]], [[3.0, 2.0]]])
    out = oracle.decode_step(inp, np.array(_COMP_X[2]), kc, vc, state, 2, 1, 1, 2, qk_mean_mode=mode,
                             use_value_shift=True, use_rope=False)
    np.testing.assert_array_equal(out["q"], expect_q)
    np.testing.assert_array_equal(out["k"].reshape(2), expect_k)
    np.testing.assert_array_equal(out["v"].reshape(2), [7.0, 5.0])
    np.testing.assert_array_equal(out["conv_state"], [7.0, 11.0, 14.0, 22.0, 7.0, 11.0])
