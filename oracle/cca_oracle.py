"""CPU float64 oracle of one CCA / CCGQA attention block (prefill forward).

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
CPU-baseline leg may import this module. The CUDA library never calls it and
shares no code with it.

Written from "Compressed Convolutional Attention: Efficient Attention in a
Compressed Latent Space" (gist.science/es/paper/2510.04476 and its French
twin gist.science/fr/paper/2510.04476). The pages print no equations, so the
exact form of each step is the plainest reading of their prose:

  1. down-projection of Q, K, V to a latent of width E/C  (es section 2.A;
     fr section 2, "Projection vers l'Espace Latent")
  2. QK-mean taken before the convolutions               (es 2.B item 2)
  3. causal depthwise convolution along the sequence     (es 2.B item 1)
  4. convolution across the channels of each head        (es 2.B item 1)
  5. QK-mean taken after the convolutions, and combine   (es 2.B item 2)
  6. RoPE applied directly in the latent                 (es section 3 item 2)
  7. value shift: half the value channels come from the previous token
                                                         (es 2.B item 3)
  8. causal softmax attention on the compressed heads, K/V heads shared by
     groups of query heads                               (es 2.A, 2.C)
  9. output projection back to width E (implied: the block's output is
     E wide and no up-projection happens before attention, es 2.A)
 10. one decode step (the same steps for one more token, es 1 item 2)
 11. the backward pass: the gradients of every input, the chain rule through
     steps 1-9 in reverse (es 4 reports the backward's speed; its form
     follows from the forward)

Readings where the pages are silent (each restated in the project notes):
  * no biases anywhere; no q/k normalisation or temperature;
  * seq conv: one filter of K taps per channel, cross-correlation, tap K-1
    multiplies the current token, zero padding before each sequence start;
  * channel conv: a dense d x d mix within each head (grouped pointwise conv);
  * QK-mean: both terms are added to the conv outputs. Query head h pairs with
    KV head g(h) = h // G; the key side uses the mean over its group's query
    heads. Mode bit0 adds the before-conv term, bit1 the after-conv term;
  * RoPE: rotate-half pairs (i, i + d/2), theta_i = base^(-2i/d), angle =
    position * theta_i, positions 0..S-1 within each sequence, all d dims;
  * value shift: latent channels [0, Lkv/2) keep the current token, channels
    [Lkv/2, Lkv) take the previous token, zero at the first token;
  * softmax scale 1/sqrt(d) unless given;
  * the KV cache holds k after RoPE and v after the shift.

Every function works on numpy float64 arrays and loops over nothing faster
than the definition needs. Library primitives used as steps: matmul, einsum,
exp, cos, sin.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

QK_MEAN_PRE = 1
QK_MEAN_POST = 2


# ---------------------------------------------------------------------------
# 1. Down-projection (es 2.A: Q, K, V projected to width E/C).
# ---------------------------------------------------------------------------
def down_project(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """Latent = x W^T. x: [S, E], W: [L, E] (torch Linear layout) -> [S, L]."""
    return x @ W.T


# ---------------------------------------------------------------------------
# 2./5. QK-mean (es 2.B item 2: the mean of q and k, before and after the
# convolution, is added to the resulting tensors).
# ---------------------------------------------------------------------------
def qk_mean(q: np.ndarray, k: np.ndarray, n_q: int, n_kv: int, d: int):
    """Per-token mean terms for the query and key sides.

    q: [S, n_q*d], k: [S, n_kv*d]. Query head h pairs with KV head h // G.
    Returns (mq [S, n_q*d], mk [S, n_kv*d]) with
      mq[t, h] = (q[t, h] + k[t, h//G]) / 2
      mk[t, g] = (mean over the group's query heads of q[t, .] + k[t, g]) / 2
    """
    S = q.shape[0]
    G = n_q // n_kv
    qh = q.reshape(S, n_q, d)
    kh = k.reshape(S, n_kv, d)
    mq = np.empty_like(qh)
    for h in range(n_q):
        mq[:, h, :] = 0.5 * (qh[:, h, :] + kh[:, h // G, :])
    mk = np.empty_like(kh)
    for g in range(n_kv):
        group_mean = qh[:, g * G:(g + 1) * G, :].mean(axis=1)
        mk[:, g, :] = 0.5 * (group_mean + kh[:, g, :])
    return mq.reshape(S, n_q * d), mk.reshape(S, n_kv * d)


# ---------------------------------------------------------------------------
# 3. Sequence convolution (es 2.B item 1: causal, as the convolutions that
# help SSMs like Mamba).
# ---------------------------------------------------------------------------
def seq_conv_causal(z: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Depthwise causal conv along the sequence.

    z: [S, L] one sequence, w: [L, K]. out[t, c] = sum_j w[c, j] * z[t-K+1+j, c]
    with z = 0 before the first token.
    """
    S, L = z.shape
    K = w.shape[1]
    out = np.zeros_like(z)
    for j in range(K):
        lag = K - 1 - j  # tap j reads the token `lag` steps back
        if lag == 0:
            out += w[:, j] * z
        elif lag < S:
            out[lag:] += w[:, j] * z[:-lag]
    return out


# ---------------------------------------------------------------------------
# 4. Channel convolution (es 2.B item 1: mixing along the channel dimension,
# within each head).
# ---------------------------------------------------------------------------
def channel_conv(s: np.ndarray, Wc: np.ndarray, n_heads: int, d: int) -> np.ndarray:
    """Dense d x d mix inside each head: out[t,h,i] = sum_j Wc[h,i,j] s[t,h,j]."""
    S = s.shape[0]
    sh = s.reshape(S, n_heads, d)
    return np.einsum("thj,hij->thi", sh, Wc).reshape(S, n_heads * d)


# ---------------------------------------------------------------------------
# 6. RoPE in the latent (es section 3 item 2; fr section 2).
# ---------------------------------------------------------------------------
def rope_angles(positions: np.ndarray, d: int, base: float) -> np.ndarray:
    """angle[t, i] = positions[t] * base^(-2i/d), i < d/2, in float64."""
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    return positions.astype(np.float64)[:, None] * theta[None, :]


def rope(z: np.ndarray, n_heads: int, d: int, base: float,
         positions: Optional[np.ndarray] = None) -> np.ndarray:
    """Rotate-half RoPE of every head: pair (i, i + d/2) turns by angle[t, i]."""
    S = z.shape[0]
    if positions is None:
        positions = np.arange(S)
    ang = rope_angles(positions, d, base)
    cos = np.cos(ang)[:, None, :]
    sin = np.sin(ang)[:, None, :]
    zh = z.reshape(S, n_heads, d)
    half = d // 2
    x1 = zh[:, :, :half]
    x2 = zh[:, :, half:]
    out = np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=2)
    return out.reshape(S, n_heads * d)


# ---------------------------------------------------------------------------
# 7. Value shift (es 2.B item 3: one kind of value from the current input and
# one from the previous input; half the heads cannot see the present token).
# ---------------------------------------------------------------------------
def value_shift(v: np.ndarray, boundary: Optional[int] = None) -> np.ndarray:
    """Channels [0, b) keep token t; channels [b, L) take token t-1 (0 at t=0), b = L/2 unless
    given (a block holding some of a wider block's KV groups shifts from the wider block's half)."""
    S, L = v.shape
    half = L // 2 if boundary is None else min(max(int(boundary), 0), L)
    out = v.copy()
    out[:, half:] = 0.0
    if S > 1:
        out[1:, half:] = v[:-1, half:]
    return out


# ---------------------------------------------------------------------------
# 8. Causal softmax attention on the compressed heads (es 2.A, 2.C).
# ---------------------------------------------------------------------------
def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, n_q: int, n_kv: int,
                     d: int, scale: float, rows: Optional[Sequence[int]] = None,
                     block: int = 256, return_probs: bool = False):
    """O[t, h] = sum_{s<=t} softmax_s(q[t,h].k[s,g(h)] * scale) v[s,g(h)].

    q: [S, n_q*d], k, v: [S, n_kv*d]. Exact (two-pass) softmax per row. Only
    the query rows in `rows` are computed (all rows by default); the result
    has one row per entry of `rows`. With return_probs the full probability
    matrices [n_q, len(rows), S] are returned too (small cases only).
    """
    S = q.shape[0]
    G = n_q // n_kv
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), n_q * d))
    probs = np.zeros((n_q, len(rows), S)) if return_probs else None
    for h in range(n_q):
        g = h // G
        qh = q[:, h * d:(h + 1) * d]
        kh = k[:, g * d:(g + 1) * d]
        vh = v[:, g * d:(g + 1) * d]
        for start in range(0, len(rows), block):
            r = rows[start:start + block]
            hi = int(r.max()) + 1
            scores = (qh[r] @ kh[:hi].T) * scale
            masked = np.arange(hi)[None, :] > r[:, None]
            scores[masked] = -np.inf
            scores -= scores.max(axis=1, keepdims=True)
            p = np.exp(scores)
            p /= p.sum(axis=1, keepdims=True)
            out[start:start + len(r), h * d:(h + 1) * d] = p @ vh[:hi]
            if return_probs:
                probs[h, start:start + len(r), :hi] = p
    if return_probs:
        return out, probs
    return out


# ---------------------------------------------------------------------------
# The whole block.
# ---------------------------------------------------------------------------
def default_scale(d: int, softmax_scale: float = 0.0) -> float:
    return softmax_scale if softmax_scale else 1.0 / math.sqrt(d)


def cca_block(inp: Dict[str, np.ndarray], n_q: int, n_kv: int, d: int, *,
              qk_mean_mode: int = 3, use_value_shift: bool = True,
              use_rope: bool = True, rope_base: float = 10000.0,
              softmax_scale: float = 0.0, rows: Optional[Sequence[int]] = None,
              return_probs: bool = False, value_shift_from: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Prefill forward of one block, per sequence, in float64.

    inp holds float64 arrays: x [B,S,E], W_q [Lq,E], W_k/W_v [Lkv,E],
    convq_seq [Lq,K], convq_chan [n_q,d,d], convk_seq [Lkv,K],
    convk_chan [n_kv,d,d], W_o [E,Lq].

    Returns y [B, R, E] for the R query rows in `rows` (all S by default),
    the KV cache k_cache / v_cache [B,S,n_kv,d], the conv state and every
    intermediate ([B,S,...]): q_lat, k_lat, v_lat, q (attention input),
    o [B,R,Lq].
    """
    x = inp["x"]
    B, S, E = x.shape
    Lq, Lkv = n_q * d, n_kv * d
    K = inp["convq_seq"].shape[1]
    scale = default_scale(d, softmax_scale)
    R = S if rows is None else len(rows)
    res = {name: [] for name in ("q_lat", "k_lat", "v_lat", "q", "k_cache", "v_cache",
                                 "o", "y", "conv_state_q", "conv_state_k", "conv_state_v")}
    probs_all = []
    for b in range(B):
        xb = x[b]
        q_lat = down_project(xb, inp["W_q"])
        k_lat = down_project(xb, inp["W_k"])
        v_lat = down_project(xb, inp["W_v"])

        mq_pre, mk_pre = qk_mean(q_lat, k_lat, n_q, n_kv, d)
        cq = channel_conv(seq_conv_causal(q_lat, inp["convq_seq"]), inp["convq_chan"], n_q, d)
        ck = channel_conv(seq_conv_causal(k_lat, inp["convk_seq"]), inp["convk_chan"], n_kv, d)
        mq_post, mk_post = qk_mean(cq, ck, n_q, n_kv, d)
        q = cq.copy()
        k = ck.copy()
        if qk_mean_mode & QK_MEAN_PRE:
            q += mq_pre
            k += mk_pre
        if qk_mean_mode & QK_MEAN_POST:
            q += mq_post
            k += mk_post
        if use_rope:
            q = rope(q, n_q, d, rope_base)
            k = rope(k, n_kv, d, rope_base)
        v = value_shift(v_lat, value_shift_from) if use_value_shift else v_lat.copy()

        att = causal_attention(q, k, v, n_q, n_kv, d, scale, rows=rows,
                               return_probs=return_probs)
        if return_probs:
            o, p = att
            probs_all.append(p)
        else:
            o = att
        y = o @ inp["W_o"].T

        # Conv state for a later decode step: the last K-1 pre-conv latents of
        # q and k and the last v latent (zero rows before the sequence start).
        def tail(z, n):
            st = np.zeros((n, z.shape[1]))
            take = min(n, S)
            if take:
                st[n - take:] = z[S - take:]
            return st
        res["conv_state_q"].append(tail(q_lat, K - 1))
        res["conv_state_k"].append(tail(k_lat, K - 1))
        res["conv_state_v"].append(tail(v_lat, 1))

        res["q_lat"].append(q_lat)
        res["k_lat"].append(k_lat)
        res["v_lat"].append(v_lat)
        res["q"].append(q)
        res["k_cache"].append(k.reshape(S, n_kv, d))
        res["v_cache"].append(v.reshape(S, n_kv, d))
        res["o"].append(o)
        res["y"].append(y)
    out = {k2: np.stack(v2) for k2, v2 in res.items()}
    assert out["y"].shape == (B, R, E)
    if return_probs:
        out["probs"] = np.stack(probs_all)
    return out


# ---------------------------------------------------------------------------
# 10. One decode step: the same steps as cca_block for one more token of one
# sequence, from the state a prefill of the earlier tokens leaves (the KV cache
# and the last K-1 pre-conv latents of q and k plus the last v latent; es 1
# item 2: the compressed cache is what decoding reads).
# ---------------------------------------------------------------------------
def decode_step(inp: Dict[str, np.ndarray], x_t: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                conv_state: np.ndarray, t: int, n_q: int, n_kv: int, d: int, *, qk_mean_mode: int = 3,
                use_value_shift: bool = True, use_rope: bool = True, rope_base: float = 10000.0,
                softmax_scale: float = 0.0) -> Dict[str, np.ndarray]:
    """Token t of one sequence. x_t [E]; k_cache, v_cache [>= t, n_kv, d] (rows 0..t-1 are read);
    conv_state [(K-1)*(Lq+Lkv) + Lkv]: the last K-1 rows of q~, then of k~, then the last row of v~
    (zero rows before the sequence start). Returns y [E], q [Lq], k [n_kv, d], v [n_kv, d] (the new
    cache rows) and the conv state advanced by this token."""
    Lq, Lkv = n_q * d, n_kv * d
    K = inp["convq_seq"].shape[1]
    q_lat = down_project(x_t[None, :], inp["W_q"])
    k_lat = down_project(x_t[None, :], inp["W_k"])
    v_lat = down_project(x_t[None, :], inp["W_v"])
    q_rows = conv_state[:(K - 1) * Lq].reshape(K - 1, Lq)
    k_rows = conv_state[(K - 1) * Lq:(K - 1) * (Lq + Lkv)].reshape(K - 1, Lkv)
    v_prev = conv_state[(K - 1) * (Lq + Lkv):]
    # the seq conv over the window of the K-1 earlier latents and this one, at its last row
    cq = channel_conv(seq_conv_causal(np.vstack([q_rows, q_lat]), inp["convq_seq"])[-1:], inp["convq_chan"], n_q, d)
    ck = channel_conv(seq_conv_causal(np.vstack([k_rows, k_lat]), inp["convk_seq"])[-1:], inp["convk_chan"], n_kv, d)
    mq_pre, mk_pre = qk_mean(q_lat, k_lat, n_q, n_kv, d)
    mq_post, mk_post = qk_mean(cq, ck, n_q, n_kv, d)
    q = cq.copy()
    k = ck.copy()
    if qk_mean_mode & QK_MEAN_PRE:
        q += mq_pre
        k += mk_pre
    if qk_mean_mode & QK_MEAN_POST:
        q += mq_post
        k += mk_post
    if use_rope:
        pos = np.array([t])
        q = rope(q, n_q, d, rope_base, positions=pos)
        k = rope(k, n_kv, d, rope_base, positions=pos)
    v = v_lat.copy()
    if use_value_shift:  # channels [Lkv/2, Lkv) from the previous token
        v[0, Lkv // 2:] = v_prev[Lkv // 2:]
    keys = np.vstack([k_cache[:t].reshape(t, Lkv), k])
    values = np.vstack([v_cache[:t].reshape(t, Lkv), v])
    q_all = np.zeros((t + 1, Lq))
    q_all[t] = q[0]
    o = causal_attention(q_all, keys, values, n_q, n_kv, d, default_scale(d, softmax_scale), rows=[t])
    y = o[0] @ inp["W_o"].T
    state = np.concatenate([np.vstack([q_rows, q_lat])[1:].reshape(-1), np.vstack([k_rows, k_lat])[1:].reshape(-1),
                            v_lat[0]])
    return {"y": y, "q": q[0], "k": k.reshape(n_kv, d), "v": v.reshape(n_kv, d), "conv_state": state}


def attention_flops(batch: int, seq_len: int, n_q: int, d: int) -> float:
    """Causal attention FLOPs, masked half excluded: 2 GEMMs x 2 flop/MAC x S^2/2."""
    return 2.0 * batch * n_q * seq_len * seq_len * d


def block_flops(batch: int, seq_len: int, hidden: int, n_q: int, n_kv: int, d: int) -> Dict[str, float]:
    """Dense FLOPs of the block's contractions."""
    T = batch * seq_len
    Lq, Lkv = n_q * d, n_kv * d
    return {
        "down_proj": 2.0 * T * hidden * (Lq + 2 * Lkv),
        "channel_conv": 2.0 * T * (Lq + Lkv) * d,
        "attention": attention_flops(batch, seq_len, n_q, d),
        "out_proj": 2.0 * T * Lq * hidden,
    }


# ---------------------------------------------------------------------------
# 11. The backward pass of the block (the gradients a training step needs; es section 4 reports a
# faster backward for CCGQA): given dL/dy, the gradients of L with respect to x and every weight, by
# the chain rule through the steps of cca_block taken in reverse. Attention uses the full probability
# matrix of each head (small cases only).
# ---------------------------------------------------------------------------
def qk_mean_adjoint(dmq: np.ndarray, dmk: np.ndarray, n_q: int, n_kv: int, d: int):
    """The transpose of (a, b) -> qk_mean(a, b): given the gradients of the two mean terms, the
    gradients of the query-side input a [S, n_q*d] and the key-side input b [S, n_kv*d]."""
    S = dmq.shape[0]
    G = n_q // n_kv
    dq = dmq.reshape(S, n_q, d)
    dk = dmk.reshape(S, n_kv, d)
    da = np.empty_like(dq)
    db = np.empty_like(dk)
    for h in range(n_q):
        da[:, h, :] = 0.5 * dq[:, h, :] + (0.5 / G) * dk[:, h // G, :]
    for g in range(n_kv):
        db[:, g, :] = 0.5 * dq[:, g * G:(g + 1) * G, :].sum(axis=1) + 0.5 * dk[:, g, :]
    return da.reshape(S, n_q * d), db.reshape(S, n_kv * d)


def seq_conv_backward(z: np.ndarray, w: np.ndarray, ds: np.ndarray):
    """Gradients of the causal depthwise conv s = seq_conv_causal(z, w) for the output gradient ds:
    (dz [S, L], dw [L, K])."""
    S, L = z.shape
    K = w.shape[1]
    dz = np.zeros_like(z)
    dw = np.zeros_like(w)
    for j in range(K):
        lag = K - 1 - j
        if lag == 0:
            dz += w[:, j] * ds
            dw[:, j] += (ds * z).sum(axis=0)
        elif lag < S:
            dz[:-lag] += w[:, j] * ds[lag:]
            dw[:, j] += (ds[lag:] * z[:-lag]).sum(axis=0)
    return dz, dw


def rope_backward(dz: np.ndarray, n_heads: int, d: int, base: float) -> np.ndarray:
    """The transpose of RoPE: each pair turns back by its angle."""
    S = dz.shape[0]
    return rope(dz, n_heads, d, base, positions=-np.arange(S))


def value_shift_backward(dv: np.ndarray, boundary: Optional[int] = None) -> np.ndarray:
    """The transpose of value_shift: the shifted channels' gradient moves one token back."""
    S, L = dv.shape
    half = L // 2 if boundary is None else min(max(int(boundary), 0), L)
    out = dv.copy()
    out[:, half:] = 0.0
    if S > 1:
        out[:-1, half:] = dv[1:, half:]
    return out


def cca_block_backward(inp: Dict[str, np.ndarray], dy: np.ndarray, n_q: int, n_kv: int, d: int, *,
                       qk_mean_mode: int = 3, use_value_shift: bool = True, use_rope: bool = True,
                       rope_base: float = 10000.0, softmax_scale: float = 0.0,
                       value_shift_from: Optional[int] = None) -> Dict[str, np.ndarray]:
    """dL/d(input) for L with dL/dy = dy [B, S, E], for every input of cca_block (same names and
    shapes), in float64."""
    x = inp["x"]
    B, S, E = x.shape
    G = n_q // n_kv
    scale = default_scale(d, softmax_scale)
    R = 1.0 if qk_mean_mode & QK_MEAN_PRE else 0.0
    P = 1.0 if qk_mean_mode & QK_MEAN_POST else 0.0
    grads = {k: np.zeros_like(v) for k, v in inp.items()}
    for b in range(B):
        xb = x[b]
        # forward, keeping what the backward needs
        q_lat = down_project(xb, inp["W_q"])
        k_lat = down_project(xb, inp["W_k"])
        v_lat = down_project(xb, inp["W_v"])
        s_q = seq_conv_causal(q_lat, inp["convq_seq"])
        s_k = seq_conv_causal(k_lat, inp["convk_seq"])
        c_q = channel_conv(s_q, inp["convq_chan"], n_q, d)
        c_k = channel_conv(s_k, inp["convk_chan"], n_kv, d)
        mq_pre, mk_pre = qk_mean(q_lat, k_lat, n_q, n_kv, d)
        mq_post, mk_post = qk_mean(c_q, c_k, n_q, n_kv, d)
        qa = c_q + R * mq_pre + P * mq_post
        ka = c_k + R * mk_pre + P * mk_post
        q = rope(qa, n_q, d, rope_base) if use_rope else qa
        k = rope(ka, n_kv, d, rope_base) if use_rope else ka
        v = value_shift(v_lat, value_shift_from) if use_value_shift else v_lat
        o, probs = causal_attention(q, k, v, n_q, n_kv, d, scale, return_probs=True)
        # output projection
        grads["W_o"] += dy[b].T @ o
        do = dy[b] @ inp["W_o"]
        # attention
        dq = np.zeros_like(q)
        dk = np.zeros_like(k)
        dv = np.zeros_like(v)
        for h in range(n_q):
            g = h // G
            p = probs[h]                        # [S, S], zero above the diagonal
            qh = q[:, h * d:(h + 1) * d]
            kh = k[:, g * d:(g + 1) * d]
            vh = v[:, g * d:(g + 1) * d]
            doh = do[:, h * d:(h + 1) * d]
            dv[:, g * d:(g + 1) * d] += p.T @ doh
            dp = doh @ vh.T
            dsc = p * (dp - (dp * p).sum(axis=1, keepdims=True))
            dq[:, h * d:(h + 1) * d] = scale * (dsc @ kh)
            dk[:, g * d:(g + 1) * d] += scale * (dsc.T @ qh)
        # value shift, RoPE
        dv_lat = value_shift_backward(dv, value_shift_from) if use_value_shift else dv
        dqa = rope_backward(dq, n_q, d, rope_base) if use_rope else dq
        dka = rope_backward(dk, n_kv, d, rope_base) if use_rope else dk
        # QK-mean terms: qa, ka depend on (q~, k~) through the PRE mean, on (c_q, c_k) directly and
        # through the POST mean
        da, db = qk_mean_adjoint(dqa, dka, n_q, n_kv, d)
        dc_q = dqa + P * da
        dc_k = dka + P * db
        dq_lat = R * da
        dk_lat = R * db
        # channel conv: c[t,h,i] = sum_j W[h,i,j] s[t,h,j]
        for name, dc, s, nh in (("convq_chan", dc_q, s_q, n_q), ("convk_chan", dc_k, s_k, n_kv)):
            grads[name] += np.einsum("thi,thj->hij", dc.reshape(S, nh, d), s.reshape(S, nh, d))
        ds_q = np.einsum("thi,hij->thj", dc_q.reshape(S, n_q, d), inp["convq_chan"]).reshape(S, n_q * d)
        ds_k = np.einsum("thi,hij->thj", dc_k.reshape(S, n_kv, d), inp["convk_chan"]).reshape(S, n_kv * d)
        # sequence conv
        dz_q, dwq = seq_conv_backward(q_lat, inp["convq_seq"], ds_q)
        dz_k, dwk = seq_conv_backward(k_lat, inp["convk_seq"], ds_k)
        grads["convq_seq"] += dwq
        grads["convk_seq"] += dwk
        dq_lat = dq_lat + dz_q
        dk_lat = dk_lat + dz_k
        # down-projection
        grads["W_q"] += dq_lat.T @ xb
        grads["W_k"] += dk_lat.T @ xb
        grads["W_v"] += dv_lat.T @ xb
        grads["x"][b] = dq_lat @ inp["W_q"] + dk_lat @ inp["W_k"] + dv_lat @ inp["W_v"]
    return grads
