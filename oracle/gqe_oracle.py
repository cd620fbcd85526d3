"""Plain, slow CPU oracle for GQE (float64): causal prefill, decode and
append steps over a KV cache, the layer around them (projections, W_O) and
the backward pass.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py``; never by
the library.  It shares no code with the CUDA path: the only thing both sides
use is the seeded input generator in ``synth``, which holds none of the
method's arithmetic.

Sources (web pages; cited by title and section):

* [GQE review] "论文综述：分组查询专家——在 GQA 自注意力上引入混合专家"
  (review of *Grouped Query Experts*), §二 核心方法与创新: sub-sections
  "整体设计" (N heads, G groups, M = N/G experts), "路由器" (softmax then
  top-k), "输出怎么拼起来：三个关键部件" (hard-selected slots, renormalised
  weighted-sum slot, always-on shared head, concat feeding W_O).
* [GQE abstract] "Grouped Query Experts: Mixture-of-Experts on GQA
  Self-Attention" (1kpapers summary page), "01 In brief": 9 of 16 query
  attentions active.
* [GQA article] "AI 大模型之 GQA": §4.1 (KV bytes 2·L·G·d·S·b), §4.2 (the
  512 MiB / 2048 MiB worked value), "技术深化 分组查询的张量映射与权重转换"
  (head i reads KV head floor(i/(H/G)); explicit map vs logical repeat), and
  "工程实操 非方形因果遮罩与头分片检查" (causal mask on absolute positions).
* [MQA/GQA explainer] "MQA、GQA、稀疏/滑动窗口注意力及混合范式": the MQA and
  GQA numeric examples and the KV-cache byte examples.

Readings where the pages are silent:

* r_g is linear, ``l = x · W_r[g]`` (+ an optional per-(g, m) bias).
* Top-k is decided on the EXACT real-valued logits (softmax is strictly
  monotone, so this is the same as exact p); ties go to the lower expert
  index; the k selected experts are stored in rank order (slot j = rank).
* The weighted-sum slot is per group: ō_{i,g} = Σ_j w_{i,g,j} o_{i,g,j}.
* The shared head's query is the given Qs; it attends over KV head 0.
* Scale 1/sqrt(d), causal: key position <= query position (diagonal kept).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, the pages' worked values, brute force, invariants, central
finite differences for the gradients).
"""
from __future__ import annotations

import functools
import math
from typing import Optional, Tuple

import numpy as np

_U = 2.0 ** -53  # unit roundoff of float64


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values (finite, in bf16's normal range) to the nearest
    bf16, ties to even, in one step; returns the bit patterns.  bf16 keeps 8
    significant bits: with v = m * 2^e, 1/2 <= |m| < 1, the result is
    round_half_even(m * 2^8) * 2^(e - 8)."""
    m, e = np.frexp(np.asarray(v, dtype=np.float64))
    q = np.ldexp(np.round(m * 256.0), e - 8)  # np.round: halves to even
    return (q.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# small helpers kept separate so the pin tests can plant mistakes in them
# ---------------------------------------------------------------------------

def _kv_head_of(h: int, N: int, G: int) -> int:
    """[GQA article] 技术深化: query head i reads KV head floor(i / (H/G))."""
    return h // (N // G)


def _expert_head(g: int, m, M: int):
    """[GQE review] 整体设计: expert m of group g is query head g*M + m."""
    return g * M + m


def _scale(d: int) -> float:
    """[GQA article] 最小参考实现: scores are divided by sqrt(d)."""
    return 1.0 / math.sqrt(d)


def _visible(key_pos: np.ndarray, query_pos: np.ndarray, key_start=None) -> np.ndarray:
    """[GQA article] 工程实操 step 1: a key is visible iff key pos <= query pos.
    With padding (step 4) the causal condition is intersected with key
    validity: here the valid keys of a row are slots key_start..query pos."""
    vis = key_pos[None, :] <= query_pos[:, None]
    if key_start is not None:
        vis &= key_pos[None, :] >= key_start[:, None]
    return vis


# ---------------------------------------------------------------------------
# router
# ---------------------------------------------------------------------------

def _group_softmax(L: np.ndarray) -> np.ndarray:
    """[GQE review] 路由器: p_{i,g} = softmax(r_g(x_i)), over the group's M
    experts only (the last axis), in float64; the maximum is subtracted
    before exponentiating, which leaves the quotient unchanged."""
    mx = L.max(axis=-1, keepdims=True)
    e = np.exp(L - mx)
    return e / e.sum(axis=-1, keepdims=True)


def router_logits(x: np.ndarray, Wr: np.ndarray, bias: Optional[np.ndarray]
                  ) -> Tuple[np.ndarray, np.ndarray]:
    """Router logits l[t, g, m] = sum_j x[t, j] W_r[g, j, m] (+ bias[g, m]).

    [GQE review] 路由器: p_{i,g} = softmax(r_g(x_i)); r_g read as linear.
    Returns the float64 logits and a rigorous bound on their rounding error:
    every bf16*bf16 product is exact in float64, so a d_model-term sum plus the
    bias carries at most (d_model + 1) roundings of relative size 2^-53 of
    sum |x_j w_jm| + |bias| (any summation order).  The bound is doubled for
    the rounding of that magnitude itself.
    """
    T, dm = x.shape
    G, dm2, M = Wr.shape
    assert dm == dm2
    W2 = np.ascontiguousarray(Wr.transpose(1, 0, 2).reshape(dm, G * M))
    L = (x @ W2).reshape(T, G, M)
    A = (np.abs(x) @ np.abs(W2)).reshape(T, G, M)
    if bias is not None:
        b = np.asarray(bias, dtype=np.float64).reshape(1, G, M)
        L = L + b
        A = A + np.abs(b)
    err = 2.0 * (dm + 2) * _U * A
    return L, err


def exact_logits(x_row: np.ndarray, W_g: np.ndarray, bias_g: Optional[np.ndarray]
                 ) -> np.ndarray:
    """The M logits of one (token, group), each the exact sum of its float64
    products (exact for bf16 operands) and bias, correctly rounded to float64
    by ``math.fsum``."""
    M = W_g.shape[1]
    bias_g = np.zeros(M) if bias_g is None else np.asarray(bias_g, dtype=np.float64)
    return np.array([math.fsum((x_row * W_g[:, m]).tolist() + [float(bias_g[m])])
                     for m in range(M)])


def topk_exact_order(x_row: np.ndarray, W_g: np.ndarray, bias_g: Optional[np.ndarray]
                     ) -> list:
    """All M experts of one (token, group) ordered by EXACT logit, desc.

    Exact ties are broken towards the lower expert index.  The sign of
    l_a - l_b is taken from ``math.fsum`` over the exact float64 products
    (x_j * w_ja, -x_j * w_jb, bias_a, -bias_b): fsum returns the correctly
    rounded exact sum, so its sign is the sign of the exact difference.
    """
    M = W_g.shape[1]
    bias_g = np.zeros(M) if bias_g is None else np.asarray(bias_g, dtype=np.float64)
    prods = [(x_row * W_g[:, m]).tolist() for m in range(M)]

    def before(a: int, b: int) -> int:
        s = math.fsum(prods[a] + [-v for v in prods[b]] + [float(bias_g[a]), -float(bias_g[b])])
        if s > 0 or (s == 0 and a < b):
            return -1
        return 1

    return sorted(range(M), key=functools.cmp_to_key(before))


def route(x_bits: np.ndarray, Wr_bits: np.ndarray, bias: Optional[np.ndarray], k: int):
    """GQE router: logits -> softmax over the group's M experts -> top-k -> w.

    [GQE review] 路由器 and 三个关键部件 (renormalised weights
    w = p / sum_{m' in K_g} p).  x_bits [B,S,dm] and Wr_bits [G,dm,M] are bf16
    bit patterns.  Returns (topk_idx int32 [B,S,G,k] in rank order,
    p float64 [B,S,G,M], w float64 [B,S,G,k], n_exact) where n_exact counts
    the (token, group) pairs decided by the exact comparison.
    """
    B, S, dm = x_bits.shape
    G, _, M = Wr_bits.shape
    if not 1 <= k <= M:
        raise ValueError("need 1 <= k <= M")
    Wr = bf16_to_f64(Wr_bits)
    xb = np.asarray(x_bits).reshape(B * S, dm)
    # tokens are independent: evaluate them in blocks to bound memory
    blk = 1 << 16
    L = np.empty((B * S, G, M))
    err = np.empty((B * S, G, M))
    for t0 in range(0, B * S, blk):
        L[t0:t0 + blk], err[t0:t0 + blk] = router_logits(bf16_to_f64(xb[t0:t0 + blk]), Wr, bias)

    # candidate order from the float64 estimate (stable: lower index first)
    order = np.argsort(-L, axis=-1, kind="stable")
    Ls = np.take_along_axis(L, order, axis=-1)
    Es = np.take_along_axis(err, order, axis=-1)
    lo = Ls - Es
    hi = Ls + Es
    certain = np.ones(L.shape[:2], dtype=bool)
    for r in range(min(k, M - 1)):
        # rank r must be certainly above every later rank
        rest_hi = hi[..., r + 1:].max(axis=-1)
        certain &= lo[..., r] > rest_hi
    idx = order[..., :k].copy()

    unsure = np.argwhere(~certain)
    for t, g in unsure:
        xt = bf16_to_f64(xb[t])
        bg = None if bias is None else bias[g]
        ordr = topk_exact_order(xt, Wr[g], bg)
        idx[t, g] = ordr[:k]
        # where the float64 estimate cannot order the experts it cannot serve
        # the softmax either (products that cancel by far more than 2^53):
        # take the correctly rounded logits of this pair
        L[t, g] = exact_logits(xt, Wr[g], bg)

    p = _group_softmax(L)
    psel = np.take_along_axis(p, idx, axis=-1)
    den = np.zeros(psel.shape[:-1])
    for j in range(k):  # ascending slot order
        den = den + psel[..., j]
    w = psel / den[..., None]
    return (idx.reshape(B, S, G, k).astype(np.int32), p.reshape(B, S, G, M),
            w.reshape(B, S, G, k), int(len(unsure)))


# ---------------------------------------------------------------------------
# bucketing
# ---------------------------------------------------------------------------

def bucket(topk_idx: np.ndarray, M: int) -> Tuple[np.ndarray, np.ndarray]:
    """Stable per-(batch, group, expert) lists of token positions.

    For b, g, m in that order: the tokens i (ascending) whose selected set
    K_g(x_i) contains m ([GQE review] 路由器: only selected heads compute).
    Returns (bucket_off int64 [B*G*M+1] exclusive scan, bucket_tok int32).
    """
    B, S, G, k = topk_idx.shape
    off = [0]
    toks = []
    for b in range(B):
        for g in range(G):
            sel = topk_idx[b, :, g, :]
            for m in range(M):
                members = np.nonzero((sel == m).any(axis=-1))[0]
                toks.append(members.astype(np.int32))
                off.append(off[-1] + len(members))
    return np.asarray(off, dtype=np.int64), (np.concatenate(toks) if toks else
                                             np.zeros(0, np.int32))


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def causal_attention(q: np.ndarray, pos: np.ndarray, K: np.ndarray, V: np.ndarray,
                     dtype=np.float64, row_chunk: int = 0, key_start=None) -> np.ndarray:
    """Softmax attention of query rows at absolute positions ``pos``.

    o_r = sum_{t <= pos_r} softmax_t(q_r . K_t / sqrt(d)) V_t.
    [GQA article] 最小参考实现 (scaled dot product, softmax, times V) and
    工程实操 (mask by absolute position, not by a top-left triangle).  With
    ``key_start`` (one per row; padding, 工程实操 step 4) the sum runs over
    key_start_r <= t <= pos_r only.
    Rows are independent; they are processed in chunks only to bound memory.
    """
    q = np.asarray(q, dtype=dtype)
    K = np.asarray(K, dtype=dtype)
    V = np.asarray(V, dtype=dtype)
    pos = np.asarray(pos, dtype=np.int64)
    if key_start is not None:
        key_start = np.asarray(key_start, dtype=np.int64)
    R, d = q.shape
    out = np.empty((R, V.shape[1]), dtype=dtype)
    sc = dtype(_scale(d))
    if row_chunk <= 0:  # about 2^25 scores per block
        row_chunk = max(1, min(512, (1 << 25) // max(1, int(pos.max()) + 1)))
    for s in range(0, R, row_chunk):
        e = min(R, s + row_chunk)
        pm = int(pos[s:e].max())
        keys = np.arange(pm + 1)
        sco = (q[s:e] @ K[: pm + 1].T) * sc
        ks = None if key_start is None else key_start[s:e]
        sco = np.where(_visible(keys, pos[s:e], ks), sco, -np.inf)
        mx = sco.max(axis=1, keepdims=True)
        p = np.exp(sco - mx)
        out[s:e] = (p @ V[: pm + 1]) / p.sum(axis=1, keepdims=True)
    return out


def gqe_prefill(Q_bits, Qs_bits, K_bits, V_bits, topk_idx, w, dtype=np.float64):
    """Routed GQE causal prefill: selected heads, weighted-sum slot, shared head.

    [GQE review] 三个关键部件: O_i are the selected heads' outputs (slot j =
    rank j of the selection), ō_{i,g} = sum_j w_{i,g,j} o_{i,g,j}, and the
    always-on shared head s(x_i); the three are concatenated before W_O.
    Q [B,S,N,d], Qs [B,S,d], K/V [B,S,G,d] as bf16 bits.  Returns
    (O_sel [B,S,G,k,d], o_bar [B,S,G,d], s [B,S,d]).
    """
    B, S = Q_bits.shape[:2]
    O_sel, o_bar, s_out = gqe_prefill_rows(Q_bits, Qs_bits, K_bits, V_bits, topk_idx, w,
                                           rows=[np.arange(S)] * B, dtype=dtype)
    return np.stack(O_sel), np.stack(o_bar), np.stack(s_out)


def gqe_prefill_rows(Q_bits, Qs_bits, K_bits, V_bits, topk_idx, w, rows, dtype=np.float64):
    """Like :func:`gqe_prefill` but only for token positions ``rows[b]``.

    Returns three lists over b of arrays indexed by the requested rows.
    """
    B, S, N, d = Q_bits.shape
    G = K_bits.shape[2]
    M = N // G
    k = topk_idx.shape[-1]
    O_sel, o_bar, s_out = [], [], []
    for b in range(B):
        r = np.asarray(rows[b], dtype=np.int64)
        Kb = bf16_to_f64(K_bits[b])
        Vb = bf16_to_f64(V_bits[b])
        Ob = np.zeros((len(r), G, k, d), dtype=dtype)
        for g in range(G):
            for j in range(k):
                heads = _expert_head(g, topk_idx[b, r, g, j].astype(np.int64), M)
                q = bf16_to_f64(Q_bits[b, r, heads])
                Ob[:, g, j] = causal_attention(q, r, Kb[:, g], Vb[:, g], dtype=dtype)
        wb = np.asarray(w[b, r], dtype=dtype)
        ob = np.zeros((len(r), G, d), dtype=dtype)
        for j in range(k):  # ascending slot order
            ob = ob + wb[:, :, j, None] * Ob[:, :, j]
        sb = causal_attention(bf16_to_f64(Qs_bits[b, r]), r, Kb[:, 0], Vb[:, 0], dtype=dtype)
        O_sel.append(Ob)
        o_bar.append(ob)
        s_out.append(sb)
    return O_sel, o_bar, s_out


def gqe_decode_step(x_bits, Wr_bits, bias, Q_bits, Qs_bits, Kc_bits, Vc_bits, pos, k,
                    dtype=np.float64, kv_start=None):
    """One incremental decode step of GQE, for each sequence b of a batch.

    [GQA article] 工程实操 非方形因果遮罩: at an incremental decode step the query
    length is 1 and the key length is the whole history; the mask is taken on
    the query's absolute position.  The new token of sequence b sits at
    position pos[b]; its own K/V are already in the caches at that position
    (Kc, Vc [B, T, G, d] with T > pos[b]) and later slots are not visible.  It
    routes as in prefill ([GQE review] §二 路由器), each selected head attends
    with its group's KV head, the shared head with KV head 0, and ō is the
    weighted sum of the slots (三个关键部件).  x [B, dm], Q [B, N, d], Qs [B, d]
    are bf16 bit patterns.  ``kv_start`` [B] (padding, 工程实操 step 4: causal
    condition intersected with key validity) makes slots before kv_start[b]
    invalid: sequence b then sees slots kv_start[b]..pos[b].  Returns
    (topk_idx [B,G,k], p [B,G,M], w [B,G,k], O_sel [B,G,k,d], o_bar [B,G,d],
    s [B,d]).
    """
    B = x_bits.shape[0]
    idx, p, w, _ = route(np.asarray(x_bits)[:, None, :], Wr_bits, bias, k)
    idx, p, w = idx[:, 0], p[:, 0], w[:, 0]
    N, d = Q_bits.shape[1], Q_bits.shape[2]
    G = Kc_bits.shape[2]
    M = N // G
    O_sel = np.zeros((B, G, k, d), dtype=dtype)
    o_bar = np.zeros((B, G, d), dtype=dtype)
    s_out = np.zeros((B, d), dtype=dtype)
    for b in range(B):
        r = np.array([int(pos[b])])
        ks = None if kv_start is None else np.array([int(kv_start[b])])
        Kb, Vb = bf16_to_f64(Kc_bits[b]), bf16_to_f64(Vc_bits[b])
        for g in range(G):
            for j in range(k):
                h = _expert_head(g, int(idx[b, g, j]), M)
                q = bf16_to_f64(Q_bits[b, h])[None, :]
                O_sel[b, g, j] = causal_attention(q, r, Kb[:, g], Vb[:, g], dtype=dtype,
                                                  key_start=ks)[0]
        for j in range(k):  # ascending slot order
            o_bar[b] = o_bar[b] + np.asarray(w[b, :, j, None], dtype=dtype) * O_sel[b, :, j]
        s_out[b] = causal_attention(bf16_to_f64(Qs_bits[b])[None, :], r, Kb[:, 0], Vb[:, 0],
                                    dtype=dtype, key_start=ks)[0]
    return idx, p, w, O_sel, o_bar, s_out


def gqe_append_step(x_bits, Wr_bits, bias, Q_bits, Qs_bits, Kc_bits, Vc_bits, pos, k,
                    dtype=np.float64, kv_start=None):
    """n new tokens per sequence over a cache (short chunked prefill).

    [GQA article] 工程实操 非方形因果遮罩: Sq queries at the end of Sk keys;
    the mask is taken on absolute positions, so new token r of sequence b,
    at slot pos[b] + r, sees slots kv_start[b]..pos[b] + r (its own K/V and
    those of the earlier new tokens are already in the cache).  Each row is
    the decode step of its own token.  x [B, n, dm], Q [B, n, N, d],
    Qs [B, n, d]; returns the decode step's arrays with an n axis after B.
    """
    n = np.asarray(x_bits).shape[1]
    rows = [gqe_decode_step(x_bits[:, r], Wr_bits, bias, Q_bits[:, r], Qs_bits[:, r], Kc_bits,
                            Vc_bits, np.asarray(pos) + r, k, dtype=dtype, kv_start=kv_start)
            for r in range(n)]
    return tuple(np.stack([row[i] for row in rows], axis=1) for i in range(6))


def dense_gqa(Q_bits, K_bits, V_bits, dtype=np.float64, rows=None):
    """Dense GQA (every query head active), explicit head -> KV-head map.

    [GQA article] 最小参考实现 (first form: loop over heads, g = i // (H/G));
    [GQE review] §四: the all-active GQA baseline.  Returns O [B,S,N,d]
    (or [B][rows] lists when ``rows`` is given).
    """
    B, S, N, d = Q_bits.shape
    G = K_bits.shape[2]
    outs = []
    for b in range(B):
        r = np.arange(S) if rows is None else np.asarray(rows[b], dtype=np.int64)
        Kb = bf16_to_f64(K_bits[b])
        Vb = bf16_to_f64(V_bits[b])
        Ob = np.zeros((len(r), N, d), dtype=dtype)
        for h in range(N):
            g = _kv_head_of(h, N, G)
            Ob[:, h] = causal_attention(bf16_to_f64(Q_bits[b, r, h]), r, Kb[:, g], Vb[:, g],
                                        dtype=dtype)
        outs.append(Ob)
    return np.stack(outs) if rows is None else outs


def dense_gqa_repeat(Q_bits, K_bits, V_bits, dtype=np.float64):
    """Dense GQA by logical repeat of the KV heads (the second form).

    [GQA article] 最小参考实现: K and V repeated H/G times along the head axis,
    then one batched causal attention over all heads.  Only for small inputs.
    """
    B, S, N, d = Q_bits.shape
    G = K_bits.shape[2]
    Q = bf16_to_f64(Q_bits).astype(dtype)
    Kr = np.repeat(bf16_to_f64(K_bits), N // G, axis=2).astype(dtype)
    Vr = np.repeat(bf16_to_f64(V_bits), N // G, axis=2).astype(dtype)
    q = Q.transpose(0, 2, 1, 3)    # [B,N,S,d]
    kk = Kr.transpose(0, 2, 3, 1)  # [B,N,d,S]
    vv = Vr.transpose(0, 2, 1, 3)  # [B,N,S,d]
    sco = (q @ kk) * dtype(_scale(d))
    pos = np.arange(S)
    sco = np.where(_visible(pos, pos)[None, None], sco, -np.inf)
    p = np.exp(sco - sco.max(axis=-1, keepdims=True))
    o = (p @ vv) / p.sum(axis=-1, keepdims=True)
    return o.transpose(0, 2, 1, 3)


def kv_cache_bytes(L: int, G: int, S: int, d: int, b: int, B: int = 1) -> int:
    """[GQA article] §4.1: KV bytes per sequence = 2 * L * G * d * S * b (times B)."""
    return 2 * L * G * d * S * b * B


# ---------------------------------------------------------------------------
# the whole attention layer around the path (projections and W_O)
# ---------------------------------------------------------------------------

def gqe_layer_prefill(x_bits, Wq_bits, Wk_bits, Wv_bits, Ws_bits, Wr_bits, Wo_bits, bias, k):
    """GQE attention layer, causal prefill, from x to y.

    [GQE review] §二: the router picks k query heads per (token, group); only
    the selected query heads are computed at all, so their query projection
    runs for the selected (token, head) pairs only; the layer output is
    y_i = Concat(O_i, ō_i, s(x_i)) W_O.  The projections themselves are
    plain linear maps (the pages give them no special form):
      q_{i,h} = x_i W_Q[h] (selected h only), K_{i,g} = x_i W_K[g],
      V_{i,g} = x_i W_V[g], and the shared head's query x_i W_s.
    They are rounded to bf16, the element type the attention takes.
    Shapes: x [B,S,dm]; W_Q [N,dm,d]; W_K, W_V [G,dm,d]; W_s [dm,d];
    W_r [G,dm,M]; W_O [(G*k + G + 1)*d, dm], rows in concat order; all bf16
    bits.  Returns a dict with y [B,S,dm] (float64) and the intermediates
    (Q bits with unselected heads left zero, K, V, Qs bits, topk_idx, w,
    concat).
    """
    x = bf16_to_f64(x_bits)
    Wq, Wk, Wv = bf16_to_f64(Wq_bits), bf16_to_f64(Wk_bits), bf16_to_f64(Wv_bits)
    Ws, Wo = bf16_to_f64(Ws_bits), bf16_to_f64(Wo_bits)
    B, S, dm = x.shape
    N, _, d = Wq.shape
    G = Wk.shape[0]
    M = N // G
    idx, p, w, _ = route(x_bits, Wr_bits, bias, k)
    Q_bits = np.zeros((B, S, N, d), dtype=np.uint16)
    for g in range(G):
        for m in range(M):
            h = _expert_head(g, m, M)
            rows = np.nonzero((idx[:, :, g, :] == m).any(axis=-1))  # (b, i) that selected m
            if rows[0].size:
                Q_bits[rows[0], rows[1], h] = f64_to_bf16_bits(x[rows] @ Wq[h])
    K_bits = f64_to_bf16_bits(np.einsum("bsc,gcd->bsgd", x, Wk))
    V_bits = f64_to_bf16_bits(np.einsum("bsc,gcd->bsgd", x, Wv))
    Qs_bits = f64_to_bf16_bits(x @ Ws)
    O_sel, o_bar, s_out = gqe_prefill(Q_bits, Qs_bits, K_bits, V_bits, idx, w)
    concat = np.concatenate([O_sel.reshape(B, S, -1), o_bar.reshape(B, S, -1), s_out], axis=-1)
    return dict(y=concat @ Wo, Q=Q_bits, K=K_bits, V=V_bits, Qs=Qs_bits, topk_idx=idx, p=p,
                w=w, concat=concat)


# ---------------------------------------------------------------------------
# backward pass (gradients of the path's outputs), on float64 values
# ---------------------------------------------------------------------------

def causal_attention_backward(q, pos, K, V, dO):
    """Gradients of o_r = softmax_t(q_r . K_t / sqrt(d), t <= pos_r) V for one
    query head: returns (dq, dK, dV) for the upstream gradient dO.

    With S = q K^T / sqrt(d) (masked), P = softmax_rows(S), O = P V:
    dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
    dq = dS K / sqrt(d), dK = dS^T q / sqrt(d).  Rows of dS outside the mask
    are zero because P is.
    """
    q, K, V, dO = (np.asarray(a, dtype=np.float64) for a in (q, K, V, dO))
    pos = np.asarray(pos, dtype=np.int64)
    d = q.shape[1]
    sc = _scale(d)
    keys = np.arange(K.shape[0])
    s = np.where(_visible(keys, pos), (q @ K.T) * sc, -np.inf)
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    O = P @ V
    dV = P.T @ dO
    dP = dO @ V.T
    dS = P * (dP - (dO * O).sum(axis=1, keepdims=True))
    return (dS @ K) * sc, (dS.T @ q) * sc, dV


def gqe_prefill_values(Q, Qs, K, V, topk_idx, w):
    """:func:`gqe_prefill` on float64 values instead of bf16 bits (for
    finite-difference checks of the backward pass)."""
    Q, Qs, K, V, w = (np.asarray(a, dtype=np.float64) for a in (Q, Qs, K, V, w))
    B, S, N, d = Q.shape
    G = K.shape[2]
    M = N // G
    k = topk_idx.shape[-1]
    r = np.arange(S)
    O_sel = np.zeros((B, S, G, k, d))
    s_out = np.zeros((B, S, d))
    for b in range(B):
        for g in range(G):
            for j in range(k):
                heads = _expert_head(g, topk_idx[b, :, g, j].astype(np.int64), M)
                O_sel[b, :, g, j] = causal_attention(Q[b, r, heads], r, K[b, :, g], V[b, :, g])
        s_out[b] = causal_attention(Qs[b], r, K[b, :, 0], V[b, :, 0])
    o_bar = np.zeros((B, S, G, d))
    for j in range(k):
        o_bar = o_bar + w[:, :, :, j, None] * O_sel[:, :, :, j]
    return O_sel, o_bar, s_out


def gqe_prefill_backward(Q, Qs, K, V, topk_idx, w, dO_sel, do_bar, ds):
    """Gradients of the path's outputs (O_sel, ō, s) with respect to its
    inputs, for upstream gradients dO_sel [B,S,G,k,d], do_bar [B,S,G,d],
    ds [B,S,d].  Returns dict(dQ [B,S,N,d] (zero for heads a token did not
    select), dQs, dK, dV [B,S,G,d], dw [B,S,G,k]).

    [GQA article] 训练与部署 共享键值的梯度归约: each query head's attention
    backward is computed on its own, and dK, dV of a shared KV head are the
    SUM of the contributions of every head that reads it (here the selected
    routed heads of the group, plus the shared head for KV head 0); query
    gradients stay with their own head.  [GQE review] 三个关键部件: ō =
    sum_j w_j o_j, so slot j's output receives dO_sel_j + w_j dō and
    dw_j = <dō, o_j> -- the differentiable signal the weighted-sum slot
    gives the router.
    """
    Q, Qs, K, V, w = (np.asarray(a, dtype=np.float64) for a in (Q, Qs, K, V, w))
    B, S, N, d = Q.shape
    G = K.shape[2]
    M = N // G
    k = topk_idx.shape[-1]
    r = np.arange(S)
    dQ, dQs = np.zeros_like(Q), np.zeros_like(Qs)
    dK, dV = np.zeros_like(K), np.zeros_like(V)
    dw = np.zeros((B, S, G, k))
    for b in range(B):
        for g in range(G):
            for j in range(k):
                heads = _expert_head(g, topk_idx[b, :, g, j].astype(np.int64), M)
                q = Q[b, r, heads]
                o = causal_attention(q, r, K[b, :, g], V[b, :, g])
                dw[b, :, g, j] = (do_bar[b, :, g] * o).sum(axis=1)
                dO = dO_sel[b, :, g, j] + w[b, :, g, j, None] * do_bar[b, :, g]
                dq, dk, dv = causal_attention_backward(q, r, K[b, :, g], V[b, :, g], dO)
                dQ[b, r, heads] += dq
                dK[b, :, g] += dk
                dV[b, :, g] += dv
        dq, dk, dv = causal_attention_backward(Qs[b], r, K[b, :, 0], V[b, :, 0], ds[b])
        dQs[b] = dq
        dK[b, :, 0] += dk
        dV[b, :, 0] += dv
    return dict(dQ=dQ, dQs=dQs, dK=dK, dV=dV, dw=dw)


def router_values(x, Wr, bias, topk_idx):
    """Router p and w on float64 values for a FIXED selection topk_idx
    (the selection is discrete; gradients are taken with it held)."""
    x, Wr = np.asarray(x, dtype=np.float64), np.asarray(Wr, dtype=np.float64)
    l = np.einsum("bsc,gcm->bsgm", x, Wr)
    if bias is not None:
        l = l + np.asarray(bias, dtype=np.float64)
    p = np.exp(l - l.max(axis=-1, keepdims=True))
    p /= p.sum(axis=-1, keepdims=True)
    ps = np.take_along_axis(p, topk_idx.astype(np.int64), axis=-1)
    return p, ps / ps.sum(axis=-1, keepdims=True)


def router_backward(x, Wr, bias, topk_idx, dw, dp_extra=None):
    """Gradients through the router for upstream dw [B,S,G,k] (and an optional
    direct dp [B,S,G,M], e.g. from an auxiliary loss).  [GQE review] 路由器
    and 三个关键部件: w_j = p_{m_j} / sum_{j'} p_{m_j'} over the selected m_j,
    p = softmax(l), l = x W_r[g] (+ bias).  Returns dict(dlogits, dx, dWr,
    dbias).  At k = 1, w = 1 for any p, so dw carries no gradient.
    """
    x, Wr = np.asarray(x, dtype=np.float64), np.asarray(Wr, dtype=np.float64)
    p, w = router_values(x, Wr, bias, topk_idx)
    idx = topk_idx.astype(np.int64)
    ps_sum = np.take_along_axis(p, idx, axis=-1).sum(axis=-1, keepdims=True)
    dps = (dw - (dw * w).sum(axis=-1, keepdims=True)) / ps_sum  # d/dp of the selected ones
    dp = np.zeros_like(p)
    np.put_along_axis(dp, idx, dps, axis=-1)
    if dp_extra is not None:
        dp = dp + dp_extra
    dl = p * (dp - (dp * p).sum(axis=-1, keepdims=True))
    return dict(dlogits=dl, dx=np.einsum("bsgm,gcm->bsc", dl, Wr),
                dWr=np.einsum("bsc,bsgm->gcm", x, dl), dbias=dl.sum(axis=(0, 1)))


def load_balance_loss(p, topk_idx, alpha=1.0):
    """Auxiliary load-balancing loss and its gradient with respect to p.

    [GQE review] 为什么需要这些设计: training adds the standard MoE
    load-balancing loss against routing collapse; the pages give no formula.
    Reading: the Switch-Transformer form applied per group and averaged over
    groups, L = alpha * mean_g M * sum_m f_{g,m} * P_{g,m}, with f the share of
    the group's k*T selections that went to expert m (not differentiable) and
    P the mean router probability of m over the T = B*S tokens.  Returns
    (L, dL/dp [B,S,G,M]).
    """
    p = np.asarray(p, dtype=np.float64)
    B, S, G, M = p.shape
    T = B * S
    k = topk_idx.shape[-1]
    f = np.zeros((G, M))
    for g in range(G):
        f[g] = np.bincount(topk_idx[:, :, g, :].reshape(-1).astype(np.int64),
                           minlength=M)[:M] / (T * k)
    P = p.reshape(T, G, M).mean(axis=0)
    L = alpha * M * (f * P).sum(axis=1).mean()
    dp = np.broadcast_to(alpha * M * f / (G * T), p.shape).copy()
    return L, dp
