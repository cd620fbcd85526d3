"""Pins for the CPU oracle: facts fixed by the pages or by mathematics.

Each ``check_*`` function raises AssertionError when the oracle is wrong.  The
``test_*`` functions run them; ``test_planted_*`` plant a plausible mistake in
one oracle helper (on the CPU) and require that some pin catches it.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import oracle.gqe_oracle as og
from synth import f32_to_bf16_bits, normal_bf16, bf16_bits_to_f32

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return f32_to_bf16_bits(np.asarray(a, dtype=np.float32))


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# KV-cache bytes (GQA article §4.1/§4.2; MQA/GQA explainer 数值示例)
# --------------------------------------------------------------------------

def check_kv_bytes():
    for c in _gold("kv_cache_bytes.json")["cases"]:
        got = oracle.kv_cache_bytes(c["L"], c["G"], c["S"], c["d"], c["b"])
        if "bytes" in c:
            assert got == c["bytes"], (c["cite"], got)
        if "MiB" in c:
            assert got == c["MiB"] * 2 ** 20, (c["cite"], got)


def test_kv_cache_bytes_pages():
    check_kv_bytes()


# --------------------------------------------------------------------------
# worked GQA / MQA examples (MQA/GQA explainer)
# --------------------------------------------------------------------------

def _example_tensors(ex):
    h, G, d = ex["h"], ex["G"], ex["d"]
    Q = np.asarray(ex["Q"], dtype=np.float32).reshape(1, 1, h, d)
    K = np.asarray(ex["K"], dtype=np.float32).reshape(1, 1, G, d)
    V = np.asarray(ex["V"], dtype=np.float32).reshape(1, 1, G, d)
    return _bits(Q), _bits(K), _bits(V)


def check_worked_examples():
    g = _gold("gqa_examples.json")
    for key in ("gqa", "mqa"):
        ex = g[key]
        Q, K, V = _example_tensors(ex)
        out = oracle.dense_gqa(Q, K, V)
        assert out.reshape(-1).tolist() == ex["expect_concat"], (ex["cite"], out.reshape(-1))
        # the scaled score of head 0 against its own KV head
        q0 = np.asarray(ex["Q"][0], float)
        k0 = np.asarray(ex["K"][0], float)
        s = float(q0 @ k0) * og._scale(ex["d"])
        assert abs(s - ex["expect_scaled_score"]) < 5e-5, (ex["cite"], s)


def test_worked_gqa_mqa_examples():
    check_worked_examples()


def check_worked_example_routed():
    """The GQA example through the routed path with k = M (every head selected)."""
    ex = _gold("gqa_examples.json")["gqa"]
    Q, K, V = _example_tensors(ex)
    M = ex["h"] // ex["G"]
    idx = np.tile(np.arange(M, dtype=np.int32), (1, 1, ex["G"], 1))  # [1,1,G,M]
    w = np.full((1, 1, ex["G"], M), 1.0 / M)
    Qs = _bits(np.zeros((1, 1, ex["d"])))
    O_sel, _, _ = oracle.gqe_prefill(Q, Qs, K, V, idx, w)
    assert O_sel.reshape(-1).tolist() == ex["expect_concat"]


def test_worked_example_routed():
    check_worked_example_routed()


def test_active_head_count():
    a = _gold("gqa_examples.json")["active_heads"]
    from synth import WORKLOADS
    w = WORKLOADS["layer250m"]
    assert (w.N, w.G, w.k) == (a["N"], a["G"], a["k"])
    assert w.G * w.k + 1 == a["active"]
    assert math.isclose(w.useful_flop_routed() / w.useful_flop_dense(), a["active"] / a["N"])


# --------------------------------------------------------------------------
# causal attention closed forms
# --------------------------------------------------------------------------

def check_geometric_scores():
    """Scores s_t = t (after the 1/sqrt(d) scale) and one-hot V give the
    softmax itself, whose closed form is a geometric series:
    o_t = e^t (e - 1) / (e^(P+1) - 1) for t <= P."""
    S, d = 12, 4
    q = np.zeros((S, d)); q[:, 0] = 2.0          # q . K_t = 2t, / sqrt(4) = t
    K = np.zeros((S, d)); K[:, 0] = np.arange(S)
    V = np.eye(S)
    pos = np.arange(S)
    o = oracle.causal_attention(q, pos, K, V)
    e = math.e
    for P in range(S):
        for t in range(S):
            want = (e ** t) * (e - 1) / (e ** (P + 1) - 1) if t <= P else 0.0
            assert abs(o[P, t] - want) < 1e-12, (P, t, o[P, t], want)


def test_geometric_closed_form():
    check_geometric_scores()


def check_nonsquare_positions():
    """Queries at absolute positions 5 and 6 over keys 0..6 see 6 and 7 keys."""
    c = _gold("gqa_examples.json")["nonsquare_causal"]
    n = c["n_keys"]
    q = np.ones((2, 8))
    K = np.ones((n, 8))        # identical keys: uniform weights over visible keys
    V = np.eye(n)
    o = oracle.causal_attention(q, np.asarray(c["query_pos"]), K, V)
    for r, nv in enumerate(c["visible"]):
        want = np.array([1.0 / nv] * nv + [0.0] * (n - nv))
        assert np.allclose(o[r], want, atol=1e-15, rtol=0), (r, o[r])


def test_nonsquare_causal_positions():
    check_nonsquare_positions()


def check_padding_key_validity():
    """[GQA article] 工程实操 step 4: with padding the visible keys are the
    intersection of the causal condition and key validity.  Identical keys
    make the weights uniform over exactly the visible slots, so the output is
    the mean of V over key_start..pos (one-hot V rows show which slots);
    key_start = pos leaves one key, whose V comes back exactly."""
    n = 9
    q = np.ones((4, 8))
    K = np.ones((n, 8))
    V = np.eye(n)
    pos = np.array([8, 8, 5, 3])
    start = np.array([0, 3, 5, 1])
    o = oracle.causal_attention(q, pos, K, V, key_start=start)
    for r in range(4):
        nv = pos[r] - start[r] + 1
        want = np.zeros(n)
        want[start[r]: pos[r] + 1] = 1.0 / nv
        assert np.allclose(o[r], want, atol=1e-15, rtol=0), (r, o[r])
    assert np.array_equal(o[2], V[5])


def test_padding_key_validity():
    check_padding_key_validity()


def test_left_padded_decode_equals_unpadded():
    """A sequence stored at cache slots s..s+n-1 behind s padding slots (any
    finite garbage there) decodes, with kv_start = s, exactly as the same
    sequence stored from slot 0."""
    B, n, s, N, G, k, d, dm = 2, 23, 7, 8, 4, 2, 16, 32
    x = normal_bf16((B, dm), 19200)
    W = normal_bf16((G, dm, N // G), 19201, std=dm ** -0.5)
    Q = normal_bf16((B, N, d), 19202)
    Qs = normal_bf16((B, d), 19203)
    K = normal_bf16((B, n, G, d), 19204)
    V = normal_bf16((B, n, G, d), 19205)
    pad = f32_to_bf16_bits(np.full((B, s, G, d), 2.5e3, np.float32))
    Kp, Vp = np.concatenate([pad, K], axis=1), np.concatenate([-pad, V], axis=1)
    pos = np.array([n - 1, 10])
    ref = oracle.gqe_decode_step(x, W, None, Q, Qs, K, V, pos, k)
    got = oracle.gqe_decode_step(x, W, None, Q, Qs, Kp, Vp, pos + s, k,
                                 kv_start=np.array([s, s]))
    for a_, b_ in zip(ref, got):
        assert np.allclose(a_, b_, rtol=1e-12, atol=1e-12)
    # without the validity bound the padding would be attended
    bad = oracle.gqe_decode_step(x, W, None, Q, Qs, Kp, Vp, pos + s, k)
    assert not np.allclose(bad[3], ref[3], atol=1e-3)


def check_head_to_kv_map():
    """8 query heads, 2 KV heads: heads 0-3 read KV 0, heads 4-7 read KV 1.
    KV heads are made numerically distinct (GQA article: make KV heads differ
    so a mapping bug shows); identical K rows make each output the prefix
    mean of its KV head's V."""
    c = _gold("gqa_examples.json")["nonsquare_causal"]
    H, G, S, d = c["H"], c["G"], 6, 4
    Q = np.ones((1, S, H, d), np.float32)
    K = np.ones((1, S, G, d), np.float32)
    V = np.zeros((1, S, G, d), np.float32)
    for g in range(G):
        V[0, :, g, :] = (np.arange(S)[:, None] + 1) * (10.0 ** g)
    out = oracle.dense_gqa(_bits(Q), _bits(K), _bits(V))
    for h in range(H):
        g = c["kv_of_head"][h]
        for i in range(S):
            want = np.mean(np.arange(1, i + 2)) * (10.0 ** g)
            assert np.allclose(out[0, i, h], want, rtol=1e-14), (h, i, out[0, i, h], want)


def test_head_to_kv_map():
    check_head_to_kv_map()


def check_row0_and_hull():
    rng = np.random.default_rng(0)
    S, d = 40, 16
    q = rng.standard_normal((S, d)); K = rng.standard_normal((S, d)); V = rng.standard_normal((S, d))
    o = oracle.causal_attention(q, np.arange(S), K, V)
    assert np.array_equal(o[0], V[0])            # row 0 sees only key 0
    for i in range(S):                           # convex combination of visible V
        assert np.all(o[i] <= V[: i + 1].max(0) + 1e-12)
        assert np.all(o[i] >= V[: i + 1].min(0) - 1e-12)
    Vc = np.tile(rng.standard_normal((1, d)), (S, 1))   # constant V -> constant output
    oc = oracle.causal_attention(q, np.arange(S), K, Vc)
    assert np.allclose(oc, Vc, rtol=0, atol=1e-14)


def test_row0_hull_constant_v():
    check_row0_and_hull()


def check_explicit_equals_repeat():
    """GQA article 最小参考实现: explicit head map and logical repeat agree
    (the page reports max_abs_error 0.0); KV heads are offset so they differ."""
    B, S, N, G, d = 2, 33, 8, 2, 16
    Q = normal_bf16((B, S, N, d), 11)
    K = bf16_bits_to_f32(normal_bf16((B, S, G, d), 12))
    V = bf16_bits_to_f32(normal_bf16((B, S, G, d), 13))
    for g in range(G):
        K[:, :, g] += 3.0 * g
        V[:, :, g] += 5.0 * g
    Kb, Vb = _bits(K), _bits(V)
    a = oracle.dense_gqa(Q, Kb, Vb)
    b = oracle.dense_gqa_repeat(Q, Kb, Vb)
    assert np.max(np.abs(a - b)) <= 1e-12, np.max(np.abs(a - b))


def test_explicit_equals_repeat():
    check_explicit_equals_repeat()


def test_fp32_variant_close_to_fp64():
    rng_bits = normal_bf16((1, 128, 16, 64), 21)
    K = normal_bf16((1, 128, 8, 64), 22)
    V = normal_bf16((1, 128, 8, 64), 23)
    a = oracle.dense_gqa(rng_bits, K, V, dtype=np.float64)
    b = oracle.dense_gqa(rng_bits, K, V, dtype=np.float32)
    rel = np.linalg.norm(a - b) / np.linalg.norm(a)
    assert rel < 1e-5, rel


# --------------------------------------------------------------------------
# router
# --------------------------------------------------------------------------

def _exact_logits(xb, Wb, bias):
    """Exact rational logits of bf16 inputs (independent of math.fsum)."""
    x = bf16_bits_to_f32(xb).astype(np.float64)
    W = bf16_bits_to_f32(Wb).astype(np.float64)
    B, S, dm = x.shape
    G, _, M = W.shape
    out = {}
    for b in range(B):
        for i in range(S):
            xs = [Fraction(float(v)) for v in x[b, i]]
            for g in range(G):
                for m in range(M):
                    v = sum((xs[j] * Fraction(float(W[g, j, m])) for j in range(dm)), Fraction(0))
                    if bias is not None:
                        v += Fraction(float(bias[g, m]))
                    out[(b, i, g, m)] = v
    return out


def check_topk_bruteforce(xb, Wb, bias, k):
    B, S, dm = xb.shape
    G, _, M = Wb.shape
    idx, p, w, _ = oracle.route(xb, Wb, bias, k)
    ex = _exact_logits(xb, Wb, bias)

    def beats(a, b, key):
        la, lb = ex[key + (a,)], ex[key + (b,)]
        return la > lb or (la == lb and a < b)

    for b in range(B):
        for i in range(S):
            for g in range(G):
                key = (b, i, g)
                valid = [set(c) for c in itertools.combinations(range(M), k)
                         if all(beats(a, o, key) for a in c for o in range(M) if o not in c)]
                assert len(valid) == 1, (key, valid)
                got = list(idx[b, i, g])
                assert set(got) == valid[0], (key, got, valid)
                for j in range(k - 1):      # slots in rank order
                    assert beats(got[j], got[j + 1], key), (key, got)
    return idx, p, w


def test_topk_bruteforce_random():
    dm, G, M = 16, 3, 4
    xb = normal_bf16((2, 9, dm), 31)
    Wb = normal_bf16((G, dm, M), 32, std=0.25)
    for k in (1, 2, 3, 4):
        check_topk_bruteforce(xb, Wb, None, k)


def test_topk_bruteforce_ties():
    """Duplicated W_r columns force exact ties; the lower index must win."""
    dm, G, M = 8, 2, 4
    vals = np.array([-2, -1, -0.5, 0, 0.5, 1, 2], np.float32)
    rng = np.random.default_rng(5)
    x = vals[rng.integers(0, len(vals), (1, 20, dm))]
    W = vals[rng.integers(0, len(vals), (G, dm, M))]
    W[:, :, 2] = W[:, :, 0]          # expert 2 ties expert 0 on every token
    W[1, :, 3] = W[1, :, 1]
    xb, Wb = _bits(x), _bits(W)
    for k in (1, 2, 3):
        idx, _, _ = check_topk_bruteforce(xb, Wb, None, k)
        # expert 2 can never rank above expert 0
        for t in range(20):
            got = list(idx[0, t, 0])
            if 2 in got:
                assert 0 in got and got.index(0) < got.index(2)


def test_topk_ties_with_bias_and_exact_path_used():
    dm, G, M = 8, 2, 2
    x = np.ones((1, 6, dm), np.float32)
    W = np.zeros((G, dm, M), np.float32)
    W[:, :, 0] = 0.25
    W[:, :, 1] = 0.125
    bias = np.array([[0.0, 1.0], [0.0, 1.5]], np.float32)  # group 0 exact tie, group 1 expert 1 wins
    idx, p, w, n_exact = oracle.route(_bits(x), _bits(W), bias, 1)
    assert (idx[0, :, 0, 0] == 0).all()      # tie -> lower index
    assert (idx[0, :, 1, 0] == 1).all()
    assert n_exact >= 6                      # the tie went through the exact comparison
    check_topk_bruteforce(_bits(x), _bits(W), bias, 1)


def check_router_sums():
    xb = normal_bf16((1, 64, 32), 41)
    Wb = normal_bf16((4, 32, 4), 42, std=0.2)
    for k in (1, 2, 4):
        idx, p, w, _ = oracle.route(xb, Wb, None, k)
        assert np.allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)
        assert np.allclose(w.sum(-1), 1.0, rtol=0, atol=1e-14)
        if k == 1:
            assert (w == 1.0).all()
        # top-1 is the arg-max of p
        assert (np.take_along_axis(p, idx[..., :1].astype(np.int64), -1)[..., 0]
                >= p.max(-1) - 1e-15).all()


def test_router_sums():
    check_router_sums()


def _exact_logit(x_row, w_col, bias=0.0):
    """The exact logit sum_j x_j w_j + bias as a Fraction (bf16 values and a
    float32 bias are exact binary fractions)."""
    return sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(x_row, w_col)),
               Fraction(float(bias)))


def check_router_p_values():
    """p = softmax of the group's logits ([GQE review] 路由器), pinned by facts
    the test derives without a softmax of its own:
    (a) two experts whose exact logit gap is D: p_0 = 1 / (1 + e^-D), the
        logistic function;
    (b) identical W_r columns: every expert gets exactly 1/M;
    (c) x = 0 and bias b_m = ln(m + 1): p_m = (m + 1) / 10 (up to the float32
        rounding of the logarithms), in every group;
    (d) random logits with a bias: log p_a - log p_b is the exact logit
        difference l_a - l_b."""
    # (a) M = 2: the logistic closed form
    xb = normal_bf16((1, 24, 16), 51)
    Wb = normal_bf16((3, 16, 2), 52, std=0.3)
    _, p, _, _ = oracle.route(xb, Wb, None, 1)
    xf = bf16_bits_to_f32(xb).astype(np.float64)[0]
    Wf = bf16_bits_to_f32(Wb).astype(np.float64)
    for t in range(24):
        for g in range(3):
            D = float(_exact_logit(xf[t], Wf[g][:, 0]) - _exact_logit(xf[t], Wf[g][:, 1]))
            want = 1.0 / (1.0 + math.exp(-D))
            assert abs(p[0, t, g, 0] - want) <= 1e-14, (t, g, p[0, t, g, 0], want)
            assert abs(p[0, t, g, 1] - (1.0 - want)) <= 1e-14, (t, g)
    # (b) M = 4 identical columns: 1/M exactly, w = 1/k exactly
    Wb4 = np.repeat(normal_bf16((2, 16, 1), 53, std=0.3), 4, axis=2)
    for k in (1, 2, 4):
        _, p4, w4, _ = oracle.route(xb, Wb4, None, k)
        assert (p4 == 0.25).all(), p4.min()
        assert (w4 == 1.0 / k).all()
    # (c) logits = bias = ln(m + 1): p proportional to m + 1
    zero = np.zeros((1, 8, 16), np.uint16)
    bias = np.tile(np.log(np.arange(1, 5, dtype=np.float64)).astype(np.float32), (2, 1))
    _, pc, _, _ = oracle.route(zero, Wb4, bias, 1)
    assert np.abs(pc - np.array([0.1, 0.2, 0.3, 0.4])).max() <= 1e-6, pc[0, 0]
    # (d) log-ratios are the exact logit differences (bias included)
    Wr = normal_bf16((2, 16, 3), 54, std=0.5)
    br = np.array([[0.75, -1.25, 0.0], [2.5, 0.5, -0.375]], np.float32)
    _, pd, _, _ = oracle.route(xb[:, :8], Wr, br, 1)
    Wrf = bf16_bits_to_f32(Wr).astype(np.float64)
    for t in range(8):
        for g in range(2):
            ls = [_exact_logit(xf[t], Wrf[g][:, m], br[g, m]) for m in range(3)]
            for a, b in ((0, 1), (0, 2), (1, 2)):
                got = math.log(pd[0, t, g, a]) - math.log(pd[0, t, g, b])
                assert abs(got - float(ls[a] - ls[b])) <= 1e-12, (t, g, a, b)


def test_router_p_values():
    check_router_p_values()


# --------------------------------------------------------------------------
# buckets
# --------------------------------------------------------------------------

def check_buckets(idx, M):
    B, S, G, k = idx.shape
    off, tok = oracle.bucket(idx, M)
    assert off[0] == 0 and off[-1] == B * G * S * k == len(tok)
    # brute force: walk tokens in order and append
    lists = {(b, g, m): [] for b in range(B) for g in range(G) for m in range(M)}
    for b in range(B):
        for i in range(S):
            for g in range(G):
                for j in range(k):
                    lists[(b, g, int(idx[b, i, g, j]))].append(i)
    n = 0
    for b in range(B):
        for g in range(G):
            for m in range(M):
                bi = (b * G + g) * M + m
                seg = tok[off[bi]:off[bi + 1]].tolist()
                assert seg == lists[(b, g, m)], (b, g, m)
                assert all(seg[a] < seg[a + 1] for a in range(len(seg) - 1))
                n += len(seg)
    assert n == B * G * S * k


def test_router_p_from_exact_logits_under_cancellation():
    """Products spanning ~190 binary orders cancel far below float64's reach:
    the selection comes from exact arithmetic, and so must p (softmax of the
    logits, [GQE review] 路由器).  Checked against logits summed in Fractions:
    the selected expert is the exact argmax, its p is the largest and the
    weights are finite."""
    rng = np.random.default_rng(11)
    S, dm, G, M = 64, 64, 2, 4
    mags = np.array([2.0 ** -90, 2.0 ** -40, 1.0, 2.0 ** 30, 2.0 ** 60])
    x = (mags[rng.integers(0, 5, (1, S, dm))] * rng.choice([-1, 1], (1, S, dm))).astype(np.float32)
    W = (mags[rng.integers(0, 5, (G, dm, M))] * rng.choice([-1, 1], (G, dm, M)) * 2.0 ** -20
         ).astype(np.float32)
    xb, Wb = f32_to_bf16_bits(x), f32_to_bf16_bits(W)
    idx, p, w, n_exact = oracle.route(xb, Wb, None, 1)
    assert n_exact > 0 and np.isfinite(w).all() and np.isfinite(p).all()
    xf, Wf = og.bf16_to_f64(xb)[0], og.bf16_to_f64(Wb)
    for t in range(S):
        for g in range(G):
            exact = [sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], Wf[g][:, m]))
                     for m in range(M)]
            best = max(range(M), key=lambda m: (exact[m], -m))
            assert idx[0, t, g, 0] == best
            assert p[0, t, g, best] == p[0, t, g].max()


def _decode_case(seed):
    B, S, N, G, k, d, dm = 2, 40, 8, 4, 2, 16, 32
    return (B, S, N, G, k, d, dm), dict(
        x=normal_bf16((B, S, dm), seed), W_r=normal_bf16((G, dm, N // G), seed + 1, std=dm ** -0.5),
        Q=normal_bf16((B, S, N, d), seed + 2), Qs=normal_bf16((B, S, d), seed + 3),
        K=normal_bf16((B, S, G, d), seed + 4), V=normal_bf16((B, S, G, d), seed + 5))


def test_decode_step_equals_prefill_row():
    """A decode step at position t over the caches of the first t+1 tokens is
    prefill's row t: the same routing, slots, weighted sum and shared head."""
    (B, S, N, G, k, d, dm), c = _decode_case(19000)
    idx, p, w, _ = oracle.route(c["x"], c["W_r"], None, k)
    O_sel, o_bar, s = oracle.gqe_prefill(c["Q"], c["Qs"], c["K"], c["V"], idx, w)
    for pos in ([0, 0], [17, 39], [39, 5]):
        b_ = np.arange(B)
        t = np.array(pos)
        di, dp, dw, dO, dob, ds = oracle.gqe_decode_step(
            c["x"][b_, t], c["W_r"], None, c["Q"][b_, t], c["Qs"][b_, t], c["K"], c["V"], t, k)
        assert np.array_equal(di, idx[b_, t])
        assert np.allclose(dp, p[b_, t], rtol=0, atol=1e-15)
        assert np.allclose(dO, O_sel[b_, t], rtol=1e-12, atol=1e-12)
        assert np.allclose(dob, o_bar[b_, t], rtol=1e-12, atol=1e-12)
        assert np.allclose(ds, s[b_, t], rtol=1e-12, atol=1e-12)


def test_decode_step_ignores_later_cache_slots_and_position0():
    """Slots after the query's position are invisible (garbage there changes
    nothing); at position 0 every head returns V[0] of its KV head exactly."""
    (B, S, N, G, k, d, dm), c = _decode_case(19100)
    t = np.array([0, 11])
    b_ = np.arange(B)
    args = (c["x"][b_, t], c["W_r"], None, c["Q"][b_, t], c["Qs"][b_, t])
    ref = oracle.gqe_decode_step(*args, c["K"], c["V"], t, k)
    K2, V2 = c["K"].copy(), c["V"].copy()
    for b in range(B):
        K2[b, t[b] + 1:] = f32_to_bf16_bits(np.full(K2[b, t[b] + 1:].shape, 3.0e4, np.float32))
        V2[b, t[b] + 1:] = f32_to_bf16_bits(np.full(V2[b, t[b] + 1:].shape, -7.0e3, np.float32))
    got = oracle.gqe_decode_step(*args, K2, V2, t, k)
    for a_, b2 in zip(ref, got):
        assert np.array_equal(a_, b2)
    V0 = og.bf16_to_f64(c["V"][0, 0])          # [G, d]
    assert np.array_equal(ref[3][0], np.repeat(V0[:, None, :], k, axis=1))
    assert np.array_equal(ref[5][0], V0[0])


def test_bucket_bruteforce():
    xb = normal_bf16((3, 50, 16), 51)
    Wb = normal_bf16((4, 16, 4), 52, std=0.3)
    for k in (1, 2, 4):
        idx, _, _, _ = oracle.route(xb, Wb, None, k)
        check_buckets(idx, 4)


def test_bucket_empty_expert():
    idx = np.zeros((1, 10, 2, 1), np.int32)   # expert 1 never chosen
    off, tok = oracle.bucket(idx, 2)
    assert off.tolist() == [0, 10, 10, 20, 20]
    check_buckets(idx, 2)


# --------------------------------------------------------------------------
# routed prefill
# --------------------------------------------------------------------------

def _small_problem(B=2, S=40, N=8, G=4, d=16, dm=16, seed=60):
    return dict(
        x=normal_bf16((B, S, dm), seed), Wr=normal_bf16((G, dm, N // G), seed + 1, std=0.25),
        Q=normal_bf16((B, S, N, d), seed + 2), Qs=normal_bf16((B, S, d), seed + 3),
        K=normal_bf16((B, S, G, d), seed + 4), V=normal_bf16((B, S, G, d), seed + 5))


def check_routed_kM_equals_dense():
    P = _small_problem()
    N, G = P["Q"].shape[2], P["K"].shape[2]
    M = N // G
    idx, p, w, _ = oracle.route(P["x"], P["Wr"], None, M)
    O_sel, _, s = oracle.gqe_prefill(P["Q"], P["Qs"], P["K"], P["V"], idx, w)
    dense = oracle.dense_gqa(P["Q"], P["K"], P["V"])
    B, S = P["Q"].shape[:2]
    for b in range(B):
        for i in range(S):
            for g in range(G):
                for j in range(M):
                    h = g * M + int(idx[b, i, g, j])
                    assert np.array_equal(O_sel[b, i, g, j], dense[b, i, h]), (b, i, g, j)


def test_routed_kM_equals_dense():
    check_routed_kM_equals_dense()


def check_shared_head_is_dense_head_on_kv0():
    P = _small_problem(seed=70)
    idx, p, w, _ = oracle.route(P["x"], P["Wr"], None, 1)
    _, _, s = oracle.gqe_prefill(P["Q"], P["Qs"], P["K"], P["V"], idx, w)
    B, S, d = P["Qs"].shape
    # a single-head, single-KV-head dense GQA over (Qs, K[:, :, 0], V[:, :, 0])
    ref = oracle.dense_gqa(P["Qs"].reshape(B, S, 1, d), P["K"][:, :, :1], P["V"][:, :, :1])
    assert np.array_equal(s, ref[:, :, 0])


def test_shared_head_kv0():
    check_shared_head_is_dense_head_on_kv0()


def check_k1_obar():
    P = _small_problem(seed=80)
    idx, p, w, _ = oracle.route(P["x"], P["Wr"], None, 1)
    assert (w == 1.0).all()
    O_sel, o_bar, _ = oracle.gqe_prefill(P["Q"], P["Qs"], P["K"], P["V"], idx, w)
    assert np.array_equal(o_bar, O_sel[:, :, :, 0])


def test_k1_weights_and_obar():
    check_k1_obar()


def check_obar_weighted_sum_k2():
    """ō with k=2 is the w-weighted sum of the two selected heads, each of
    which equals the dense output of that head."""
    P = _small_problem(seed=90)
    idx, p, w, _ = oracle.route(P["x"], P["Wr"], None, 2)
    O_sel, o_bar, _ = oracle.gqe_prefill(P["Q"], P["Qs"], P["K"], P["V"], idx, w)
    dense = oracle.dense_gqa(P["Q"], P["K"], P["V"])
    M = P["Q"].shape[2] // P["K"].shape[2]
    b, i, g = 1, 17, 2
    want = sum(w[b, i, g, j] * dense[b, i, g * M + idx[b, i, g, j]] for j in range(2))
    assert np.allclose(o_bar[b, i, g], want, rtol=1e-14, atol=1e-15)
    # w is p restricted to the selection, renormalised
    ps = p[b, i, g, idx[b, i, g]]
    assert np.allclose(w[b, i, g], ps / ps.sum(), rtol=1e-15)


def test_obar_weighted_sum_k2():
    check_obar_weighted_sum_k2()


def test_rows_subset_matches_full():
    P = _small_problem(seed=100)
    idx, p, w, _ = oracle.route(P["x"], P["Wr"], None, 2)
    full = oracle.gqe_prefill(P["Q"], P["Qs"], P["K"], P["V"], idx, w)
    rows = [np.array([0, 5, 39]), np.array([3, 38])]
    sub = oracle.gqe_prefill_rows(P["Q"], P["Qs"], P["K"], P["V"], idx, w, rows)
    for t in range(3):
        for b in range(2):
            assert np.allclose(sub[t][b], full[t][b][rows[b]], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# --------------------------------------------------------------------------

ALL_CHECKS = [check_kv_bytes, check_worked_examples, check_worked_example_routed,
              check_geometric_scores, check_nonsquare_positions, check_head_to_kv_map,
              check_row0_and_hull, check_explicit_equals_repeat, check_router_sums,
              check_routed_kM_equals_dense, check_shared_head_is_dense_head_on_kv0,
              check_k1_obar, check_obar_weighted_sum_k2, check_padding_key_validity,
              check_router_p_values]


def _caught(monkeypatch, name, fn):
    monkeypatch.setattr(og, name, fn)
    failed = []
    for c in ALL_CHECKS:
        try:
            c()
        except AssertionError:
            failed.append(c.__name__)
    return failed


@pytest.mark.parametrize("name,fn", [
    ("_visible", lambda k, q, s=None: k[None, :] < q[:, None]),       # diagonal dropped
    ("_visible", lambda k, q, s=None: k[None, :] <= q[:, None] + 1),  # one key of the future
    ("_visible", lambda k, q, s=None: k[None, :] <= q[:, None]),      # padding ignored
    ("_visible", lambda k, q, s=None: (k[None, :] <= q[:, None]) &    # first valid key dropped
     (True if s is None else k[None, :] > s[:, None])),
    ("_scale", lambda d: 1.0),                                      # scale dropped
    ("_scale", lambda d: 1.0 / d),                                  # wrong scale
    ("_kv_head_of", lambda h, N, G: h % G),                         # interleaved map
    ("_expert_head", lambda g, m, M: m * M + g),                    # transposed roles
    ("_group_softmax", lambda L: _plain_softmax(2.0 * L)),          # temperature 1/2
    ("_group_softmax", lambda L: _plain_softmax(0.5 * L)),          # temperature 2
    ("_group_softmax", lambda L: _plain_softmax(-L)),               # sign of the logits
    ("_group_softmax", lambda L: _plain_softmax(                     # over every head of
        L.reshape(*L.shape[:-2], -1)).reshape(L.shape)),            # the token, not the group
])
def test_planted_mistakes_are_caught(monkeypatch, name, fn):
    failed = _caught(monkeypatch, name, fn)
    assert failed, f"planted mistake in {name} went unnoticed"


def _plain_softmax(L):
    """Softmax over the last axis; used only to build planted mistakes."""
    e = np.exp(L - L.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def test_planted_router_bias_sign_is_caught(monkeypatch):
    """A bias entering the logits with the wrong sign must fail a pin."""
    good = og.router_logits
    monkeypatch.setattr(og, "router_logits",
                        lambda x, Wr, bias: good(x, Wr, None if bias is None else -bias))
    with pytest.raises(AssertionError):
        check_router_p_values()


def test_planted_kv_bytes_mistake(monkeypatch):
    monkeypatch.setattr(oracle, "kv_cache_bytes", lambda L, G, S, d, b, B=1: L * G * d * S * b * B)
    with pytest.raises(AssertionError):
        check_kv_bytes()


# --------------------------------------------------------------------------
# the attention layer around the path: projections and W_O
# --------------------------------------------------------------------------

def test_f64_to_bf16_rounding():
    """Nearest bf16, ties to even: agrees with the input generator's float32
    rounding on float32 values, lands on a neighbour within half an ulp, and
    sends exact midpoints to the even significand."""
    rng = np.random.default_rng(3)
    v32 = (rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000))).astype(np.float32)
    assert np.array_equal(og.f64_to_bf16_bits(v32.astype(np.float64)), f32_to_bf16_bits(v32))
    v = rng.standard_normal(4000) * 7.0
    q = og.bf16_to_f64(og.f64_to_bf16_bits(v))
    ulp = 2.0 ** (np.floor(np.log2(np.abs(v))) - 7)
    assert (np.abs(q - v) <= ulp / 2).all()
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even significand is 1
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    mids = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])
    assert og.bf16_to_f64(og.f64_to_bf16_bits(mids)).tolist() == [1.0, 1 + 2.0 ** -6, -1.0]


def _layer_case(seed, B=1, S=6, N=4, G=2, d=2, dm=10):
    M = N // G
    return dict(
        x=normal_bf16((B, S, dm), seed), Wq=normal_bf16((N, dm, d), seed + 1, std=0.5),
        Wk=normal_bf16((G, dm, d), seed + 2, std=0.5), Wv=normal_bf16((G, dm, d), seed + 3),
        Ws=normal_bf16((dm, d), seed + 4, std=0.5),
        Wr=normal_bf16((G, dm, M), seed + 5, std=dm ** -0.5))


def check_layer_bruteforce():
    """Every step of the layer written out with loops on a tiny case: routed
    query projection for the selected heads only, K/V/shared projections,
    causal softmax attention per selected head, ō, concat, W_O."""
    k = 1
    c = _layer_case(19300)
    B, S, dm = c["x"].shape
    N, _, d = c["Wq"].shape
    G = c["Wk"].shape[0]
    M = N // G
    width = (G * k + G + 1) * d
    Wo = normal_bf16((width, dm), 19306, std=0.3)
    out = oracle.gqe_layer_prefill(c["x"], c["Wq"], c["Wk"], c["Wv"], c["Ws"], c["Wr"], Wo,
                                   None, k)
    X, f = og.bf16_to_f64(c["x"]), og.bf16_to_f64
    rb = lambda v: float(f(og.f64_to_bf16_bits(np.array([v])))[0])  # noqa: E731

    def proj(row, W):  # W [dm, d]
        return [rb(math.fsum(row[c_] * W[c_, e] for c_ in range(dm))) for e in range(d)]

    idx = out["topk_idx"]
    for b in range(B):
        K = [[proj(X[b, t], f(c["Wk"][g])) for g in range(G)] for t in range(S)]
        V = [[proj(X[b, t], f(c["Wv"][g])) for g in range(G)] for t in range(S)]
        for i in range(S):
            def attend(q, g):
                sc = [math.fsum(q[e] * K[t][g][e] for e in range(d)) / math.sqrt(d)
                      for t in range(i + 1)]
                mx = max(sc)
                ex = [math.exp(s_ - mx) for s_ in sc]
                z = math.fsum(ex)
                return [math.fsum(ex[t] * V[t][g][e] for t in range(i + 1)) / z for e in range(d)]
            row = []
            obar = []
            for g in range(G):
                m = int(idx[b, i, g, 0])
                q = proj(X[b, i], f(c["Wq"][g * M + m]))
                assert np.array_equal(out["Q"][b, i, g * M + m],
                                      og.f64_to_bf16_bits(np.array(q)))
                o = attend(q, g)
                row += o
                obar += o                           # k = 1: w = 1
            row += obar + attend(proj(X[b, i], f(c["Ws"])), 0)
            y = [math.fsum(row[r] * f(Wo)[r, c_] for r in range(width)) for c_ in range(dm)]
            assert np.allclose(out["y"][b, i], y, rtol=1e-12, atol=1e-12), (b, i)
            # unselected heads are never projected
            for g in range(G):
                for m in range(M):
                    if m != idx[b, i, g, 0]:
                        assert not out["Q"][b, i, g * M + m].any()


def test_layer_bruteforce():
    check_layer_bruteforce()


ALL_CHECKS.append(check_layer_bruteforce)  # planted mistakes must show here too


def test_layer_with_identity_output_projection_is_the_concat():
    """W_O = I (d_model equal to the concat width) returns the concat buffer,
    which is the path's output on the projected inputs."""
    k = 2
    c = _layer_case(19400, B=2, S=9, N=8, G=2, d=2, dm=(2 * 2 + 2 + 1) * 2)
    dm = c["x"].shape[2]
    eye = og.f64_to_bf16_bits(np.eye(dm))
    out = oracle.gqe_layer_prefill(c["x"], c["Wq"], c["Wk"], c["Wv"], c["Ws"], c["Wr"], eye,
                                   None, k)
    assert np.array_equal(out["y"], out["concat"])
    O_sel, o_bar, s = oracle.gqe_prefill(out["Q"], out["Qs"], out["K"], out["V"],
                                         out["topk_idx"], out["w"])
    B, S = O_sel.shape[:2]
    assert np.array_equal(out["concat"], np.concatenate(
        [O_sel.reshape(B, S, -1), o_bar.reshape(B, S, -1), s], axis=-1))


def test_append_step_equals_prefill_rows():
    """n new tokens appended at slots t..t+n-1 of the full sequence's cache
    are prefill's rows t..t+n-1 (the non-square causal case Sq = n over
    Sk = t + n keys)."""
    (B, S, N, G, k, d, dm), c = _decode_case(19500)
    idx, p, w, _ = oracle.route(c["x"], c["W_r"], None, k)
    O_sel, o_bar, s = oracle.gqe_prefill(c["Q"], c["Qs"], c["K"], c["V"], idx, w)
    for t, n in ((5, 2), (0, 3), (30, 10)):
        sl = slice(t, t + n)
        got = oracle.gqe_append_step(c["x"][:, sl], c["W_r"], None, c["Q"][:, sl],
                                     c["Qs"][:, sl], c["K"], c["V"], np.array([t] * B), k)
        assert np.array_equal(got[0], idx[:, sl])
        assert np.allclose(got[3], O_sel[:, sl], rtol=1e-12, atol=1e-12)
        assert np.allclose(got[4], o_bar[:, sl], rtol=1e-12, atol=1e-12)
        assert np.allclose(got[5], s[:, sl], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# backward pass: every analytic gradient against central finite differences
# --------------------------------------------------------------------------

def _fd(f, x, eps=1e-6):
    """Central differences of the scalar f at x (float64 array), all entries."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        hi = f()
        x[i] = old - eps
        lo = f()
        x[i] = old
        g[i] = (hi - lo) / (2 * eps)
    return g


def test_attention_backward_matches_finite_differences():
    rng = np.random.default_rng(11)
    S, d = 6, 3
    q, K, V = rng.standard_normal((S, d)), rng.standard_normal((S, d)), rng.standard_normal((S, d))
    dO = rng.standard_normal((S, d))
    pos = np.arange(S)
    loss = lambda: float((oracle.causal_attention(q, pos, K, V) * dO).sum())  # noqa: E731
    dq, dK, dV = oracle.causal_attention_backward(q, pos, K, V, dO)
    for got, x in ((dq, q), (dK, K), (dV, V)):
        assert np.allclose(got, _fd(loss, x), atol=1e-8, rtol=1e-6)
    # the last key is seen by the last row only; row 0 sees key 0 only
    assert np.allclose(dq[0], 0.0)           # one visible key: softmax weight 1, no q dependence


def _bwd_case(seed, B=1, S=5, N=4, G=2, k=2, d=3):
    rng = np.random.default_rng(seed)
    M = N // G
    idx = np.stack([rng.permutation(M)[:k] for _ in range(B * S * G)]).reshape(B, S, G, k)
    w = rng.uniform(0.1, 1.0, (B, S, G, k))
    w /= w.sum(axis=-1, keepdims=True)
    t = dict(Q=rng.standard_normal((B, S, N, d)), Qs=rng.standard_normal((B, S, d)),
             K=rng.standard_normal((B, S, G, d)), V=rng.standard_normal((B, S, G, d)), w=w)
    up = dict(dO_sel=rng.standard_normal((B, S, G, k, d)), do_bar=rng.standard_normal((B, S, G, d)),
              ds=rng.standard_normal((B, S, d)))
    return idx, t, up


def check_prefill_backward():
    idx, t, up = _bwd_case(12)

    def loss():
        O, ob, s = oracle.gqe_prefill_values(t["Q"], t["Qs"], t["K"], t["V"], idx, t["w"])
        return float((O * up["dO_sel"]).sum() + (ob * up["do_bar"]).sum() + (s * up["ds"]).sum())
    g = oracle.gqe_prefill_backward(t["Q"], t["Qs"], t["K"], t["V"], idx, t["w"], up["dO_sel"],
                                    up["do_bar"], up["ds"])
    for name, key in (("dQ", "Q"), ("dQs", "Qs"), ("dK", "K"), ("dV", "V"), ("dw", "w")):
        assert np.allclose(g[name], _fd(loss, t[key]), atol=1e-8, rtol=1e-6), name
    # a head a token did not select gets no query gradient
    N, G = t["Q"].shape[2], t["K"].shape[2]
    M = N // G
    for i in range(t["Q"].shape[1]):
        for g_ in range(G):
            for m in range(M):
                if m not in idx[0, i, g_]:
                    assert not g["dQ"][0, i, g_ * M + m].any()


def test_prefill_backward_matches_finite_differences():
    check_prefill_backward()


def test_shared_kv_gradient_is_the_sum_over_its_heads():
    """[GQA article] 训练与部署: the shared K/V gradient equals the reduction
    (a sum, not a mean) of the backward run with K/V logically repeated per
    query head.  Here: k = M (every head of a group active), the routed
    backward against per-head backwards on repeated K/V."""
    idx, t, up = _bwd_case(13, k=2)
    B, S, N, d = t["Q"].shape
    G = t["K"].shape[2]
    M = N // G
    g = oracle.gqe_prefill_backward(t["Q"], t["Qs"], t["K"], t["V"], idx, t["w"], up["dO_sel"],
                                    up["do_bar"], up["ds"])
    pos = np.arange(S)
    dK = np.zeros_like(t["K"])
    for g_ in range(G):
        for m in range(M):
            # rows whose slot j selected expert m, with their upstream gradient
            dO = np.zeros((S, d))
            sel = np.zeros(S, bool)
            for j in range(2):
                hit = idx[0, :, g_, j] == m
                dO[hit] = up["dO_sel"][0, hit, g_, j] + t["w"][0, hit, g_, j, None] * up["do_bar"][0, hit, g_]
                sel |= hit
            assert sel.all()                  # k = M: every token uses every head
            Krep = t["K"][0, :, g_].copy()    # this head's own copy of the shared K
            _, dk, _ = oracle.causal_attention_backward(t["Q"][0, :, g_ * M + m], pos, Krep,
                                                        t["V"][0, :, g_], dO)
            dK[0, :, g_] += dk
    _, dk, _ = oracle.causal_attention_backward(t["Qs"][0], pos, t["K"][0, :, 0], t["V"][0, :, 0],
                                                up["ds"][0])
    dK[0, :, 0] += dk
    assert np.allclose(g["dK"], dK, atol=1e-12)
    assert not np.allclose(g["dK"][0, :, 1], dK[0, :, 1] / M)   # a mean would differ


def test_router_backward_matches_finite_differences():
    rng = np.random.default_rng(14)
    B, S, G, M, dm, k = 1, 4, 2, 4, 5, 2
    x = rng.standard_normal((B, S, dm))
    Wr = rng.standard_normal((G, dm, M)) * 0.5
    bias = rng.standard_normal((G, M)) * 0.1
    p, _ = oracle.router_values(x, Wr, bias, np.zeros((B, S, G, k), np.int64))
    idx = np.argsort(-p, axis=-1, kind="stable")[..., :k]
    dw = rng.standard_normal((B, S, G, k))
    dpx = rng.standard_normal((B, S, G, M))

    def loss():
        p_, w_ = oracle.router_values(x, Wr, bias, idx)
        return float((w_ * dw).sum() + (p_ * dpx).sum())
    g = oracle.router_backward(x, Wr, bias, idx, dw, dp_extra=dpx)
    assert np.allclose(g["dx"], _fd(loss, x), atol=1e-8, rtol=1e-6)
    assert np.allclose(g["dWr"], _fd(loss, Wr), atol=1e-8, rtol=1e-6)
    assert np.allclose(g["dbias"], _fd(loss, bias), atol=1e-8, rtol=1e-6)
    # k = 1: w is 1 for any p, so the weighted-sum slot gives the router nothing
    g1 = oracle.router_backward(x, Wr, bias, idx[..., :1], dw[..., :1])
    assert np.allclose(g1["dlogits"], 0.0, atol=1e-15)


def test_load_balance_loss_values_and_gradient():
    """Balanced routing and uniform p give alpha; everything on one expert
    with p concentrated there gives alpha * M; the gradient in p is exact."""
    B, S, G, M, k = 2, 8, 3, 4, 1
    p = np.full((B, S, G, M), 1.0 / M)
    idx = (np.arange(B * S * G) % M).reshape(B, S, G, 1)
    L, _ = oracle.load_balance_loss(p, idx, alpha=0.5)
    assert np.isclose(L, 0.5)
    p1 = np.zeros((B, S, G, M))
    p1[..., 0] = 1.0
    L1, _ = oracle.load_balance_loss(p1, np.zeros((B, S, G, 1), np.int64), alpha=0.5)
    assert np.isclose(L1, 0.5 * M)
    rng = np.random.default_rng(15)
    pr = rng.uniform(size=(B, S, G, M))
    pr /= pr.sum(-1, keepdims=True)
    idr = rng.integers(0, M, (B, S, G, 2))
    _, dp = oracle.load_balance_loss(pr, idr)
    assert np.allclose(dp, _fd(lambda: oracle.load_balance_loss(pr, idr)[0], pr), atol=1e-9)


ALL_CHECKS.append(check_prefill_backward)
