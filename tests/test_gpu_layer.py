"""The attention layer around the path on the GPU: gqe_linear (the dense
projections and W_O), gqe_routed_q_project (the query projection of the
selected heads only, [GQE review] §二 路由器) and the whole layer
gqe_layer_prefill (y = Concat(O, o_bar, s) W_O, §二 三个关键部件), against the
oracle's gqe_layer_prefill; and the all-active baseline layer.

Projections are bf16 x bf16 with float32 accumulation, rounded to bf16 for
the attention: a value whose float64 result lies within the float32
accumulation error of a bf16 rounding midpoint may round the other way, so
projections are compared to that error bound plus one bf16 unit in the last
place, with almost all elements equal.  The concat buffer feeds W_O as bf16,
so it is held to the bf16 output mode's bound of the attention call; y is
checked exactly against that concat times W_O (float32 accumulation bound)
and against the oracle's y within the concat's rounding carried through W_O
(5e-3 relative L2).
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.gqe_oracle as og
from gpu_util import check_close, dev_bf16
from synth import normal_bf16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqeLayer  # noqa: E402


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _bound_linear(A, W, K):
    """Any float32 summation order of K exact products: |err| <= K u sum|a w|."""
    return K * 2.0 ** -24 * 1.01 * (np.abs(A) @ np.abs(W))


@pytest.mark.parametrize("rows,K,nb,nc,c_fp32", [(300, 128, 4, 64, 1), (129, 256, 1, 128, 1),
                                                (517, 192, 2, 128, 0), (1000, 64, 1, 1024, 1),
                                                (64, 1088, 1, 256, 1)])
def test_linear_against_float64(rows, K, nb, nc, c_fp32):
    A = normal_bf16((rows, K), 31 + rows)
    W = normal_bf16((nb, K, nc), 37 + K, std=K ** -0.5)
    Af, Wf = og.bf16_to_f64(A), og.bf16_to_f64(W)
    ref = np.concatenate([Af @ Wf[i] for i in range(nb)], axis=1)
    bound = np.concatenate([_bound_linear(Af, Wf[i], K) for i in range(nb)], axis=1)
    dt = torch.float32 if c_fp32 else torch.bfloat16
    C = torch.full((rows, nb * nc), float("nan"), dtype=dt, device="cuda")
    gqe.gqe_linear(rows, K, nb, nc, dev_bf16(A), K, dev_bf16(W), C, nb * nc, c_fp32)
    torch.cuda.synchronize()
    got = _f64(C)
    assert np.isfinite(got).all()
    if c_fp32:
        assert (np.abs(got - ref) <= bound + 1e-30).all(), np.abs(got - ref).max()
    else:  # plus the rounding to bf16: half a unit in the last place
        assert (np.abs(got - ref) <= bound + np.abs(ref) * 2.0 ** -8 + 1e-30).all()


def test_linear_refuses_unsupported_shapes():
    t = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    assert gqe.gqe_linear(10, 100, 1, 64, t, 100, t, t, 64, 1, check=False) == 2   # K % 64
    assert gqe.gqe_linear(10, 64, 1, 96, t, 64, t, t, 96, 1, check=False) == 2     # nc % 64
    assert gqe.gqe_linear(10, 64, 1, 64, t, 60, t, t, 64, 1, check=False) == 1     # lda < K


def _layer_case(B, S, N, G, k, d, dm, seed, bias0=0.0):
    M = N // G
    inp = dict(x=normal_bf16((B, S, dm), seed), W_Q=normal_bf16((N, dm, d), seed + 1, std=dm ** -0.5),
               W_K=normal_bf16((G, dm, d), seed + 2, std=dm ** -0.5),
               W_V=normal_bf16((G, dm, d), seed + 3, std=dm ** -0.5),
               W_s=normal_bf16((dm, d), seed + 4, std=dm ** -0.5),
               W_r=normal_bf16((G, dm, M), seed + 5, std=dm ** -0.5),
               W_O=normal_bf16(((G * k + G + 1) * d, dm), seed + 6, std=((G * k + G + 1) * d) ** -0.5))
    bias = None
    if bias0:
        bias = np.zeros((G, M), np.float32)
        bias[:, 0] = bias0
    return inp, bias


def _ulp_close(got_bits, ref_bits, bound, what, max_frac=1e-2):
    """got = bf16(a) with a within `bound` of the exact value, ref = bf16 of
    the exact value: |got - ref| <= bound + one bf16 unit in the last place."""
    g, r = og.bf16_to_f64(got_bits), og.bf16_to_f64(ref_bits)
    diff = np.abs(g - r)
    ulp = np.maximum(np.abs(r), np.abs(g)) * 2.0 ** -7  # one bf16 unit (8 significant bits)
    assert (diff <= ulp + bound + 1e-38).all(), f"{what}: a difference above the bound"
    frac = float((diff > 0).mean())
    assert frac <= max_frac, f"{what}: {frac:.2e} of the elements differ"


def _proj_bound(x, W, dm):
    """float32 accumulation of dm exact products, any order: dm u sum|x w|."""
    return dm * 2.0 ** -24 * 1.01 * (np.abs(x) @ np.abs(W))


@pytest.mark.parametrize("shape", [(2, 300, 8, 4, 2, 64, 128), (1, 260, 8, 2, 1, 128, 256),
                                   (1, 200, 16, 8, 1, 64, 64)])
def test_layer_prefill_matches_oracle(shape):
    B, S, N, G, k, d, dm = shape
    inp, bias = _layer_case(B, S, N, G, k, d, dm, 1200 + S)
    L = GqeLayer(B, S, N, G, k, d, dm)
    dv = {n: dev_bf16(v) for n, v in inp.items()}
    dbias = None if bias is None else torch.from_numpy(bias).cuda()
    L.forward(dv["x"], dv["W_Q"], dv["W_K"], dv["W_V"], dv["W_s"], dv["W_r"], dbias, dv["W_O"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    ref = oracle.gqe_layer_prefill(inp["x"], inp["W_Q"], inp["W_K"], inp["W_V"], inp["W_s"],
                                   inp["W_r"], inp["W_O"], bias, k)
    idx = ref["topk_idx"]
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    bits = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    x = og.bf16_to_f64(inp["x"])
    bK = np.stack([_proj_bound(x, og.bf16_to_f64(inp["W_K"][g]), dm) for g in range(G)], axis=2)
    bV = np.stack([_proj_bound(x, og.bf16_to_f64(inp["W_V"][g]), dm) for g in range(G)], axis=2)
    bQ = np.stack([_proj_bound(x, og.bf16_to_f64(inp["W_Q"][h]), dm) for h in range(N)], axis=2)
    _ulp_close(bits(L.K), ref["K"], bK, "K")
    _ulp_close(bits(L.V), ref["V"], bV, "V")
    _ulp_close(bits(L.Qs), ref["Qs"], _proj_bound(x, og.bf16_to_f64(inp["W_s"]), dm), "Qs")
    # Q: the rows of the selected heads only
    M = N // G
    sel = np.zeros((B, S, N), bool)
    for g in range(G):
        for j in range(k):
            np.put_along_axis(sel[:, :, g * M:(g + 1) * M], idx[:, :, g, j:j + 1], True, axis=-1)
    _ulp_close(bits(L.Q)[sel], ref["Q"][sel], bQ[sel], "Q (selected heads)")
    # the concat buffer is bf16 here: the float32 bound plus half an ulp of
    # rounding, and the k > 1 weighted sum reads the rounded slots (another
    # half ulp), as in the bf16 output mode of the attention call
    cat = L.concat.float().cpu().numpy().astype(np.float64).reshape(ref["concat"].shape)
    rc = ref["concat"]
    assert (np.abs(cat - rc) <= 1e-2 + 2.0 ** -8 * np.abs(rc)).all(), "concat"
    check_close(cat, rc, "concat", atol=1e-2 + 2.0 ** -8 * float(np.abs(rc).max()), rtol_l2=5e-3)
    # W_O: y is the float32-accumulated product of that bf16 concat and W_O
    Wo = og.bf16_to_f64(inp["W_O"])
    y = L.y.cpu().numpy().astype(np.float64)
    y_own = cat @ Wo
    K = cat.shape[-1]
    assert (np.abs(y - y_own) <= K * 2.0 ** -24 * 1.01 * (np.abs(cat) @ np.abs(Wo)) + 1e-30).all()
    # and against the oracle's y: the concat's rounding to bf16 (2^-8
    # relative at most, 2^-9 typical) carried through W_O
    check_close(y, ref["y"], "y", atol=1e-2, rtol_l2=5e-3)


def test_routed_q_project_writes_only_selected_rows():
    B, S, N, G, k, d, dm = 1, 333, 8, 4, 1, 64, 128
    inp, _ = _layer_case(B, S, N, G, k, d, dm, 1400)
    idx, _, _, _ = oracle.route(inp["x"], inp["W_r"], None, k)
    dm_ = gqe.dims(B, S, N, G, k, d, dm, 1)
    ws = torch.zeros(gqe.gqe_workspace_size(dm_), dtype=torch.uint8, device="cuda")
    Q = torch.full((B, S, N, d), 7.0, dtype=torch.bfloat16, device="cuda")
    gqe.gqe_routed_q_project(dm_, dev_bf16(inp["x"]), dev_bf16(inp["W_Q"]),
                             torch.from_numpy(idx).cuda(), Q, ws)
    torch.cuda.synchronize()
    x, Wq = og.bf16_to_f64(inp["x"]), og.bf16_to_f64(inp["W_Q"])
    got = _f64(Q)
    M = N // G
    for g in range(G):
        for m in range(M):
            h = g * M + m
            rows = (idx[0, :, g, 0] == m)
            ref = x[0][rows] @ Wq[h]
            assert (np.abs(got[0, rows, h] - ref) <= np.abs(ref) * 2.0 ** -8
                    + _bound_linear(x[0][rows], Wq[h], dm)).all()
            assert (got[0, ~rows, h] == 7.0).all()   # unselected rows untouched


def test_dense_layer_matches_oracle_pieces():
    B, S, N, G, d, dm = 1, 257, 8, 4, 64, 128
    inp, _ = _layer_case(B, S, N, G, 1, d, dm, 1500)
    W_Od = normal_bf16((N * d, dm), 1507, std=(N * d) ** -0.5)
    L = GqeLayer(B, S, N, G, 1, d, dm)
    dv = {n: dev_bf16(v) for n, v in inp.items()}
    y = L.dense(dv["x"], dv["W_Q"], dv["W_K"], dv["W_V"], dev_bf16(W_Od))
    torch.cuda.synchronize()
    assert L.device_status() == 0
    x = og.bf16_to_f64(inp["x"])
    Qb = og.f64_to_bf16_bits(np.einsum("bsc,hcd->bshd", x, og.bf16_to_f64(inp["W_Q"])))
    Kb = og.f64_to_bf16_bits(np.einsum("bsc,gcd->bsgd", x, og.bf16_to_f64(inp["W_K"])))
    Vb = og.f64_to_bf16_bits(np.einsum("bsc,gcd->bsgd", x, og.bf16_to_f64(inp["W_V"])))
    O = oracle.dense_gqa(Qb, Kb, Vb)
    y_ref = og.bf16_to_f64(og.f64_to_bf16_bits(O.reshape(B, S, N * d))) @ og.bf16_to_f64(W_Od)
    check_close(y.cpu().numpy(), y_ref, "dense layer y")
