"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Routing indices and buckets must match bit for bit; floating-point outputs
(float32) must be within 1e-2 max-abs and 1e-3 relative L2 of the float64
oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_close, make_case, upload, dev_bf16
from synth import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402

# (B, S, N, G, k, d, d_model): tiny workload, ragged tails, k>1, d=128,
# k = M, M = 1, G = 1, a single token
SHAPES = [
    (1, 128, 16, 8, 1, 64, 256),
    (2, 300, 8, 4, 2, 64, 64),
    (1, 200, 16, 4, 2, 128, 128),
    (1, 384, 32, 8, 2, 128, 256),
    (1, 1, 16, 8, 1, 64, 64),
    (1, 129, 16, 8, 1, 64, 64),
    (1, 256, 8, 4, 2, 64, 64),
    (1, 130, 8, 8, 1, 64, 64),
    (1, 257, 8, 1, 3, 64, 64),
]


def _run(shape, seed, out_fp32=True, bias0=0.0):
    B, S, N, G, k, d, dm = shape
    inp = make_case(B, S, N, G, k, d, dm, seed, bias0=bias0)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm, out_fp32=out_fp32)
    L.forward(dev["x"], dev["W_r"], dev["bias"], dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return inp, L


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_routed_prefill_parity(shape):
    B, S, N, G, k, d, dm = shape
    inp, L = _run(shape, seed=1000 + sum(shape))
    idx, p, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx), "top-k indices differ"
    check_close(L.p.cpu().numpy(), p, "p", atol=1e-5, rtol_l2=1e-5)
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


@pytest.mark.parametrize("shape", SHAPES[:4], ids=lambda s: "x".join(map(str, s)))
def test_bucket_bit_exact(shape):
    B, S, N, G, k, d, dm = shape
    inp, L = _run(shape, seed=2000 + sum(shape))
    idx = L.topk_idx.cpu().numpy()
    off = torch.empty(B * G * (N // G) + 1, dtype=torch.int32, device="cuda")
    tok = torch.empty(B * G * S * k, dtype=torch.int32, device="cuda")
    gqe.gqe_bucket(L.dims, L.topk_idx, off, tok, L.ws)
    torch.cuda.synchronize()
    ro, rt = oracle.bucket(idx, N // G)
    assert np.array_equal(off.cpu().numpy().astype(np.int64), ro)
    assert np.array_equal(tok.cpu().numpy(), rt)


@pytest.mark.parametrize("shape", [SHAPES[0], SHAPES[1], SHAPES[2], SHAPES[4], SHAPES[8]],
                         ids=lambda s: "x".join(map(str, s)))
def test_dense_gqa_parity(shape):
    B, S, N, G, k, d, dm = shape
    inp = make_case(B, S, N, G, k, d, dm, seed=3000 + sum(shape))
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm)
    O = L.dense(dev["Q"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    ref = oracle.dense_gqa(inp["Q"], inp["K"], inp["V"])
    check_close(O.cpu().numpy(), ref, "dense O")


def test_bf16_output_mode():
    shape = (1, 300, 16, 8, 2, 64, 64)
    B, S, N, G, k, d, dm = shape
    inp, L = _run(shape, seed=4000, out_fp32=False)
    idx, p, w, _ = oracle.route(inp["x"], inp["W_r"], None, k)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    # Rounding the output to bf16 adds up to half an ulp (2^-9 relative), and
    # the k>1 weighted sum reads the already rounded slots (another 2^-9), so
    # the bound is the float32 one plus 2^-8 |ref| elementwise.
    for got, ref, what in ((L.O_sel(), O_sel, "O_sel"), (L.o_bar(), o_bar, "o_bar"),
                           (L.s_out(), s, "s")):
        g = got.float().cpu().numpy()
        assert (np.abs(g - ref) <= 1e-2 + 2 ** -8 * np.abs(ref)).all(), what
        check_close(g, ref, what, atol=1e-2 + 2 ** -8 * float(np.abs(ref).max()),
                    rtol_l2=5e-3)


def test_router_exact_ties_and_bias():
    """Duplicated W_r columns force exact ties (lower index wins); values from
    a small set make many logits tie exactly, so the exact path is used."""
    B, S, N, G, k, d, dm = 1, 512, 16, 4, 2, 64, 64
    M = N // G
    rng = np.random.default_rng(7)
    vals = np.array([-2, -1, -0.5, 0, 0.5, 1, 2], np.float32)
    x = f32_to_bf16_bits(vals[rng.integers(0, 7, (B, S, dm))])
    W = vals[rng.integers(0, 7, (G, dm, M))] * 0.125
    W[:, :, 2] = W[:, :, 0]
    Wb = f32_to_bf16_bits(W)
    bias = np.zeros((G, M), np.float32)
    bias[1, 3] = 0.25
    L = GqePrefill(B, S, N, G, k, d, dm)
    L.route(dev_bf16(x), dev_bf16(Wb), torch.from_numpy(bias).cuda())
    torch.cuda.synchronize()
    assert L.device_status() == 0
    idx, p, w, n_exact = oracle.route(x, Wb, bias, k)
    assert n_exact > 0
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)


def test_empty_bucket():
    """A large bias sends every token of every group to expert 0: the other
    experts' buckets are empty."""
    shape = (2, 200, 16, 8, 1, 64, 64)
    inp, L = _run(shape, seed=5000, bias0=100.0)
    idx = L.topk_idx.cpu().numpy()
    assert (idx == 0).all()
    _, _, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], 1)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.s_out().cpu().numpy(), s, "s")


def test_k1_weights_and_obar_copy():
    inp, L = _run((1, 256, 16, 8, 1, 64, 128), seed=6000)
    assert (L.w.cpu() == 1.0).all()
    assert torch.equal(L.o_bar(), L.O_sel()[:, :, :, 0])


def test_repeat_calls_are_deterministic():
    shape = (2, 300, 8, 4, 2, 64, 64)
    inp, L = _run(shape, seed=7000)
    first = L.concat.clone()
    dev = upload(inp)
    for _ in range(3):
        L.forward(dev["x"], dev["W_r"], None, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert torch.equal(first, L.concat)


def test_bounded_wait_reports_timeout():
    L = GqePrefill(1, 128, 16, 8, 1, 64, 64)
    gqe.gqe_selftest_bounded_wait(L.ws, 2000)
    assert L.device_status(clear=True) == 4      # GQE_ERR_TIMEOUT, context still usable
    assert L.device_status(clear=True) == 0
    inp, L2 = _run((1, 128, 16, 8, 1, 64, 256), seed=8000)
    assert L2.device_status() == 0


def test_router_exact_wide_exponent_range():
    """Exact ties whose products span ~170 binary orders of magnitude: the
    exact comparison cannot use its register window and must take the full
    fixed-point accumulator."""
    B, S, N, G, k, d, dm = 1, 256, 8, 2, 1, 64, 64
    M = N // G
    rng = np.random.default_rng(11)
    mags = np.array([2.0 ** -90, 2.0 ** -40, 1.0, 2.0 ** 30, 2.0 ** 60], np.float64)
    x = (mags[rng.integers(0, 5, (B, S, dm))] * rng.choice([-1, 1], (B, S, dm))).astype(np.float32)
    W = (mags[rng.integers(0, 5, (G, dm, M))] * rng.choice([-1, 1], (G, dm, M)) * 2.0 ** -20
         ).astype(np.float32)
    W[:, :, 1] = W[:, :, 0]                 # experts 0 and 1 tie exactly everywhere
    xb, Wb = f32_to_bf16_bits(x), f32_to_bf16_bits(W)
    L = GqePrefill(B, S, N, G, k, d, dm)
    L.route(dev_bf16(xb), dev_bf16(Wb), None)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    idx, p, w, n_exact = oracle.route(xb, Wb, None, k)
    assert n_exact > 0
    got = L.topk_idx.cpu().numpy()
    assert np.array_equal(got, idx)
    assert not (got == 1).any()             # the tie always goes to expert 0
    # p of the re-decided pairs comes from their exact (or float64) logits on
    # both sides, so it stays a proper distribution even where the products
    # cancel far below float32's reach
    gp = L.p.cpu().numpy()
    assert np.isfinite(gp).all() and np.isfinite(L.w.cpu().numpy()).all()
    check_close(gp, p, "p", atol=1e-5, rtol_l2=1e-5)


# more shapes: d = 128 with every expert selected (k = M), a batch of 3 with
# biased routing and k = 2, and the bf16 output at d = 128
MORE = [
    ((1, 300, 16, 4, 4, 128, 128), 0.0),
    ((3, 257, 16, 4, 2, 64, 64), 1.5),
]


@pytest.mark.parametrize("shape,bias0", MORE, ids=lambda v: "x".join(map(str, v))
                         if isinstance(v, tuple) else str(v))
def test_routed_prefill_parity_more(shape, bias0):
    B, S, N, G, k, d, dm = shape
    inp, L = _run(shape, seed=17000 + sum(shape), bias0=bias0)
    idx, p, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx), "top-k indices differ"
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


def test_bf16_output_mode_d128():
    shape = (1, 300, 16, 4, 2, 128, 128)
    B, S, N, G, k, d, dm = shape
    inp, L = _run(shape, seed=18000, out_fp32=False)
    idx, p, w, _ = oracle.route(inp["x"], inp["W_r"], None, k)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    # float32 bound plus 2^-8 |ref|: half an ulp for the bf16 output, half
    # for the k > 1 sum of already rounded slots
    for got, ref, what in ((L.O_sel(), O_sel, "O_sel"), (L.o_bar(), o_bar, "o_bar"),
                           (L.s_out(), s, "s")):
        g = got.float().cpu().numpy()
        assert (np.abs(g - ref) <= 1e-2 + 2 ** -8 * np.abs(ref)).all(), what


def test_right_padded_batch_rows_are_exact():
    """Right padding ([GQA article] 工程实操 step 4): a valid row i < len_b
    sees keys t <= i < len_b only, so the causal mask already implies key
    validity and the padded tail (garbage tokens, routed like any other)
    cannot reach it.  Each sequence's valid rows equal the oracle on that
    sequence cut to its length."""
    shape = (3, 300, 16, 8, 2, 64, 64)
    B, S, N, G, k, d, dm = shape
    lens = [300, 177, 1]
    inp, L = _run(shape, seed=18500)
    go, gb, gs = L.O_sel().cpu().numpy(), L.o_bar().cpu().numpy(), L.s_out().cpu().numpy()
    gi = L.topk_idx.cpu().numpy()
    for b, n in enumerate(lens):
        cut = {key: inp[key][b:b + 1, :n] for key in ("x", "Q", "Qs", "K", "V")}
        idx, p, w, _ = oracle.route(cut["x"], inp["W_r"], None, k)
        assert np.array_equal(gi[b:b + 1, :n], idx)
        O_sel, o_bar, s = oracle.gqe_prefill(cut["Q"], cut["Qs"], cut["K"], cut["V"], idx, w)
        check_close(go[b:b + 1, :n], O_sel, f"O_sel b={b}")
        check_close(gb[b:b + 1, :n], o_bar, f"o_bar b={b}")
        check_close(gs[b:b + 1, :n], s, f"s b={b}")
