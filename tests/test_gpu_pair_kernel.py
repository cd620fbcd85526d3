"""The d = 64 pair kernel: two 128-row query tiles of one KV head per CTA,
sharing every K/V tile load.  The library picks it for routed calls when K and
V outgrow L2; these tests force it on small shapes with
gqe_set_pair_threshold(0) and check it against the oracle, and bit for bit
against the one-tile kernel (both run the same arithmetic on every tile)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_close, make_case, upload
from synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402

# d = 64 shapes: tiny, ragged tails, k > 1, a single token, M = 1, G = 1 with
# k = 3 of M = 8 (odd tile counts leave pairs with an empty second tile)
SHAPES = [
    (1, 128, 16, 8, 1, 64, 256),
    (2, 300, 8, 4, 2, 64, 64),
    (1, 1, 16, 8, 1, 64, 64),
    (1, 129, 16, 8, 1, 64, 64),
    (1, 256, 8, 4, 2, 64, 64),
    (1, 130, 8, 8, 1, 64, 64),
    (1, 257, 8, 1, 3, 64, 64),
]
ids = lambda s: "x".join(map(str, s))  # noqa: E731


@pytest.fixture
def pair_kernel():
    prev = gqe.gqe_set_pair_threshold(0)
    yield
    gqe.gqe_set_pair_threshold(prev)


def _forward(shape, seed, bias0=0.0):
    B, S, N, G, k, d, dm = shape
    inp = make_case(B, S, N, G, k, d, dm, seed, bias0=bias0)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm, out_fp32=True)
    L.forward(dev["x"], dev["W_r"], dev["bias"], dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return inp, dev, L


@pytest.mark.parametrize("shape", SHAPES, ids=ids)
def test_routed_parity_pair_kernel(shape, pair_kernel):
    k = shape[4]
    inp, _, L = _forward(shape, seed=11000 + sum(shape))
    idx, p, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


def test_biased_batch_pair_kernel(pair_kernel):
    """A batch of 3 with routing biased towards expert 0 (uneven buckets, so
    uneven pairs) and k = 2."""
    shape = (3, 257, 16, 4, 2, 64, 64)
    inp, _, L = _forward(shape, seed=16000, bias0=1.5)
    idx, _, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], 2)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


def test_empty_buckets_pair_kernel(pair_kernel):
    """Every token picks expert 0: the other buckets are empty and some pairs
    have an empty second tile."""
    shape = (2, 200, 16, 8, 1, 64, 64)
    inp, _, L = _forward(shape, seed=13000, bias0=100.0)
    idx = L.topk_idx.cpu().numpy()
    assert (idx == 0).all()
    _, _, w, _ = oracle.route(inp["x"], inp["W_r"], inp["bias"], 1)
    O_sel, _, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.s_out().cpu().numpy(), s, "s")


def test_bf16_output_pair_kernel(pair_kernel):
    """bf16 concat output through the pair kernel's staged stores: within the
    float32 bound plus 2^-8 |ref| (half an ulp for the output, half for the
    k > 1 sum of rounded slots)."""
    shape = (1, 300, 16, 8, 2, 64, 64)
    B, S, N, G, k, d, dm = shape
    inp = make_case(B, S, N, G, k, d, dm, 14000)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm, out_fp32=False)
    L.forward(dev["x"], dev["W_r"], None, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    idx, _, w, _ = oracle.route(inp["x"], inp["W_r"], None, k)
    O_sel, o_bar, s = oracle.gqe_prefill(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx, w)
    for got, ref, what in ((L.O_sel(), O_sel, "O_sel"), (L.o_bar(), o_bar, "o_bar"),
                           (L.s_out(), s, "s")):
        g = got.float().cpu().numpy()
        assert (np.abs(g - ref) <= 1e-2 + 2 ** -8 * np.abs(ref)).all(), what


def test_static_entry_with_pair_kernel(pair_kernel):
    """The no-workspace entry takes the same kernel decision: with the pair
    kernel forced it writes what the workspace call writes, bit for bit."""
    shape = (2, 300, 16, 8, 2, 64, 64)
    inp, dev, L = _forward(shape, seed=15000)
    out = torch.full_like(L.concat, float("nan"))
    a = L.G * L.k * L.d
    gqe.gqe_attention_prefill_static(L.dims, dev["Q"], dev["Qs"], dev["K"], dev["V"],
                                     L.topk_idx, L.w, out, out.view(-1)[a:],
                                     out.view(-1)[a + L.G * L.d:], L.row)
    torch.cuda.synchronize()
    assert torch.equal(out, L.concat)


@pytest.mark.parametrize("name", ["layer250m", "imbalanced32k"])
def test_pair_kernel_equals_one_tile_kernel(name):
    """Both kernels agree on a full-size workload (the pair kernel sends 1 of
    8 exponential pairs to the FMA polynomial, the one-tile kernel 2, so the
    bits differ within the polynomial's 7.5e-5 relative error); dense calls
    keep the one-tile kernel whatever the threshold (same bits)."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    dev = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(torch.bfloat16).cuda()
           for k, v in inp.items() if k != "bias"}
    bias = None if inp.get("bias") is None else torch.from_numpy(inp["bias"]).cuda()
    L = GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True)
    outs = []
    for thr in (-1, 0):
        prev = gqe.gqe_set_pair_threshold(thr)
        try:
            L.forward(dev["x"], dev["W_r"], bias, dev["Q"], dev["Qs"], dev["K"], dev["V"])
            O = L.dense(dev["Q"], dev["K"], dev["V"])
            torch.cuda.synchronize()
            assert L.device_status() == 0
            outs.append((L.concat.clone(), O.clone()))
        finally:
            gqe.gqe_set_pair_threshold(prev)
    check_close(outs[1][0].cpu().numpy(), outs[0][0].cpu().numpy(), "pair vs one-tile",
                atol=1e-3, rtol_l2=1e-4)
    assert torch.equal(outs[0][1], outs[1][1]), "dense output differs"


def test_threshold_roundtrip():
    prev = gqe.gqe_set_pair_threshold(123)
    try:
        assert gqe.gqe_set_pair_threshold(456) == 123
    finally:
        gqe.gqe_set_pair_threshold(prev)
