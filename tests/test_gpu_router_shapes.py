"""The router at every (d_model, G*M) shape class its kernels take: top-k
indices bit-exact against the oracle, p and w within float32 rounding.

The router keeps W_r in shared memory when W_r (float32) fits and d_model
splits into whole 8-value groups per K slice, and streams it from a float32
copy otherwise; by default the resident kernel also needs 3 tiles of 64
tokens per SM, so every test here runs twice: with the resident kernel forced
wherever it fits, and with the default choice (the streamed kernel at these
token counts).  The shapes reach every column-group split of the resident
kernel (G*M = 4, 8, 16, 32) and the streamed fallbacks, with Gaussian data
(certified decisions), with a value set that makes many logits tie exactly
(the exact fix-up), and with products spread over many binary orders (the
wide fixed-point accumulator).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_close, dev_bf16
from synth import f32_to_bf16_bits

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402


@pytest.fixture(params=[1, 0], ids=["resident", "default"])
def resident(request):
    prev = gqe.gqe_set_router_resident(request.param)
    yield request.param
    gqe.gqe_set_router_resident(prev)

# (G, M, k, d_model)
SHAPES = [
    (8, 2, 1, 128),    # G*M = 16: 16 K slices of 8 values
    (8, 2, 1, 256),
    (8, 2, 1, 512),
    (8, 2, 1, 1024),   # the 250M-layer and long-context shapes
    (2, 2, 1, 256),    # G*M = 4
    (4, 2, 2, 1024),   # G*M = 8, k = M
    (8, 4, 2, 512),    # G*M = 32: two column groups, 8 K slices
    (4, 2, 2, 2048),   # G*M = 8 with 64 KB of W_r
    (8, 4, 2, 4096),   # streamed: W_r does not fit (the wide-grouping shape)
    (8, 2, 1, 64),     # streamed: d_model not a multiple of 128
]


def _route(x, Wb, bias, G, M, k, dm):
    B, S = x.shape[:2]
    L = GqePrefill(B, S, G * M, G, k, 64, dm)
    L.route(dev_bf16(x), dev_bf16(Wb), None if bias is None else torch.from_numpy(bias).cuda())
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return L


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_router_gaussian(shape, resident):
    G, M, k, dm = shape
    rng = np.random.default_rng(31000 + G * 1000 + dm)
    S = 1000  # ragged against every tile size
    x = f32_to_bf16_bits(rng.standard_normal((1, S, dm)).astype(np.float32))
    Wb = f32_to_bf16_bits((rng.standard_normal((G, dm, M)) / np.sqrt(dm)).astype(np.float32))
    bias = (0.1 * rng.standard_normal((G, M))).astype(np.float32)
    L = _route(x, Wb, bias, G, M, k, dm)
    idx, p, w, _ = oracle.route(x, Wb, bias, k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    check_close(L.p.cpu().numpy(), p, "p", atol=1e-5, rtol_l2=1e-5)
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_router_exact_ties(shape, resident):
    """Duplicated columns tie exactly everywhere (the lower index must win);
    x and W_r from a small value set tie many other logits too."""
    G, M, k, dm = shape
    rng = np.random.default_rng(32000 + G * 1000 + dm)
    S = 333 if dm <= 512 else 97
    vals = np.array([-2, -1, -0.5, 0, 0.5, 1, 2], np.float32)
    x = f32_to_bf16_bits(vals[rng.integers(0, 7, (1, S, dm))])
    W = vals[rng.integers(0, 7, (G, dm, M))] * 0.125
    W[:, :, M - 1] = W[:, :, 0]
    Wb = f32_to_bf16_bits(W)
    L = _route(x, Wb, None, G, M, k, dm)
    idx, p, w, n_exact = oracle.route(x, Wb, None, k)
    assert n_exact > 0
    got = L.topk_idx.cpu().numpy()
    assert np.array_equal(got, idx)
    if k == 1:
        assert not (got == M - 1).any()     # the tie goes to expert 0
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)


@pytest.mark.parametrize("shape", [SHAPES[1], SHAPES[3], SHAPES[6], SHAPES[9]],
                         ids=lambda s: "x".join(map(str, s)))
def test_router_wide_exponent_range(shape, resident):
    G, M, k, dm = shape
    rng = np.random.default_rng(33000 + dm)
    S = 200
    mags = np.array([2.0 ** -90, 2.0 ** -40, 1.0, 2.0 ** 30, 2.0 ** 60], np.float64)
    x = (mags[rng.integers(0, 5, (1, S, dm))] * rng.choice([-1, 1], (1, S, dm))).astype(np.float32)
    W = (mags[rng.integers(0, 5, (G, dm, M))] * rng.choice([-1, 1], (G, dm, M)) * 2.0 ** -20
         ).astype(np.float32)
    W[:, :, 1] = W[:, :, 0]
    xb, Wb = f32_to_bf16_bits(x), f32_to_bf16_bits(W)
    L = _route(xb, Wb, None, G, M, k, dm)
    idx, p, w, n_exact = oracle.route(xb, Wb, None, k)
    assert n_exact > 0
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    assert np.isfinite(L.p.cpu().numpy()).all() and np.isfinite(L.w.cpu().numpy()).all()
    check_close(L.p.cpu().numpy(), p, "p", atol=1e-5, rtol_l2=1e-5)
