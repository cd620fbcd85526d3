"""gqe_attention_prefill_static: the attention call that needs no workspace.

It exists for callers that cannot allocate device memory (a plugin whose host
framework owns every allocation, or a loop that must not pay cudaMalloc's
device-wide synchronisation): its scratch is a fixed device array inside the
library.  These tests check that it writes exactly what gqe_attention_prefill
writes (the same kernels on the same work list), on two calls in a row (the
array keeps the first call's contents); that a call allocates no device
memory; that errors found on the device are reported through
gqe_static_device_status; and that a shape too large for the array is
refused.  This file is collected last.
"""
import pytest
import torch

from gpu_util import make_case, upload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402

GQE_ERR_WORKSPACE, GQE_ERR_BAD_INDEX, GQE_ERR_NONFINITE = 5, 6, 7


def _with_workspace(shape, seed):
    B, S, N, G, k, d, dm = shape
    inp = make_case(B, S, N, G, k, d, dm, seed)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm)
    L.forward(dev["x"], dev["W_r"], None, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    return dev, L


def _static_into(L, dev):
    out = torch.full_like(L.concat, float("nan"))
    L.attention_static(dev["Q"], dev["Qs"], dev["K"], dev["V"], out=out)
    torch.cuda.synchronize()
    return out


def test_static_matches_workspace_call_twice():
    # two different shapes back to back: the second call must not see the
    # first call's leftovers in the shared array
    GqePrefill.static_device_status(clear=True)
    for shape, seed in (((2, 300, 16, 8, 2, 64, 64), 900), ((1, 1000, 16, 8, 1, 64, 128), 901)):
        dev, L = _with_workspace(shape, seed)
        got = _static_into(L, dev)
        assert torch.equal(got, L.concat), f"static differs from the workspace call {shape}"
        assert GqePrefill.static_device_status() == 0


def test_static_call_allocates_no_device_memory():
    dev, L = _with_workspace((1, 700, 16, 8, 1, 64, 64), 902)
    out = torch.empty_like(L.concat)
    L.attention_static(dev["Q"], dev["Qs"], dev["K"], dev["V"], out=out)  # warm-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    reserved0 = torch.cuda.memory_reserved()
    L.attention_static(dev["Q"], dev["Qs"], dev["K"], dev["V"], out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert torch.equal(out, L.concat)


def test_static_reports_device_errors():
    dev, L = _with_workspace((1, 260, 16, 8, 1, 64, 64), 903)
    GqePrefill.static_device_status(clear=True)
    # V beyond the fp16 range: the V conversion latches GQE_ERR_NONFINITE
    V = dev["V"].clone()
    V[0, 5, 3, 7] = 1.0e5
    _static_into(L, dict(dev, V=V))
    assert GqePrefill.static_device_status(clear=False) == GQE_ERR_NONFINITE
    assert GqePrefill.static_device_status(clear=True) == GQE_ERR_NONFINITE  # still latched
    assert GqePrefill.static_device_status() == 0                            # cleared
    # an expert index outside [0, M): the bucketing latches GQE_ERR_BAD_INDEX
    L.topk_idx[0, 17, 2, 0] = L.M
    _static_into(L, dev)
    assert GqePrefill.static_device_status() == GQE_ERR_BAD_INDEX
    # and a clean call afterwards reports nothing
    L.forward(dev["x"], dev["W_r"], None, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0
    got = _static_into(L, dev)
    assert GqePrefill.static_device_status() == 0
    assert torch.equal(got, L.concat)


def test_static_rejects_shape_beyond_its_array():
    # S = 1M tokens needs ~1 GiB of fp16 V: more than the fixed array holds
    dm = gqe.dims(1, 1 << 20, 16, 8, 1, 64, 1024, 1)
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    r = gqe.gqe_attention_prefill_static(dm, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                         17 * 64, check=False)
    assert r == GQE_ERR_WORKSPACE
