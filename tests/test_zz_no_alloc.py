"""gqe_attention_prefill_static: the attention call that needs no workspace.

It exists for callers that cannot allocate device memory (a plugin whose host
framework owns every allocation, or a loop that must not pay cudaMalloc's
device-wide synchronisation): its scratch is a fixed device array inside the
library.  These tests check that it writes what gqe_attention_prefill writes,
on two calls in a row (the array keeps the first call's contents), and that a
shape too large for the array is refused.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from gpu_util import check_close, make_case, upload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402


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
    a = L.G * L.k * L.d
    gqe.gqe_attention_prefill_static(L.dims, dev["Q"], dev["Qs"], dev["K"], dev["V"],
                                     L.topk_idx, L.w, out, out.view(-1)[a:],
                                     out.view(-1)[a + L.G * L.d:], L.row)
    torch.cuda.synchronize()
    return out


def test_static_matches_workspace_call_twice():
    # two different shapes back to back: the second call must not see the
    # first call's leftovers in the shared array
    for shape, seed in (((2, 300, 16, 8, 2, 64, 64), 900), ((1, 1000, 16, 8, 1, 64, 128), 901)):
        dev, L = _with_workspace(shape, seed)
        got = _static_into(L, dev)
        check_close(got.cpu().numpy(), L.concat.cpu().numpy(), f"static vs workspace {shape}")


def test_static_rejects_shape_beyond_its_array():
    # S = 1M tokens needs ~1 GiB of fp16 V: more than the fixed array holds
    dm = gqe.dims(1, 1 << 20, 16, 8, 1, 64, 1024, 1)
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    r = gqe.gqe_attention_prefill_static(dm, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                         17 * 64, check=False)
    assert r == 5  # GQE_ERR_WORKSPACE
