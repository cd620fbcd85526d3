"""Backward pass of the prefill path on the GPU (gqe_attention_prefill_train,
gqe_prefill_backward) against the oracle's gqe_prefill_backward.

The oracle follows "AI 大模型之 GQA", 训练与部署 共享键值的梯度归约 (per-head
attention backward; the gradients of a KV head are the SUM over every head
that reads it) and the weighted-sum slot of the GQE review (§二 三个关键部件:
slot j receives dO_sel_j + w_j d(o_bar); dw_j = <d(o_bar), o_j>); it is pinned
by central finite differences on the CPU.

Tolerance, from the arithmetic: the tensor-core products take bf16 operands,
so the effective dO, P and dS are each rounded to bf16 (relative error at
most 2^-9 each, float32 accumulation); the gradients are held to 1e-2
relative L2 and 2e-2 of their largest magnitude elementwise.  dw is a float32
dot product with the forward's output o_j, so it carries the forward's 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle.gqe_oracle as og
from gpu_util import check_close, make_case, upload
from synth import normal_bf16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402

SHAPES = [(2, 300, 16, 8, 1, 64, 64, 0.0), (1, 260, 8, 4, 2, 64, 64, 0.0),
          (1, 200, 8, 2, 2, 128, 64, 0.0), (2, 257, 16, 8, 1, 64, 128, 1.5)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda v: "x".join(map(str, v)))
def test_backward_matches_oracle(shape):
    B, S, N, G, k, d, dm, bias0 = shape
    inp = make_case(B, S, N, G, k, d, dm, 51000 + S + d, bias0=bias0)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm)
    L.forward_train(dev["x"], dev["W_r"], dev["bias"], dev["Q"], dev["Qs"], dev["K"], dev["V"])
    row = L.row
    dcat_bits = normal_bf16((B * S, row), 52000 + S)
    dcat = og.bf16_to_f64(dcat_bits)
    grads = L.backward(torch.from_numpy(dcat.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    assert L.device_status() == 0
    assert gqe.gqe_get_device_status(L._bws) == 0
    idx = L.topk_idx.cpu().numpy()
    _, _, w, _ = og.route(inp["x"], inp["W_r"], inp["bias"], k)
    a = G * k * d
    ref = og.gqe_prefill_backward(
        og.bf16_to_f64(inp["Q"]), og.bf16_to_f64(inp["Qs"]), og.bf16_to_f64(inp["K"]),
        og.bf16_to_f64(inp["V"]), idx, w, dcat[:, :a].reshape(B, S, G, k, d),
        dcat[:, a:a + G * d].reshape(B, S, G, d), dcat[:, a + G * d:].reshape(B, S, d))
    for name in ("dQ", "dQs", "dK", "dV"):
        got = grads[name].cpu().numpy()
        r = ref[name]
        check_close(got, r, name, atol=2e-2 * float(np.abs(r).max()), rtol_l2=1e-2)
    # dw = <d(o_bar), o_j> reads the forward's o_j, so it carries the forward
    # output's tolerance (relative L2 1e-3)
    check_close(grads["dw"].cpu().numpy(), ref["dw"], "dw",
                atol=1e-3 * float(np.abs(ref["dw"]).max()) + 1e-6, rtol_l2=1e-3)


def test_backward_zero_upstream_gives_zero_gradients():
    B, S, N, G, k, d, dm = 1, 200, 16, 8, 2, 64, 64
    inp = make_case(B, S, N, G, k, d, dm, 53000)
    dev = upload(inp)
    L = GqePrefill(B, S, N, G, k, d, dm)
    L.forward_train(dev["x"], dev["W_r"], None, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    grads = L.backward(torch.zeros(B * S, L.row, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    for name, t in grads.items():
        assert torch.count_nonzero(t).item() == 0, name
