"""Full-size workloads in the launch configuration the bench times.

Routing is compared bit for bit over every token; attention outputs are
compared on sampled rows (first and last 128 positions plus seeded random
ones) that the oracle computes one by one.  All four long workloads run by
default, the 131k-token d = 128, k = 2 one and the 1M-token one (the pair
kernel) included.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_close, dev_bf16
from synth import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from moe_routed_grouped_b200.layer import GqePrefill  # noqa: E402

def _rows(S, seed, n_rand=128):
    rng = np.random.default_rng(seed)
    r = np.concatenate([np.arange(min(128, S)), np.arange(max(0, S - 128), S),
                        rng.integers(0, S, n_rand)])
    return np.unique(r)


@pytest.mark.parametrize("name", ["layer250m", "imbalanced32k", "wide131k", "million"])
def test_workload_sampled_parity(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    bias = inp.get("bias")
    L = GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True)
    dev = {k: dev_bf16(v) for k, v in inp.items() if k != "bias"}
    dbias = None if bias is None else torch.from_numpy(bias).cuda()
    L.forward(dev["x"], dev["W_r"], dbias, dev["Q"], dev["Qs"], dev["K"], dev["V"])
    O_dense = L.dense(dev["Q"], dev["K"], dev["V"])
    torch.cuda.synchronize()
    assert L.device_status() == 0

    idx, p, wts, n_exact = oracle.route(inp["x"], inp["W_r"], bias, w.k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx), "top-k differs"
    check_close(L.w.cpu().numpy(), wts, "w", atol=1e-5, rtol_l2=1e-5)
    if w.bias0:
        share0 = float((idx[..., 0] == 0).mean())
        assert 0.75 < share0 < 0.95, share0   # the biased split of the workload

    rows = [_rows(w.S, 10 * w.cid + b, n_rand=96 if w.S >= 1 << 20 else 128) for b in range(w.B)]
    O_sel, o_bar, s = oracle.gqe_prefill_rows(inp["Q"], inp["Qs"], inp["K"], inp["V"], idx,
                                              wts, rows)
    dense = oracle.dense_gqa(inp["Q"], inp["K"], inp["V"], rows=rows)
    go, gb, gs = L.O_sel().cpu().numpy(), L.o_bar().cpu().numpy(), L.s_out().cpu().numpy()
    gd = O_dense.cpu().numpy()
    for b in range(w.B):
        r = rows[b]
        check_close(go[b, r], O_sel[b], f"O_sel b={b}")
        check_close(gb[b, r], o_bar[b], f"o_bar b={b}")
        check_close(gs[b, r], s[b], f"s b={b}")
        check_close(gd[b, r], dense[b], f"dense b={b}")
