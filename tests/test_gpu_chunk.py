"""Chunked and left-padded prefill on the tensor-core attention kernel
(gqe_attention_prefill_chunk) against the oracle's append step.

"AI 大模型之 GQA", 工程实操 非方形因果遮罩: S new queries at the end of the
keys, the mask taken on absolute positions; step 4: the causal condition
intersected with key validity.  Row i of sequence b sits at q_off[b] + i and
sees slots kv_start[b]..q_off[b] + i.  The oracle's append step computes each
row as its own decode step over the same caches.  Chunks here are longer
than the decode kernels' 64-token limit.  Rows before kv_start[b] (padding)
see no key: they must come back as zeros.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_close, dev_bf16
from synth import normal_bf16

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from moe_routed_grouped_b200.layer import GqeChunk, GqePrefill  # noqa: E402

GQE_ERR_BAD_POSITION = 8


def _case(B, S, T, N, G, k, d, dm, seed):
    M = N // G
    return dict(x=normal_bf16((B, S, dm), seed), W_r=normal_bf16((G, dm, M), seed + 1, std=dm ** -0.5),
                Q=normal_bf16((B, S, N, d), seed + 2), Qs=normal_bf16((B, S, d), seed + 3),
                Kc=normal_bf16((B, T, G, d), seed + 4), Vc=normal_bf16((B, T, G, d), seed + 5))


def _i32(v):
    return None if v is None else torch.tensor(v, dtype=torch.int32, device="cuda")


# (B, S chunk, T cache, N, G, k, d, d_model), q_off, kv_start
CHUNKS = [
    ((2, 300, 700, 16, 8, 1, 64, 128), [100, 400], None),
    ((2, 300, 700, 16, 8, 1, 64, 128), [0, 383], [37, 500]),
    ((1, 260, 520, 32, 8, 2, 128, 256), [260], [129]),
    ((3, 129, 129, 16, 4, 3, 64, 64), [0, 0, 0], [0, 1, 128]),   # left-padded plain prefill
]


@pytest.mark.parametrize("shape,q_off,kv_start", CHUNKS,
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, (tuple, list))
                         else str(v))
def test_chunk_parity(shape, q_off, kv_start):
    B, S, T, N, G, k, d, dm = shape
    c = _case(B, S, T, N, G, k, d, dm, 41000 + S + T)
    L = GqeChunk(B, S, T, N, G, k, d, dm)
    L.forward(dev_bf16(c["x"]), dev_bf16(c["W_r"]), None, dev_bf16(c["Q"]), dev_bf16(c["Qs"]),
              dev_bf16(c["Kc"]), dev_bf16(c["Vc"]), _i32(q_off), _i32(kv_start))
    torch.cuda.synchronize()
    assert L.device_status() == 0
    idx, p, w, O_sel, o_bar, s = oracle.gqe_append_step(
        c["x"], c["W_r"], None, c["Q"], c["Qs"], c["Kc"], c["Vc"], np.asarray(q_off), k,
        kv_start=None if kv_start is None else np.asarray(kv_start))
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    go, gb, gs = L.O_sel().cpu().numpy(), L.o_bar().cpu().numpy(), L.s_out().cpu().numpy()
    ks = np.zeros(B, np.int64) if kv_start is None else np.asarray(kv_start)
    for b in range(B):
        valid = q_off[b] + np.arange(S) >= ks[b]
        check_close(go[b, valid], O_sel[b, valid], f"O_sel b={b}")
        check_close(gb[b, valid], o_bar[b, valid], f"o_bar b={b}")
        check_close(gs[b, valid], s[b, valid], f"shared b={b}")
        assert (go[b, ~valid] == 0).all() and (gs[b, ~valid] == 0).all(), "padding rows not zero"


def test_chunk_without_offsets_is_the_plain_prefill():
    """q_off = kv_start = None and T = S: bit for bit gqe_attention_prefill."""
    B, S, N, G, k, d, dm = 2, 333, 16, 8, 2, 64, 128
    c = _case(B, S, S, N, G, k, d, dm, 42000)
    dv = {n: dev_bf16(v) for n, v in c.items()}
    P = GqePrefill(B, S, N, G, k, d, dm)
    P.forward(dv["x"], dv["W_r"], None, dv["Q"], dv["Qs"], dv["Kc"], dv["Vc"])
    C = GqeChunk(B, S, S, N, G, k, d, dm)
    C.forward(dv["x"], dv["W_r"], None, dv["Q"], dv["Qs"], dv["Kc"], dv["Vc"])
    torch.cuda.synchronize()
    assert P.device_status() == 0 and C.device_status() == 0
    assert torch.equal(P.concat, C.concat)


def test_chunk_offset_out_of_range_is_reported():
    B, S, T, N, G, k, d, dm = 1, 200, 300, 16, 8, 1, 64, 64
    c = _case(B, S, T, N, G, k, d, dm, 43000)
    L = GqeChunk(B, S, T, N, G, k, d, dm)
    L.forward(dev_bf16(c["x"]), dev_bf16(c["W_r"]), None, dev_bf16(c["Q"]), dev_bf16(c["Qs"]),
              dev_bf16(c["Kc"]), dev_bf16(c["Vc"]), _i32([T - S + 1]), None)
    torch.cuda.synchronize()
    assert L.device_status() == GQE_ERR_BAD_POSITION
    assert torch.isfinite(L.concat).all()   # taken as q_off = 0: a defined result
