"""GPU parity of the decode step (query length 1 over a KV cache) through the
C ABI against the CPU oracle's decode step.

Routing indices must match bit for bit; float32 outputs must be within 1e-2
max-abs and 1e-3 relative L2 of the float64 oracle.  The positions are chosen
on the split-KV chunk edges (the first and last key of a chunk, a single key)
so that the chunk merge is exercised with ragged tails.
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

import moe_routed_grouped_b200 as gqe  # noqa: E402
from moe_routed_grouped_b200.layer import GqeDecode, GqePrefill  # noqa: E402


def _case(B, T, N, G, k, d, dm, seed, bias0=0.0):
    M = N // G
    c = dict(
        x=normal_bf16((B, dm), seed),
        W_r=normal_bf16((G, dm, M), seed + 1, std=dm ** -0.5),
        Q=normal_bf16((B, N, d), seed + 2),
        Qs=normal_bf16((B, d), seed + 3),
        Kc=normal_bf16((B, T, G, d), seed + 4),
        Vc=normal_bf16((B, T, G, d), seed + 5),
        bias=None,
    )
    if bias0:
        b = np.zeros((G, M), np.float32)
        b[:, 0] = bias0
        c["bias"] = b
    return c


def _run(shape, pos, seed, out_fp32=True, bias0=0.0, kv_start=None):
    B, T, N, G, k, d, dm = shape
    c = _case(B, T, N, G, k, d, dm, seed, bias0)
    L = GqeDecode(B, T, N, G, k, d, dm, out_fp32=out_fp32)
    bias = None if c["bias"] is None else torch.from_numpy(c["bias"]).cuda()
    pos_d = torch.tensor(pos, dtype=torch.int32, device="cuda")
    ks_d = None if kv_start is None else torch.tensor(kv_start, dtype=torch.int32, device="cuda")
    L.forward(dev_bf16(c["x"]), dev_bf16(c["W_r"]), bias, dev_bf16(c["Q"]), dev_bf16(c["Qs"]),
              dev_bf16(c["Kc"]), dev_bf16(c["Vc"]), pos_d, ks_d)
    torch.cuda.synchronize()
    return c, L


def _oracle(c, pos, k, kv_start=None):
    return oracle.gqe_decode_step(c["x"], c["W_r"], c["bias"], c["Q"], c["Qs"], c["Kc"], c["Vc"],
                                  np.asarray(pos), k,
                                  kv_start=None if kv_start is None else np.asarray(kv_start))


# (B, T, N, G, k, d, d_model), positions.  With a short cache the chunk is
# 256 keys: positions 255 / 256 are the last key of chunk 0 and the first of
# chunk 1.  k = 1 runs two head slots per CTA, k >= 2 four, k = 5 (six slots
# with the shared head) two passes.
CASES = [
    ((4, 700, 16, 8, 1, 64, 256), [0, 255, 256, 699]),
    ((2, 1000, 32, 8, 2, 128, 512), [999, 517]),
    ((3, 300, 8, 4, 2, 64, 64), [1, 299, 128]),
    ((2, 600, 32, 4, 5, 64, 128), [599, 300]),
    ((1, 1, 16, 8, 1, 64, 64), [0]),
    ((2, 513, 16, 8, 1, 128, 64), [512, 511]),
]


@pytest.mark.parametrize("shape,pos", CASES, ids=lambda v: "x".join(map(str, v)))
def test_decode_parity(shape, pos):
    B, T, N, G, k, d, dm = shape
    c, L = _run(shape, pos, seed=30000 + sum(shape))
    assert L.device_status() == 0
    idx, p, w, O_sel, o_bar, s = _oracle(c, pos, k)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx), "top-k indices differ"
    check_close(L.p.cpu().numpy(), p, "p", atol=1e-5, rtol_l2=1e-5)
    check_close(L.w.cpu().numpy(), w, "w", atol=1e-5, rtol_l2=1e-5)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")
    if k == 1:  # w = 1 exactly, so o_bar is the selected slot bit for bit
        assert torch.equal(L.o_bar(), L.O_sel()[:, :, 0])


def test_decode_long_cache_many_chunks():
    """A 40k cache: chunks longer than the minimum (several hundred keys), a
    biased router, positions inside and at the end of the cache."""
    shape = (2, 40000, 16, 8, 1, 64, 256)
    pos = [39999, 12345]
    c, L = _run(shape, pos, seed=31000, bias0=1.5)
    assert L.device_status() == 0
    idx, p, w, O_sel, o_bar, s = _oracle(c, pos, 1)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


# left padding: (shape, positions, first valid slots); the first slot falls
# inside a chunk, on a chunk edge (256), at 0, and equal to the position
PADDED = [
    ((4, 700, 16, 8, 1, 64, 256), [699, 300, 40, 600], [200, 0, 40, 256]),
    ((2, 1000, 32, 8, 2, 128, 512), [999, 517], [255, 1]),
    ((3, 600, 32, 4, 5, 64, 128), [599, 300, 512], [511, 299, 512]),
]


@pytest.mark.parametrize("shape,pos,kv_start", PADDED, ids=lambda v: "x".join(map(str, v)))
def test_decode_left_padding_parity(shape, pos, kv_start):
    """The causal condition intersected with key validity: sequence b sees
    slots kv_start[b]..pos[b] only."""
    B, T, N, G, k, d, dm = shape
    c, L = _run(shape, pos, seed=35000 + B + T, kv_start=kv_start)
    assert L.device_status() == 0
    idx, p, w, O_sel, o_bar, s = _oracle(c, pos, k, kv_start)
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


def test_decode_bf16_output():
    shape = (2, 700, 32, 8, 2, 128, 256)
    pos = [699, 256]
    c, L = _run(shape, pos, seed=32000, out_fp32=False)
    assert L.device_status() == 0
    _, _, _, O_sel, o_bar, s = _oracle(c, pos, 2)
    # half a bf16 ulp (2^-9 relative) on top of the float32 bound; o_bar is
    # summed from unrounded slots, so the same bound covers it
    for got, ref, what in ((L.O_sel(), O_sel, "O_sel"), (L.o_bar(), o_bar, "o_bar"),
                           (L.s_out(), s, "s")):
        g = got.float().cpu().numpy()
        assert (np.abs(g - ref) <= 1e-2 + 2 ** -9 * np.abs(ref)).all(), what


def test_decode_matches_prefill_rows():
    """Decode at position t over the prefill's own K/V is prefill's row t:
    identical routing, outputs equal within rounding (two different kernels)."""
    B, S, N, G, k, d, dm = 2, 520, 16, 8, 2, 64, 128
    M = N // G
    seed = 33000
    x = normal_bf16((B, S, dm), seed)
    W = normal_bf16((G, dm, M), seed + 1, std=dm ** -0.5)
    Q = normal_bf16((B, S, N, d), seed + 2)
    Qs = normal_bf16((B, S, d), seed + 3)
    K = normal_bf16((B, S, G, d), seed + 4)
    V = normal_bf16((B, S, G, d), seed + 5)
    P = GqePrefill(B, S, N, G, k, d, dm)
    Kd, Vd, Wd = dev_bf16(K), dev_bf16(V), dev_bf16(W)
    P.forward(dev_bf16(x), Wd, None, dev_bf16(Q), dev_bf16(Qs), Kd, Vd)
    D = GqeDecode(B, S, N, G, k, d, dm)
    for t in ([0, 519], [257, 3]):
        b_ = np.arange(B)
        tt = np.array(t)
        D.forward(dev_bf16(x[b_, tt]), Wd, None, dev_bf16(Q[b_, tt]), dev_bf16(Qs[b_, tt]), Kd, Vd,
                  torch.tensor(t, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert D.device_status() == 0
        ti = torch.tensor(t, device="cuda")
        bi = torch.arange(B, device="cuda")
        assert torch.equal(D.topk_idx, P.topk_idx[bi, ti])
        for a, b, what in ((D.O_sel(), P.O_sel()[bi, ti], "O_sel"),
                           (D.o_bar(), P.o_bar()[bi, ti], "o_bar"),
                           (D.s_out(), P.s_out()[bi, ti], "s")):
            # prefill rounds P to fp16 for its tensor-core P.V product
            err = (a - b).abs().max().item()
            assert err <= 5e-3, (what, t, err)
    assert P.device_status() == 0


def test_decode_rejects_bad_position_and_index_on_device():
    """Positions and expert indices live on the device, so the kernels check
    them: an out-of-range value latches a status code, its outputs are NaN,
    and the other sequences are unaffected."""
    B, T, N, G, k, d, dm = 3, 300, 16, 8, 1, 64, 64
    c = _case(B, T, N, G, k, d, dm, 34000)
    L = GqeDecode(B, T, N, G, k, d, dm)
    dev = {n: dev_bf16(c[n]) for n in ("x", "W_r", "Q", "Qs", "Kc", "Vc")}
    L.route(dev["x"], dev["W_r"])
    pos = torch.tensor([T, 5, -1], dtype=torch.int32, device="cuda")
    L.attention(dev["Q"], dev["Qs"], dev["Kc"], dev["Vc"], pos)
    assert L.device_status(clear=True) == 8          # GQE_ERR_BAD_POSITION
    out = L.concat.cpu()
    assert torch.isnan(out[0]).all() and torch.isnan(out[2]).all()
    assert torch.isfinite(out[1]).all()
    ref = _oracle(c, [0, 5, 0], k)
    check_close(L.O_sel()[1].cpu().numpy(), ref[3][1], "O_sel of the valid sequence")

    # a first valid slot after the position is rejected the same way
    L.attention(dev["Q"], dev["Qs"], dev["Kc"], dev["Vc"],
                torch.tensor([7, 5, 9], dtype=torch.int32, device="cuda"),
                torch.tensor([0, 6, 0], dtype=torch.int32, device="cuda"))
    assert L.device_status(clear=True) == 8
    out = L.concat.cpu()
    assert torch.isnan(out[1]).all() and torch.isfinite(out[0]).all()
    assert torch.isfinite(out[2]).all()

    good = torch.tensor([7, 5, 299], dtype=torch.int32, device="cuda")
    L.topk_idx[1, 3, 0] = N // G                     # expert index == M
    L.attention(dev["Q"], dev["Qs"], dev["Kc"], dev["Vc"], good)
    assert L.device_status(clear=True) == 6          # GQE_ERR_BAD_INDEX
    assert torch.isnan(L.O_sel()[1, 3]).all() and torch.isnan(L.o_bar()[1, 3]).all()
    assert torch.isfinite(L.O_sel()[1, :3]).all() and torch.isfinite(L.s_out()).all()
    assert torch.isfinite(L.O_sel()[0]).all() and torch.isfinite(L.O_sel()[2]).all()
    assert L.device_status() == 0


def test_decode_step_replays_as_a_cuda_graph():
    """A captured decode step (router + attention) replayed on new tokens and
    positions gives the same bits as the eager calls on the same inputs."""
    B, T, N, G, k, d, dm = 2, 600, 16, 8, 2, 64, 128
    c = _case(B, T, N, G, k, d, dm, 36000)
    st = {n: dev_bf16(c[n]) for n in ("x", "W_r", "Q", "Qs", "Kc", "Vc")}
    pos = torch.tensor([599, 0], dtype=torch.int32, device="cuda")
    L = GqeDecode(B, T, N, G, k, d, dm)
    g = L.graph(st["x"], st["W_r"], None, st["Q"], st["Qs"], st["Kc"], st["Vc"], pos)
    E = GqeDecode(B, T, N, G, k, d, dm)
    for i, p_ in enumerate(([10, 599], [300, 3], [599, 599])):
        nxt = _case(B, T, N, G, k, d, dm, 36100 + 10 * i)
        for n in ("x", "Q", "Qs"):
            st[n].copy_(dev_bf16(nxt[n]))
        pos.copy_(torch.tensor(p_, dtype=torch.int32))
        g.replay()
        E.forward(st["x"], st["W_r"], None, st["Q"], st["Qs"], st["Kc"], st["Vc"], pos)
        torch.cuda.synchronize()
        assert torch.equal(L.topk_idx, E.topk_idx)
        assert torch.equal(L.concat, E.concat), p_
        ref = oracle.gqe_decode_step(nxt["x"], c["W_r"], None, nxt["Q"], nxt["Qs"], c["Kc"],
                                     c["Vc"], np.asarray(p_), k)
        check_close(L.O_sel().cpu().numpy(), ref[3], "O_sel (graph)")
    assert L.device_status() == 0 and E.device_status() == 0


# several new tokens per sequence (gqe_attention_append): (shape, n_new,
# slot of the first new token, first valid slot or None).  Chunk edges at 256;
# the last case is a whole 64-slot cache written by one call.
APPEND = [
    ((3, 700, 16, 8, 1, 64, 256), 2, [0, 254, 600], None),
    ((2, 1000, 32, 8, 2, 128, 512), 3, [997, 255], [200, 0]),
    ((2, 600, 16, 8, 1, 64, 64), 7, [250, 593], [250, 256]),
    ((1, 300, 32, 4, 5, 64, 128), 2, [298], None),
    ((2, 64, 8, 4, 2, 64, 64), 64, [0, 0], None),
]


@pytest.mark.parametrize("shape,n_new,pos,kv_start", APPEND,
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, (tuple, list))
                         else str(v))
def test_append_parity(shape, n_new, pos, kv_start):
    """New token r of sequence b at slot pos[b] + r sees slots
    kv_start[b]..pos[b] + r: Sq queries at the end of Sk keys."""
    B, T, N, G, k, d, dm = shape
    M = N // G
    seed = 37000 + B + T + n_new
    c = dict(x=normal_bf16((B, n_new, dm), seed),
             W_r=normal_bf16((G, dm, M), seed + 1, std=dm ** -0.5),
             Q=normal_bf16((B, n_new, N, d), seed + 2), Qs=normal_bf16((B, n_new, d), seed + 3),
             Kc=normal_bf16((B, T, G, d), seed + 4), Vc=normal_bf16((B, T, G, d), seed + 5))
    L = GqeDecode(B, T, N, G, k, d, dm, n_new=n_new)
    ks = None if kv_start is None else torch.tensor(kv_start, dtype=torch.int32, device="cuda")
    L.forward(dev_bf16(c["x"]), dev_bf16(c["W_r"]), None, dev_bf16(c["Q"]), dev_bf16(c["Qs"]),
              dev_bf16(c["Kc"]), dev_bf16(c["Vc"]),
              torch.tensor(pos, dtype=torch.int32, device="cuda"), ks)
    torch.cuda.synchronize()
    assert L.device_status() == 0
    idx, p, w, O_sel, o_bar, s = oracle.gqe_append_step(
        c["x"], c["W_r"], None, c["Q"], c["Qs"], c["Kc"], c["Vc"], np.asarray(pos), k,
        kv_start=None if kv_start is None else np.asarray(kv_start))
    assert np.array_equal(L.topk_idx.cpu().numpy(), idx)
    check_close(L.O_sel().cpu().numpy(), O_sel, "O_sel")
    check_close(L.o_bar().cpu().numpy(), o_bar, "o_bar")
    check_close(L.s_out().cpu().numpy(), s, "shared head")


def test_append_matches_decode_steps_and_checks_the_last_slot():
    """An append of n tokens equals n decode steps at the successive slots,
    and a call whose last new token would fall beyond the cache is refused on
    the device."""
    B, T, N, G, k, d, dm, n = 2, 520, 16, 8, 2, 64, 128, 4
    c = dict(x=normal_bf16((B, n, dm), 38000), W_r=normal_bf16((G, dm, 2), 38001, std=dm ** -0.5),
             Q=normal_bf16((B, n, N, d), 38002), Qs=normal_bf16((B, n, d), 38003),
             Kc=normal_bf16((B, T, G, d), 38004), Vc=normal_bf16((B, T, G, d), 38005))
    dv = {key: dev_bf16(v) for key, v in c.items()}
    A = GqeDecode(B, T, N, G, k, d, dm, n_new=n)
    pos = [100, 516]
    A.forward(dv["x"], dv["W_r"], None, dv["Q"], dv["Qs"], dv["Kc"], dv["Vc"],
              torch.tensor(pos, dtype=torch.int32, device="cuda"))
    D = GqeDecode(B, T, N, G, k, d, dm)
    for r in range(n):
        D.forward(dv["x"][:, r].contiguous(), dv["W_r"], None, dv["Q"][:, r].contiguous(),
                  dv["Qs"][:, r].contiguous(), dv["Kc"], dv["Vc"],
                  torch.tensor([p_ + r for p_ in pos], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert torch.equal(D.topk_idx, A.topk_idx[:, r])
        assert (D.O_sel() - A.O_sel()[:, r]).abs().max().item() <= 1e-5
        assert (D.s_out() - A.s_out()[:, r]).abs().max().item() <= 1e-5
    assert A.device_status() == 0 and D.device_status() == 0
    A.attention(dv["Q"], dv["Qs"], dv["Kc"], dv["Vc"],
                torch.tensor([100, 517], dtype=torch.int32, device="cuda"))  # 517 + 3 = T
    assert A.device_status(clear=True) == 8
    out = A.concat.view(B, n, -1).cpu()
    assert torch.isnan(out[1]).all() and torch.isfinite(out[0]).all()
