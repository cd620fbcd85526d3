"""CPU checks of the C-ABI library: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import moe_routed_grouped_b200 as gqe
from moe_routed_grouped_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gqe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gqe_[a-z_]+)\s*\(", src)))


def test_header_symbols_exported():
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.EXPORTS)


def test_kv_cache_bytes_matches_pages():
    # "AI 大模型之 GQA" §4.2 and the MQA/GQA explainer's 数值示例
    assert gqe.gqe_kv_cache_bytes(32, 8, 4096, 128, 2, 1) == 512 * 2 ** 20
    assert gqe.gqe_kv_cache_bytes(32, 32, 4096, 128, 2, 1) == 2048 * 2 ** 20
    assert gqe.gqe_kv_cache_bytes(1, 32, 1024, 128, 2, 1) == 16777216
    assert gqe.gqe_kv_cache_bytes(1, 8, 1024, 128, 2, 1) == 4194304
    assert gqe.gqe_kv_cache_bytes(1, 1, 1024, 128, 2, 1) == 524288
    assert gqe.gqe_kv_cache_bytes(1, 8, 1024, 128, 2, 3) == 3 * 4194304


def test_status_strings():
    for code in range(9):
        assert gqe.gqe_status_string(code)
    assert gqe.gqe_status_string(99) == "unknown status"


FAKE = ctypes.c_void_p(0x10000)  # 16-byte aligned, never dereferenced


def _route(dm, ws_bytes=1 << 40, x=FAKE, ws=FAKE):
    return _lib.LIB.gqe_route(ctypes.byref(dm), x, FAKE, None, FAKE, FAKE, FAKE, ws, ws_bytes,
                              None)


@pytest.mark.parametrize("args,code", [
    ((1, 16, 16, 6, 1, 64, 256), 1),    # N % G != 0 is rejected, not remapped
    ((1, 16, 16, 8, 3, 64, 256), 1),    # k > M
    ((0, 16, 16, 8, 1, 64, 256), 1),    # empty batch
    ((1, 0, 16, 8, 1, 64, 256), 1),     # empty sequence
    ((1, 16, 16, 8, 1, 96, 256), 2),    # head dim outside {64, 128}
    ((1, 16, 16, 8, 1, 64, 250), 2),    # d_model not a multiple of 8
    ((1, 16, 48, 8, 1, 64, 256), 2),    # G*M = 48 not supported by the router
    ((1, 16, 264, 4, 1, 64, 256), 2),   # M = 66 > 32
])
def test_route_rejects_bad_dims(args, code):
    dm = _lib.dims(*args)
    assert _route(dm) == code
    if code == 1:
        assert _lib.gqe_workspace_size(dm) == 0


def test_route_rejects_pointers_and_workspace():
    dm = _lib.dims(1, 16, 16, 8, 1, 64, 256)
    assert _route(dm, x=None) == 1
    assert _route(dm, x=ctypes.c_void_p(0x10008)) == 1            # misaligned
    need = _lib.gqe_workspace_size(dm)
    assert need > 0
    assert _route(dm, ws_bytes=need - 1) == 5
    assert _route(dm, ws=None) == 5


def test_attention_rejects_bad_stride_and_workspace():
    dm = _lib.dims(1, 16, 16, 8, 1, 64, 256)
    L = _lib.LIB
    def call(stride, ws_bytes=1 << 40):
        return L.gqe_attention_prefill(ctypes.byref(dm), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       FAKE, FAKE, stride, FAKE, ws_bytes, None)
    assert call(60) == 1      # not a multiple of 8
    assert call(8) == 1       # shorter than d
    assert call(17 * 64, ws_bytes=10) == 5
    assert L.gqe_dense_gqa_prefill(ctypes.byref(dm), FAKE, FAKE, None, FAKE, FAKE, 1 << 40,
                                   None) == 1


def test_workspace_grows_with_shape():
    a = _lib.gqe_workspace_size(_lib.dims(1, 128, 16, 8, 1, 64, 256))
    b = _lib.gqe_workspace_size(_lib.dims(8, 2048, 16, 8, 1, 64, 1024))
    c = _lib.gqe_workspace_size(_lib.dims(1, 131072, 32, 8, 2, 128, 4096))
    assert 0 < a < b < c


def test_pair_threshold_is_a_host_setting():
    """The d = 64 kernel choice is a process-wide host value: set, read back
    through the previous-value return, restored.  No device is touched."""
    prev = gqe.gqe_set_pair_threshold(1 << 20)
    try:
        assert gqe.gqe_set_pair_threshold(0) == 1 << 20
        assert gqe.gqe_set_pair_threshold(-1) == 0
        assert gqe.gqe_set_pair_threshold(96 << 20) == -1
    finally:
        gqe.gqe_set_pair_threshold(prev)
    assert prev == 96 << 20  # the default: 96 MiB of K/V


def test_router_resident_is_a_host_setting():
    """The router kernel choice: default 0 (by token count), set, read back
    through the previous-value return (a negative value only reads),
    restored.  No device is touched."""
    prev = gqe.gqe_set_router_resident(-1)
    assert prev == 0
    try:
        assert gqe.gqe_set_router_resident(1) == 0
        assert gqe.gqe_set_router_resident(-1) == 1
        assert gqe.gqe_set_router_resident(0) == 1
    finally:
        gqe.gqe_set_router_resident(prev)
    assert gqe.gqe_set_router_resident(-1) == 0



def test_decode_rejects_bad_arguments():
    """gqe_attention_decode validates before launching (dims.S is the cache
    capacity T); nothing here reaches a device."""
    dm = _lib.dims(2, 4096, 16, 8, 1, 64)
    L = _lib.LIB
    need = _lib.gqe_decode_workspace_size(dm)
    assert need > 512

    def call(stride=17 * 64, ws_bytes=1 << 40, pos=FAKE, d=dm, start=None):
        return L.gqe_attention_decode(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, pos, start, FAKE,
                                      FAKE, FAKE, FAKE, FAKE, stride, FAKE, ws_bytes, None)
    assert call(stride=60) == 1                      # not a multiple of 8
    assert call(pos=None) == 1                       # positions are required
    assert call(pos=ctypes.c_void_p(0x10004)) == 1   # misaligned
    assert call(start=ctypes.c_void_p(0x10004)) == 1  # misaligned first-slot array
    assert call(ws_bytes=need - 1) == 5
    assert call(d=_lib.dims(2, 4096, 16, 8, 3, 64)) == 1   # k > M
    assert call(d=_lib.dims(2, 4096, 16, 8, 1, 96)) == 2   # head dim outside {64, 128}
    assert _lib.gqe_decode_workspace_size(_lib.dims(2, 4096, 16, 8, 3, 64)) == 0


def test_decode_workspace_scales_with_the_split():
    """The split-KV scratch holds (max, sum, d outputs) per head slot (k
    routed + shared) and chunk; chunks are at least 256 keys, so a short
    cache has one chunk, and the router's counters (bytes 256..511) stay out
    of the decode scratch."""
    one = _lib.gqe_decode_workspace_size(_lib.dims(1, 200, 16, 8, 1, 64))
    # one chunk: 8 groups x 2 slots x (1 + 1 + 64) floats, each block 256-aligned
    assert one == 512 + 256 + 256 + 8 * 2 * 64 * 4
    long = _lib.gqe_decode_workspace_size(_lib.dims(1, 32768, 16, 8, 1, 64))
    wide = _lib.gqe_decode_workspace_size(_lib.dims(1, 32768, 32, 8, 2, 128))
    assert one < long < wide
    # the scratch does not grow past the CTA target once chunks are long
    assert _lib.gqe_decode_workspace_size(_lib.dims(1, 1 << 20, 16, 8, 1, 64)) <= 2 * long


def _decode_chunks(B, T, N, G, k, d, n_new):
    """Chunks per (b, g) of the decode plan, read back from the workspace
    size: 512 header bytes, then per-(slot, chunk) maxima, sums and d
    outputs in float32, each block 256-byte aligned."""
    dm = _lib.dims(B, T, N, G, k, d)
    total = (_lib.gqe_decode_workspace_size(dm) if n_new == 1
             else _lib.gqe_append_workspace_size(dm, n_new))
    if total == 0:  # a shape the library refuses (size limits): never launched
        return None
    up = lambda x: (x + 255) // 256 * 256
    per = B * G * (k + 1) * n_new
    for nc in range(1, 4097):
        parts = per * nc
        if 512 + 2 * up(4 * parts) + up(4 * parts * d) == total:
            return nc
    raise AssertionError(f"no chunk count gives {total} bytes")


def test_decode_chunks_stay_within_the_merge_staging():
    """The merge kernel stages a head's chunk maxima and sums in a fixed
    shared-memory array of 592 entries (the plan's CTA target), so no shape
    may split a (b, g) into more chunks than that."""
    worst, refused = 0, 0
    for B in (1, 2, 3, 8, 64):
        for T in (1, 255, 256, 257, 4096, 32768, 100003, 1 << 20, 1 << 22):
            for (N, G, k) in ((16, 8, 1), (32, 8, 2), (4, 1, 2)):
                for d in (64, 128):
                    for n_new in (1, 7, 64):
                        if n_new > T:
                            continue
                        nc = _decode_chunks(B, T, N, G, k, d, n_new)
                        if nc is None:
                            refused += 1
                            continue
                        assert 1 <= nc <= 592, (B, T, N, G, k, d, n_new, nc)
                        assert nc == 1 or T > 256 * (nc - 1)  # chunks hold at least 256 keys
                        worst = max(worst, nc)
    assert worst > 256  # the sweep reaches the long-chunk regime
    assert refused < 30   # only the largest caches are refused


def test_append_rejects_bad_token_counts():
    dm = _lib.dims(2, 100, 16, 8, 1, 64)
    L = _lib.LIB

    def call(n, ws_bytes=1 << 40):
        return L.gqe_attention_append(ctypes.byref(dm), n, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                                      FAKE, FAKE, FAKE, FAKE, FAKE, 17 * 64, FAKE, ws_bytes, None)
    assert call(0) == 1 and call(65) == 1          # 1 <= n_new <= 64
    assert _lib.gqe_append_workspace_size(dm, 0) == 0
    assert _lib.gqe_append_workspace_size(dm, 65) == 0
    small = _lib.dims(2, 10, 16, 8, 1, 64)
    assert _lib.gqe_append_workspace_size(small, 11) == 0   # more new tokens than slots
    need = _lib.gqe_append_workspace_size(dm, 5)
    assert need > _lib.gqe_append_workspace_size(dm, 1) == _lib.gqe_decode_workspace_size(dm)
    assert call(5, ws_bytes=need - 1) == 5


def test_decode_wrapper_buffer_views_on_host():
    """The torch wrapper's buffers and concat views (allocated on the host
    here; nothing is launched): one W_O row per new token, laid out as
    [O_sel | o_bar | shared head]."""
    from moe_routed_grouped_b200.layer import GqeDecode
    B, T, N, G, k, d, dm = 3, 600, 16, 8, 2, 64, 128
    one = GqeDecode(B, T, N, G, k, d, dm, device="cpu")
    assert one.concat.shape == (B, (G * k + G + 1) * d)
    assert one.O_sel().shape == (B, G, k, d) and one.o_bar().shape == (B, G, d)
    assert one.s_out().shape == (B, d) and one.topk_idx.shape == (B, G, k)
    many = GqeDecode(B, T, N, G, k, d, dm, device="cpu", n_new=5)
    assert many.concat.shape == (B * 5, (G * k + G + 1) * d)
    assert many.O_sel().shape == (B, 5, G, k, d) and many.s_out().shape == (B, 5, d)
    assert many.topk_idx.shape == (B, 5, G, k) and many.p.shape == (B, 5, G, N // G)
    # the views alias the concat buffer in its column order
    many.concat.zero_()
    many.o_bar()[1, 2, 3] = 1.0
    row = many.concat[1 * 5 + 2]
    assert row[G * k * d + 3 * d: G * k * d + 4 * d].eq(1).all() and row.sum() == d
    assert many.ws.numel() >= gqe.gqe_append_workspace_size(many.dims, 5)
    with pytest.raises(gqe.GqeError):
        GqeDecode(B, T, N, G, k, d, dm, device="cpu", n_new=65)


def test_prefill_wrapper_buffer_views_on_host():
    """GqePrefill's concat buffer (host allocation, nothing launched): slot j
    of group g at (g*k + j)*d, then o_bar per group, then the shared head."""
    from moe_routed_grouped_b200.layer import GqePrefill
    B, S, N, G, k, d, dm = 2, 130, 16, 4, 3, 64, 64
    L = GqePrefill(B, S, N, G, k, d, dm, device="cpu")
    width = (G * k + G + 1) * d
    assert L.concat.shape == (B * S, width)
    assert L.O_sel().shape == (B, S, G, k, d) and L.o_bar().shape == (B, S, G, d)
    assert L.s_out().shape == (B, S, d)
    L.concat.zero_()
    L.O_sel()[1, 7, 2, 1] = 2.0
    L.s_out()[1, 7] = 3.0
    row = L.concat[1 * S + 7]
    assert row[(2 * k + 1) * d:(2 * k + 2) * d].eq(2).all()
    assert row[width - d:].eq(3).all() and row.sum() == 5 * d
    assert L.ws.numel() == gqe.gqe_workspace_size(L.dims)


def test_wrappers_refuse_wrong_tensors_before_any_call():
    """Raw pointers carry no shape, so the torch wrappers check each tensor's
    shape, dtype, layout and device first (host tensors here; nothing is
    launched)."""
    import torch
    from moe_routed_grouped_b200.layer import GqeDecode, GqePrefill
    B, S, N, G, k, d, dm = 1, 64, 16, 8, 1, 64, 64
    L = GqePrefill(B, S, N, G, k, d, dm, device="cpu")
    bf = torch.bfloat16
    x = torch.zeros(B, S, dm, dtype=bf)
    W = torch.zeros(G, dm, N // G, dtype=bf)
    with pytest.raises(ValueError, match="x: shape"):
        L.route(torch.zeros(B, S + 1, dm, dtype=bf), W)
    with pytest.raises(ValueError, match="W_r: dtype"):
        L.route(x, W.float())
    with pytest.raises(ValueError, match="bias: dtype"):
        L.route(x, W, torch.zeros(G, N // G, dtype=torch.float64))
    Q = torch.zeros(B, S, N, d, dtype=bf)
    K = torch.zeros(B, S, G, d, dtype=bf)
    with pytest.raises(ValueError, match="Q: must be contiguous"):
        L.attention(Q.transpose(1, 2).contiguous().transpose(1, 2), torch.zeros(B, S, d, dtype=bf),
                    K, K)
    with pytest.raises(ValueError, match="V: shape"):
        L.dense(Q, K, torch.zeros(B, S, G, d + 1, dtype=bf))
    with pytest.raises(TypeError):
        L.dense(Q, K, object())
    D = GqeDecode(2, 100, N, G, k, d, dm, device="cpu")
    with pytest.raises(ValueError, match="pos: dtype"):
        D.attention(torch.zeros(2, N, d, dtype=bf), torch.zeros(2, d, dtype=bf),
                    torch.zeros(2, 100, G, d, dtype=bf), torch.zeros(2, 100, G, d, dtype=bf),
                    torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError, match="Kc: shape"):
        D.attention(torch.zeros(2, N, d, dtype=bf), torch.zeros(2, d, dtype=bf),
                    torch.zeros(2, 99, G, d, dtype=bf), torch.zeros(2, 100, G, d, dtype=bf),
                    torch.zeros(2, dtype=torch.int32))
    A = GqeDecode(2, 100, N, G, k, d, dm, device="cpu", n_new=3)
    with pytest.raises(ValueError, match="x: shape"):
        A.route(torch.zeros(2, dm, dtype=bf), W)      # needs the n_new axis
