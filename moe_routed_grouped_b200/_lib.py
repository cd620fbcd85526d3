"""ctypes binding of libgqe.so (argument marshalling only).

Every function here has the name and argument order of the C entry point in
``include/gqe.h``; tensors are passed as raw device pointers.  Nothing is
computed in Python: if the library cannot be loaded, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgqe.so")

EXPORTS = (
    "gqe_workspace_size", "gqe_route", "gqe_bucket", "gqe_attention_prefill",
    "gqe_dense_gqa_prefill", "gqe_get_device_status", "gqe_kv_cache_bytes",
    "gqe_status_string", "gqe_selftest_bounded_wait", "gqe_set_profile_events",
    "gqe_attention_prefill_static", "gqe_set_pair_threshold", "gqe_set_router_resident", "gqe_decode_workspace_size",
    "gqe_attention_decode", "gqe_append_workspace_size", "gqe_attention_append",
    "gqe_static_device_status", "gqe_linear", "gqe_routed_q_project", "gqe_layer_prefill",
    "gqe_dense_layer_prefill", "gqe_prefill_chunk_workspace_size", "gqe_attention_prefill_chunk",
    "gqe_attention_prefill_train", "gqe_prefill_backward_workspace_size", "gqe_prefill_backward",
)

STATUS = {0: "GQE_OK", 1: "GQE_ERR_INVALID_ARG", 2: "GQE_ERR_UNSUPPORTED", 3: "GQE_ERR_CUDA",
          4: "GQE_ERR_TIMEOUT", 5: "GQE_ERR_WORKSPACE", 6: "GQE_ERR_BAD_INDEX",
          7: "GQE_ERR_NONFINITE", 8: "GQE_ERR_BAD_POSITION"}


class GqeDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("S", ctypes.c_int32), ("N", ctypes.c_int32),
                ("G", ctypes.c_int32), ("k", ctypes.c_int32), ("d", ctypes.c_int32),
                ("d_model", ctypes.c_int32), ("out_fp32", ctypes.c_int32)]


class GqeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgqe.so not built ({LIB_PATH}); run moe_routed_grouped_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I32, I64, SZ = ctypes.c_void_p, ctypes.POINTER(GqeDims), ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "gqe_workspace_size": (SZ, [S]),
        "gqe_route": (I32, [S, P, P, P, P, P, P, P, SZ, P]),
        "gqe_bucket": (I32, [S, P, P, P, P, SZ, P]),
        "gqe_attention_prefill": (I32, [S, P, P, P, P, P, P, P, P, P, I64, P, SZ, P]),
        "gqe_dense_gqa_prefill": (I32, [S, P, P, P, P, P, SZ, P]),
        "gqe_get_device_status": (I32, [P, I32, P]),
        "gqe_kv_cache_bytes": (ctypes.c_uint64, [I32, I32, I64, I32, I32, I32]),
        "gqe_status_string": (ctypes.c_char_p, [I32]),
        "gqe_selftest_bounded_wait": (I32, [P, SZ, I32, P]),
        "gqe_set_profile_events": (None, [P, P]),
        "gqe_attention_prefill_static": (I32, [S, P, P, P, P, P, P, P, P, P, I64, P]),
        "gqe_set_pair_threshold": (I64, [I64]),
        "gqe_set_router_resident": (I32, [I32]),
        "gqe_decode_workspace_size": (SZ, [S]),
        "gqe_attention_decode": (I32, [S, P, P, P, P, P, P, P, P, P, P, P, I64, P, SZ, P]),
        "gqe_append_workspace_size": (SZ, [S, I32]),
        "gqe_attention_append": (I32, [S, I32, P, P, P, P, P, P, P, P, P, P, P, I64, P, SZ, P]),
        "gqe_static_device_status": (I32, [I32, P]),
        "gqe_linear": (I32, [I32, I32, I32, I32, P, I64, P, P, I64, I32, P]),
        "gqe_routed_q_project": (I32, [S, P, P, P, P, P, SZ, P]),
        "gqe_layer_prefill": (I32, [S] + [P] * 18 + [SZ, P]),
        "gqe_dense_layer_prefill": (I32, [S] + [P] * 11 + [SZ, P]),
        "gqe_prefill_chunk_workspace_size": (SZ, [S, I32]),
        "gqe_attention_prefill_chunk": (I32, [S, I32] + [P] * 11 + [I64, P, SZ, P]),
        "gqe_attention_prefill_train": (I32, [S] + [P] * 9 + [I64, P, P, P, SZ, P]),
        "gqe_prefill_backward_workspace_size": (SZ, [S]),
        "gqe_prefill_backward": (I32, [S] + [P] * 8 + [I64, P, P, P, P, P, I64] + [P] * 5
                                 + [P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    """A cudaStream_t: an int handle, a torch.cuda.Stream, or None for torch's
    current stream on the current device (so calls order with the caller's
    torch work and can be captured into a CUDA graph)."""
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream if isinstance(stream, int) else stream.cuda_stream)


def _check(code: int, where: str) -> int:
    if code != 0:
        raise GqeError(code, where)
    return code


def dims(B, S, N, G, k, d, d_model=8, out_fp32=1) -> GqeDims:
    return GqeDims(B, S, N, G, k, d, d_model, out_fp32)


def gqe_workspace_size(dm: GqeDims) -> int:
    return LIB.gqe_workspace_size(ctypes.byref(dm))


def gqe_route(dm, x, W_r, bias, topk_idx, p, w, ws, stream=None, check=True):
    r = LIB.gqe_route(ctypes.byref(dm), _ptr(x), _ptr(W_r), _ptr(bias), _ptr(topk_idx), _ptr(p),
                      _ptr(w), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_route") if check else r


def gqe_bucket(dm, topk_idx, bucket_off, bucket_tok, ws, stream=None, check=True):
    r = LIB.gqe_bucket(ctypes.byref(dm), _ptr(topk_idx), _ptr(bucket_off), _ptr(bucket_tok),
                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_bucket") if check else r


def gqe_attention_prefill(dm, Q, Qs, K, V, topk_idx, w, O_sel, o_bar, s_out, out_row_stride,
                          ws, stream=None, check=True):
    r = LIB.gqe_attention_prefill(ctypes.byref(dm), _ptr(Q), _ptr(Qs), _ptr(K), _ptr(V),
                                  _ptr(topk_idx), _ptr(w), _ptr(O_sel), _ptr(o_bar), _ptr(s_out),
                                  int(out_row_stride), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream))
    return _check(r, "gqe_attention_prefill") if check else r


def gqe_dense_gqa_prefill(dm, Q, K, V, O, ws, stream=None, check=True):
    r = LIB.gqe_dense_gqa_prefill(ctypes.byref(dm), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_dense_gqa_prefill") if check else r


def gqe_get_device_status(ws, clear=1, stream=None) -> int:
    return LIB.gqe_get_device_status(_ptr(ws), int(clear), _stream(stream))


def gqe_kv_cache_bytes(L, G, S, d, bytes_per_elem, B=1) -> int:
    return LIB.gqe_kv_cache_bytes(L, G, S, d, bytes_per_elem, B)


def gqe_status_string(code: int) -> str:
    return LIB.gqe_status_string(code).decode()


def gqe_selftest_bounded_wait(ws, limit_us, stream=None, check=True):
    r = LIB.gqe_selftest_bounded_wait(_ptr(ws), ws.numel() * ws.element_size(), int(limit_us),
                                      _stream(stream))
    return _check(r, "gqe_selftest_bounded_wait") if check else r


def gqe_set_profile_events(begin=None, end=None):
    """begin/end: torch.cuda.Event (already recorded once) or None."""
    b = None if begin is None else ctypes.c_void_p(begin.cuda_event)
    e = None if end is None else ctypes.c_void_p(end.cuda_event)
    LIB.gqe_set_profile_events(b, e)


def gqe_set_pair_threshold(kv_bytes):
    """Working-set size (bytes) from which d = 64 attention uses the pair
    kernel (0: always, negative: never); returns the previous value."""
    return int(LIB.gqe_set_pair_threshold(int(kv_bytes)))


def gqe_set_router_resident(on):
    """1: the W_r-resident router whenever W_r fits; 0: by token count (the
    default); negative: read only.  Returns the previous setting."""
    return int(LIB.gqe_set_router_resident(int(on)))


def gqe_attention_prefill_static(dm, Q, Qs, K, V, topk_idx, w, O_sel, o_bar, s_out,
                                 out_row_stride, stream=None, check=True):
    """gqe_attention_prefill without a workspace (scratch in the library)."""
    r = LIB.gqe_attention_prefill_static(ctypes.byref(dm), _ptr(Q), _ptr(Qs), _ptr(K), _ptr(V),
                                         _ptr(topk_idx), _ptr(w), _ptr(O_sel), _ptr(o_bar),
                                         _ptr(s_out), int(out_row_stride), _stream(stream))
    return _check(r, "gqe_attention_prefill_static") if check else r


def gqe_static_device_status(clear=1, stream=None) -> int:
    """Status word of gqe_attention_prefill_static on the current device."""
    return LIB.gqe_static_device_status(int(clear), _stream(stream))


def gqe_prefill_chunk_workspace_size(dm: GqeDims, T: int) -> int:
    return LIB.gqe_prefill_chunk_workspace_size(ctypes.byref(dm), int(T))


def gqe_attention_prefill_chunk(dm, T, Q, Qs, Kc, Vc, q_off, kv_start, topk_idx, w, O_sel, o_bar,
                                s_out, out_row_stride, ws, stream=None, check=True):
    """A chunk of dm.S queries per sequence at q_off[b] + i over caches of T
    slots; q_off / kv_start: device int32 [B] or None."""
    r = LIB.gqe_attention_prefill_chunk(
        ctypes.byref(dm), int(T), _ptr(Q), _ptr(Qs), _ptr(Kc), _ptr(Vc), _ptr(q_off),
        _ptr(kv_start), _ptr(topk_idx), _ptr(w), _ptr(O_sel), _ptr(o_bar), _ptr(s_out),
        int(out_row_stride), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_attention_prefill_chunk") if check else r


def gqe_attention_prefill_train(dm, Q, Qs, K, V, topk_idx, w, O_sel, o_bar, s_out,
                                out_row_stride, lse_sel, lse_s, ws, stream=None, check=True):
    r = LIB.gqe_attention_prefill_train(
        ctypes.byref(dm), _ptr(Q), _ptr(Qs), _ptr(K), _ptr(V), _ptr(topk_idx), _ptr(w),
        _ptr(O_sel), _ptr(o_bar), _ptr(s_out), int(out_row_stride), _ptr(lse_sel), _ptr(lse_s),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_attention_prefill_train") if check else r


def gqe_prefill_backward_workspace_size(dm: GqeDims) -> int:
    return LIB.gqe_prefill_backward_workspace_size(ctypes.byref(dm))


def gqe_prefill_backward(dm, Q, Qs, K, V, topk_idx, w, O_sel, s_out, out_row_stride, lse_sel,
                         lse_s, dO_sel, do_bar, ds, dout_row_stride, dQ, dQs, dK, dV, dw, ws,
                         stream=None, check=True):
    r = LIB.gqe_prefill_backward(
        ctypes.byref(dm), _ptr(Q), _ptr(Qs), _ptr(K), _ptr(V), _ptr(topk_idx), _ptr(w),
        _ptr(O_sel), _ptr(s_out), int(out_row_stride), _ptr(lse_sel), _ptr(lse_s), _ptr(dO_sel),
        _ptr(do_bar), _ptr(ds), int(dout_row_stride), _ptr(dQ), _ptr(dQs), _ptr(dK), _ptr(dV),
        _ptr(dw), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_prefill_backward") if check else r


def gqe_linear(rows, K, nb, nc, A, lda, W, C, ldc, c_fp32, stream=None, check=True):
    """C[rows, nb*nc] = A[rows, :K] . W[nb, K, nc] (stacked along the columns)."""
    r = LIB.gqe_linear(int(rows), int(K), int(nb), int(nc), _ptr(A), int(lda), _ptr(W), _ptr(C),
                       int(ldc), int(c_fp32), _stream(stream))
    return _check(r, "gqe_linear") if check else r


def gqe_routed_q_project(dm, x, W_Q, topk_idx, Q, ws, stream=None, check=True):
    r = LIB.gqe_routed_q_project(ctypes.byref(dm), _ptr(x), _ptr(W_Q), _ptr(topk_idx), _ptr(Q),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_routed_q_project") if check else r


def gqe_layer_prefill(dm, x, W_Q, W_K, W_V, W_s, W_r, bias, W_O, topk_idx, p, w, Q, Qs, K, V,
                      concat, y, ws, stream=None, check=True):
    r = LIB.gqe_layer_prefill(ctypes.byref(dm), *[_ptr(t) for t in (
        x, W_Q, W_K, W_V, W_s, W_r, bias, W_O, topk_idx, p, w, Q, Qs, K, V, concat, y, ws)],
        ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_layer_prefill") if check else r


def gqe_dense_layer_prefill(dm, x, W_Q, W_K, W_V, W_O, Q, K, V, O, y, ws, stream=None,
                            check=True):
    r = LIB.gqe_dense_layer_prefill(ctypes.byref(dm), *[_ptr(t) for t in (
        x, W_Q, W_K, W_V, W_O, Q, K, V, O, y, ws)], ws.numel() * ws.element_size(),
        _stream(stream))
    return _check(r, "gqe_dense_layer_prefill") if check else r


def gqe_decode_workspace_size(dm: GqeDims) -> int:
    return LIB.gqe_decode_workspace_size(ctypes.byref(dm))


def gqe_attention_decode(dm, Q, Qs, Kc, Vc, pos, kv_start, topk_idx, w, O_sel, o_bar, s_out,
                         out_row_stride, ws, stream=None, check=True):
    """One decode step; dm.S is the cache capacity T; kv_start may be None."""
    r = LIB.gqe_attention_decode(ctypes.byref(dm), _ptr(Q), _ptr(Qs), _ptr(Kc), _ptr(Vc),
                                 _ptr(pos), _ptr(kv_start), _ptr(topk_idx), _ptr(w), _ptr(O_sel),
                                 _ptr(o_bar),
                                 _ptr(s_out), int(out_row_stride), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_attention_decode") if check else r


def gqe_append_workspace_size(dm: GqeDims, n_new: int) -> int:
    return LIB.gqe_append_workspace_size(ctypes.byref(dm), int(n_new))


def gqe_attention_append(dm, n_new, Q, Qs, Kc, Vc, pos, kv_start, topk_idx, w, O_sel, o_bar,
                         s_out, out_row_stride, ws, stream=None, check=True):
    """n_new new tokens per sequence over the caches; dm.S is the capacity T."""
    r = LIB.gqe_attention_append(ctypes.byref(dm), int(n_new), _ptr(Q), _ptr(Qs), _ptr(Kc),
                                 _ptr(Vc), _ptr(pos), _ptr(kv_start), _ptr(topk_idx), _ptr(w),
                                 _ptr(O_sel), _ptr(o_bar), _ptr(s_out), int(out_row_stride),
                                 _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    return _check(r, "gqe_attention_append") if check else r
