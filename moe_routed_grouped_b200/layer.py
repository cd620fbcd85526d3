"""Torch-facing wrapper: owns the device buffers of one GQE prefill shape and
calls the C ABI.  Allocation and argument marshalling only; every step of the
computation runs in libgqe.so."""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib


def _device(device) -> torch.device:
    dev = torch.device(device)
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return dev


def _expect(t, name, shape, dtype, device):
    """The C ABI takes raw pointers and cannot see shapes, so each tensor is
    checked here: a wrong shape would otherwise be read out of bounds."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


class GqePrefill:
    """Buffers and calls for one (B, S, N, G, k, d, d_model) shape.

    ``concat`` is the W_O input buffer, one row of (G*k + G + 1)*d elements per
    token: [O_sel (G*k*d, slot j of group g at (g*k + j)*d) | o_bar (G*d) |
    shared head (d)].
    """

    def __init__(self, B, S, N, G, k, d, d_model, out_fp32=True, device="cuda"):
        if N % G:
            raise ValueError("N must be a multiple of G")
        self.B, self.S, self.N, self.G, self.k, self.d, self.d_model = B, S, N, G, k, d, d_model
        self.M = N // G
        self.dims = _lib.dims(B, S, N, G, k, d, d_model, 1 if out_fp32 else 0)
        nbytes = _lib.gqe_workspace_size(self.dims)
        if nbytes == 0:
            raise _lib.GqeError(2, "gqe_workspace_size")
        dev = _device(device)
        self.device = dev
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.out_dtype = torch.float32 if out_fp32 else torch.bfloat16
        self.row = (G * k + G + 1) * d
        self.concat = torch.empty(B * S, self.row, dtype=self.out_dtype, device=dev)
        self.topk_idx = torch.empty(B, S, G, k, dtype=torch.int32, device=dev)
        self.p = torch.empty(B, S, G, self.M, dtype=torch.float32, device=dev)
        self.w = torch.empty(B, S, G, k, dtype=torch.float32, device=dev)
        self._dense_out: Optional[torch.Tensor] = None

    # views of the concat buffer
    def O_sel(self):
        return self.concat[:, : self.G * self.k * self.d].view(self.B, self.S, self.G, self.k, self.d)

    def o_bar(self):
        a = self.G * self.k * self.d
        return self.concat[:, a: a + self.G * self.d].view(self.B, self.S, self.G, self.d)

    def s_out(self):
        return self.concat[:, (self.G * self.k + self.G) * self.d:].view(self.B, self.S, self.d)

    def route(self, x, W_r, bias=None, stream=None):
        bf, dv = torch.bfloat16, self.device
        _expect(x, "x", (self.B, self.S, self.d_model), bf, dv)
        _expect(W_r, "W_r", (self.G, self.d_model, self.M), bf, dv)
        if bias is not None:
            _expect(bias, "bias", (self.G, self.M), torch.float32, dv)
        _lib.gqe_route(self.dims, x, W_r, bias, self.topk_idx, self.p, self.w, self.ws, stream)
        return self.topk_idx, self.p, self.w

    def _check_qkv(self, Q, K, V, Qs=None):
        bf, dv = torch.bfloat16, self.device
        _expect(Q, "Q", (self.B, self.S, self.N, self.d), bf, dv)
        _expect(K, "K", (self.B, self.S, self.G, self.d), bf, dv)
        _expect(V, "V", (self.B, self.S, self.G, self.d), bf, dv)
        if Qs is not None:
            _expect(Qs, "Qs", (self.B, self.S, self.d), bf, dv)

    def attention(self, Q, Qs, K, V, stream=None):
        self._check_qkv(Q, K, V, Qs)
        a = self.G * self.k * self.d
        base = self.concat
        esz = base.element_size()
        o_bar = base.view(-1)[a:]
        s_out = base.view(-1)[a + self.G * self.d:]
        _lib.gqe_attention_prefill(self.dims, Q, Qs, K, V, self.topk_idx, self.w, base, o_bar,
                                   s_out, self.row, self.ws, stream)
        return self.concat

    def forward(self, x, W_r, bias, Q, Qs, K, V, stream=None):
        self.route(x, W_r, bias, stream)
        return self.attention(Q, Qs, K, V, stream)

    def attention_static(self, Q, Qs, K, V, out=None, stream=None):
        """The attention call without a workspace (gqe_attention_prefill_static:
        its scratch is a fixed array inside the library).  Uses this object's
        topk_idx and w; writes into ``out`` (a concat buffer shaped like
        ``concat``) or into ``concat``."""
        self._check_qkv(Q, K, V, Qs)
        dv = self.device
        _expect(self.topk_idx, "topk_idx", (self.B, self.S, self.G, self.k), torch.int32, dv)
        _expect(self.w, "w", (self.B, self.S, self.G, self.k), torch.float32, dv)
        if out is None:
            out = self.concat
        _expect(out, "out", (self.B * self.S, self.row), self.out_dtype, dv)
        a = self.G * self.k * self.d
        flat = out.view(-1)
        _lib.gqe_attention_prefill_static(self.dims, Q, Qs, K, V, self.topk_idx, self.w, out,
                                          flat[a:], flat[a + self.G * self.d:], self.row,
                                          stream)
        return out

    @staticmethod
    def static_device_status(clear=True, stream=None) -> int:
        """Errors latched by attention_static calls on the current device."""
        return _lib.gqe_static_device_status(1 if clear else 0, stream)

    def dense(self, Q, K, V, out=None, stream=None):
        self._check_qkv(Q, K, V)
        if out is not None:
            _expect(out, "out", (self.B, self.S, self.N, self.d), self.out_dtype, self.device)
        if out is None:
            if self._dense_out is None:
                self._dense_out = torch.empty(self.B, self.S, self.N, self.d, dtype=self.out_dtype,
                                              device=self.device)
            out = self._dense_out
        _lib.gqe_dense_gqa_prefill(self.dims, Q, K, V, out, self.ws, stream)
        return out

    def device_status(self, clear=True, stream=None) -> int:
        return _lib.gqe_get_device_status(self.ws, 1 if clear else 0, stream)


    # ---------------------------------------------------------- training
    def forward_train(self, x, W_r, bias, Q, Qs, K, V, stream=None):
        """forward() that also keeps each row's log-sum-exp (``lse_sel``
        [B,S,G,k], ``lse_s`` [B,S]) for :meth:`backward`; float32 outputs."""
        if self.out_dtype != torch.float32:
            raise ValueError("training needs float32 outputs (out_fp32=True)")
        self._check_qkv(Q, K, V, Qs)
        self.route(x, W_r, bias, stream)
        dv = self.device
        if not hasattr(self, "lse_sel"):
            self.lse_sel = torch.empty(self.B, self.S, self.G, self.k, dtype=torch.float32,
                                       device=dv)
            self.lse_s = torch.empty(self.B, self.S, dtype=torch.float32, device=dv)
        a = self.G * self.k * self.d
        flat = self.concat.view(-1)
        _lib.gqe_attention_prefill_train(self.dims, Q, Qs, K, V, self.topk_idx, self.w,
                                         self.concat, flat[a:], flat[a + self.G * self.d:],
                                         self.row, self.lse_sel, self.lse_s, self.ws, stream)
        self._saved = (Q, Qs, K, V)
        return self.concat

    def backward(self, dconcat, stream=None):
        """Gradients for an upstream gradient of the concat buffer (float32
        [B*S, row], the same layout): dict(dQ [B,S,N,d], dQs [B,S,d],
        dK, dV [B,S,G,d], dw [B,S,G,k]), float32.  Uses the tensors of the
        last forward_train()."""
        Q, Qs, K, V = self._saved
        dv = self.device
        _expect(dconcat, "dconcat", (self.B * self.S, self.row), torch.float32, dv)
        n = _lib.gqe_prefill_backward_workspace_size(self.dims)
        if not hasattr(self, "_bws") or self._bws.numel() < n:
            self._bws = torch.zeros(n, dtype=torch.uint8, device=dv)
        B, S, N, G, k, d = self.B, self.S, self.N, self.G, self.k, self.d
        f = torch.float32
        out = dict(dQ=torch.empty(B, S, N, d, dtype=f, device=dv),
                   dQs=torch.empty(B, S, d, dtype=f, device=dv),
                   dK=torch.empty(B, S, G, d, dtype=f, device=dv),
                   dV=torch.empty(B, S, G, d, dtype=f, device=dv),
                   dw=torch.empty(B, S, G, k, dtype=f, device=dv))
        a = G * k * d
        cf, df = self.concat.view(-1), dconcat.view(-1)
        _lib.gqe_prefill_backward(self.dims, Q, Qs, K, V, self.topk_idx, self.w, self.concat,
                                  cf[a + G * d:], self.row, self.lse_sel, self.lse_s, dconcat,
                                  df[a:], df[a + G * d:], self.row, out["dQ"], out["dQs"],
                                  out["dK"], out["dV"], out["dw"], self._bws, stream)
        return out


class GqeChunk:
    """Buffers and calls for chunked prefill: S new tokens per sequence over
    KV caches of T slots (gqe_route on the chunk, then
    gqe_attention_prefill_chunk).  ``concat`` has one W_O input row per chunk
    token (row b*S + i), laid out as in :class:`GqePrefill`."""

    def __init__(self, B, S, T, N, G, k, d, d_model, out_fp32=True, device="cuda"):
        if N % G:
            raise ValueError("N must be a multiple of G")
        self.B, self.S, self.T, self.N, self.G, self.k, self.d = B, S, T, N, G, k, d
        self.d_model, self.M = d_model, N // G
        self.dims = _lib.dims(B, S, N, G, k, d, d_model, 1 if out_fp32 else 0)
        a = _lib.gqe_workspace_size(self.dims)
        b = _lib.gqe_prefill_chunk_workspace_size(self.dims, T)
        if a == 0 or b == 0:
            raise _lib.GqeError(2, "gqe_prefill_chunk_workspace_size")
        dev = _device(device)
        self.device = dev
        self.ws = torch.zeros(max(a, b), dtype=torch.uint8, device=dev)
        self.out_dtype = torch.float32 if out_fp32 else torch.bfloat16
        self.row = (G * k + G + 1) * d
        self.concat = torch.empty(B * S, self.row, dtype=self.out_dtype, device=dev)
        self.topk_idx = torch.empty(B, S, G, k, dtype=torch.int32, device=dev)
        self.p = torch.empty(B, S, G, self.M, dtype=torch.float32, device=dev)
        self.w = torch.empty(B, S, G, k, dtype=torch.float32, device=dev)

    O_sel = GqePrefill.O_sel
    o_bar = GqePrefill.o_bar
    s_out = GqePrefill.s_out

    def route(self, x, W_r, bias=None, stream=None):
        return GqePrefill.route(self, x, W_r, bias, stream)

    def attention(self, Q, Qs, Kc, Vc, q_off=None, kv_start=None, stream=None):
        """Q [B, S, N, d], Qs [B, S, d] (the chunk), caches Kc, Vc [B, T, G, d];
        q_off, kv_start: int32 [B] on the device, or None (0)."""
        bf, dv = torch.bfloat16, self.device
        _expect(Q, "Q", (self.B, self.S, self.N, self.d), bf, dv)
        _expect(Qs, "Qs", (self.B, self.S, self.d), bf, dv)
        _expect(Kc, "Kc", (self.B, self.T, self.G, self.d), bf, dv)
        _expect(Vc, "Vc", (self.B, self.T, self.G, self.d), bf, dv)
        for t, name in ((q_off, "q_off"), (kv_start, "kv_start")):
            if t is not None:
                _expect(t, name, (self.B,), torch.int32, dv)
        a = self.G * self.k * self.d
        flat = self.concat.view(-1)
        _lib.gqe_attention_prefill_chunk(self.dims, self.T, Q, Qs, Kc, Vc, q_off, kv_start,
                                         self.topk_idx, self.w, self.concat, flat[a:],
                                         flat[a + self.G * self.d:], self.row, self.ws, stream)
        return self.concat

    def forward(self, x, W_r, bias, Q, Qs, Kc, Vc, q_off=None, kv_start=None, stream=None):
        self.route(x, W_r, bias, stream)
        return self.attention(Q, Qs, Kc, Vc, q_off, kv_start, stream)

    def device_status(self, clear=True, stream=None) -> int:
        return _lib.gqe_get_device_status(self.ws, 1 if clear else 0, stream)


class GqeDecode:
    """Buffers and calls for one decode step of B sequences over KV caches of
    capacity T (shape [B, T, G, d]); with ``n_new`` > 1, n_new new tokens per
    sequence in one call (gqe_attention_append).

    ``concat`` has one W_O input row per new token (row b * n_new + r), laid
    out as in :class:`GqePrefill`.  Per-token tensors have an n_new axis after
    B when n_new > 1 (x [B, n_new, d_model], Q [B, n_new, N, d] ...) and none
    when n_new = 1.  One workspace serves the router (run on the new tokens,
    S = n_new) and the attention, in stream order.
    """

    def __init__(self, B, T, N, G, k, d, d_model, out_fp32=True, device="cuda", n_new=1):
        if N % G:
            raise ValueError("N must be a multiple of G")
        self.B, self.T, self.N, self.G, self.k, self.d, self.d_model = B, T, N, G, k, d, d_model
        self.M = N // G
        self.n_new = n_new
        of = 1 if out_fp32 else 0
        self.route_dims = _lib.dims(B, n_new, N, G, k, d, d_model, of)
        self.dims = _lib.dims(B, T, N, G, k, d, d_model, of)
        a = _lib.gqe_workspace_size(self.route_dims)
        b = _lib.gqe_append_workspace_size(self.dims, n_new)
        if a == 0 or b == 0:
            raise _lib.GqeError(2, "gqe_append_workspace_size")
        dev = _device(device)
        self.device = dev
        self.ws = torch.zeros(max(a, b), dtype=torch.uint8, device=dev)
        self.out_dtype = torch.float32 if out_fp32 else torch.bfloat16
        self.row = (G * k + G + 1) * d
        self.concat = torch.empty(B * n_new, self.row, dtype=self.out_dtype, device=dev)
        lead = (B,) if n_new == 1 else (B, n_new)
        self._lead = lead
        self.topk_idx = torch.empty(*lead, G, k, dtype=torch.int32, device=dev)
        self.p = torch.empty(*lead, G, self.M, dtype=torch.float32, device=dev)
        self.w = torch.empty(*lead, G, k, dtype=torch.float32, device=dev)

    def O_sel(self):
        return self.concat[:, : self.G * self.k * self.d].view(*self._lead, self.G, self.k, self.d)

    def o_bar(self):
        a = self.G * self.k * self.d
        return self.concat[:, a: a + self.G * self.d].view(*self._lead, self.G, self.d)

    def s_out(self):
        return self.concat[:, (self.G * self.k + self.G) * self.d:].view(*self._lead, self.d)

    def route(self, x, W_r, bias=None, stream=None):
        """x: bf16 [B, d_model] (the new tokens; [B, n_new, d_model] if n_new > 1)."""
        bf, dv = torch.bfloat16, self.device
        _expect(x, "x", (*self._lead, self.d_model), bf, dv)
        _expect(W_r, "W_r", (self.G, self.d_model, self.M), bf, dv)
        if bias is not None:
            _expect(bias, "bias", (self.G, self.M), torch.float32, dv)
        _lib.gqe_route(self.route_dims, x, W_r, bias, self.topk_idx, self.p, self.w, self.ws,
                       stream)
        return self.topk_idx, self.p, self.w

    def attention(self, Q, Qs, Kc, Vc, pos, kv_start=None, stream=None):
        """Q [B, N, d], Qs [B, d] (n_new axis after B if n_new > 1), caches
        [B, T, G, d] (bf16), pos int32 [B] (slot of the first new token);
        kv_start int32 [B] (first valid slot, left padding) or None."""
        bf, dv = torch.bfloat16, self.device
        _expect(Q, "Q", (*self._lead, self.N, self.d), bf, dv)
        _expect(Qs, "Qs", (*self._lead, self.d), bf, dv)
        _expect(Kc, "Kc", (self.B, self.T, self.G, self.d), bf, dv)
        _expect(Vc, "Vc", (self.B, self.T, self.G, self.d), bf, dv)
        _expect(pos, "pos", (self.B,), torch.int32, dv)
        if kv_start is not None:
            _expect(kv_start, "kv_start", (self.B,), torch.int32, dv)
        a = self.G * self.k * self.d
        flat = self.concat.view(-1)
        if self.n_new == 1:
            _lib.gqe_attention_decode(self.dims, Q, Qs, Kc, Vc, pos, kv_start, self.topk_idx,
                                      self.w, self.concat, flat[a:], flat[a + self.G * self.d:],
                                      self.row, self.ws, stream)
        else:
            _lib.gqe_attention_append(self.dims, self.n_new, Q, Qs, Kc, Vc, pos, kv_start,
                                      self.topk_idx, self.w, self.concat, flat[a:],
                                      flat[a + self.G * self.d:], self.row, self.ws, stream)
        return self.concat

    def forward(self, x, W_r, bias, Q, Qs, Kc, Vc, pos, kv_start=None, stream=None):
        self.route(x, W_r, bias, stream)
        return self.attention(Q, Qs, Kc, Vc, pos, kv_start, stream)

    def graph(self, x, W_r, bias, Q, Qs, Kc, Vc, pos, kv_start=None, warmup=2):
        """Capture one decode step (router + attention: four kernel launches)
        on these tensors into a torch.cuda.CUDAGraph.  Each replay re-runs the
        step on what the tensors then hold: copy the next tokens' x, Q, Qs and
        positions (and the new cache rows) into them, then replay.  Outputs
        land in this object's buffers (``concat``, ``topk_idx``, ``p``, ``w``)."""
        cur = torch.cuda.current_stream(self.device)
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(cur)
        with torch.cuda.stream(side):  # warm-up outside the capture (one-time setup)
            for _ in range(warmup):
                self.forward(x, W_r, bias, Q, Qs, Kc, Vc, pos, kv_start)
        cur.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.forward(x, W_r, bias, Q, Qs, Kc, Vc, pos, kv_start)
        return g

    def device_status(self, clear=True, stream=None) -> int:
        return _lib.gqe_get_device_status(self.ws, 1 if clear else 0, stream)

class GqeLayer:
    """Buffers and calls for the whole GQE attention layer of one shape,
    x -> y (gqe_layer_prefill), and the all-active GQA layer baseline
    (gqe_dense_layer_prefill).

    Weights (bf16): W_Q [N, d_model, d], W_K and W_V [G, d_model, d], W_s
    [d_model, d], W_r [G, d_model, M], W_O [(G*k + G + 1)*d, d_model] (rows in
    concat order); the baseline's W_O is [N*d, d_model].  Intermediates are
    kept in this object: ``Q`` (only the selected heads' rows are written),
    ``Qs``, ``K``, ``V``, ``concat`` (bf16), ``topk_idx``, ``p``, ``w``; the
    output ``y`` is float32 [B, S, d_model].
    """

    def __init__(self, B, S, N, G, k, d, d_model, device="cuda"):
        if N % G:
            raise ValueError("N must be a multiple of G")
        self.B, self.S, self.N, self.G, self.k, self.d, self.d_model = B, S, N, G, k, d, d_model
        self.M = N // G
        self.dims = _lib.dims(B, S, N, G, k, d, d_model, 0)
        nbytes = _lib.gqe_workspace_size(self.dims)
        if nbytes == 0:
            raise _lib.GqeError(2, "gqe_workspace_size")
        dev = _device(device)
        self.device = dev
        bf = torch.bfloat16
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.row = (G * k + G + 1) * d
        self.Q = torch.zeros(B, S, N, d, dtype=bf, device=dev)
        self.Qs = torch.empty(B, S, d, dtype=bf, device=dev)
        self.K = torch.empty(B, S, G, d, dtype=bf, device=dev)
        self.V = torch.empty(B, S, G, d, dtype=bf, device=dev)
        self.concat = torch.empty(B * S, self.row, dtype=bf, device=dev)
        self.y = torch.empty(B, S, d_model, dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty(B, S, G, k, dtype=torch.int32, device=dev)
        self.p = torch.empty(B, S, G, self.M, dtype=torch.float32, device=dev)
        self.w = torch.empty(B, S, G, k, dtype=torch.float32, device=dev)
        self._dense = None

    def _check_weights(self, W_Q, W_K, W_V):
        bf, dv = torch.bfloat16, self.device
        _expect(W_Q, "W_Q", (self.N, self.d_model, self.d), bf, dv)
        _expect(W_K, "W_K", (self.G, self.d_model, self.d), bf, dv)
        _expect(W_V, "W_V", (self.G, self.d_model, self.d), bf, dv)

    def forward(self, x, W_Q, W_K, W_V, W_s, W_r, bias, W_O, stream=None):
        bf, dv = torch.bfloat16, self.device
        _expect(x, "x", (self.B, self.S, self.d_model), bf, dv)
        self._check_weights(W_Q, W_K, W_V)
        _expect(W_s, "W_s", (self.d_model, self.d), bf, dv)
        _expect(W_r, "W_r", (self.G, self.d_model, self.M), bf, dv)
        if bias is not None:
            _expect(bias, "bias", (self.G, self.M), torch.float32, dv)
        _expect(W_O, "W_O", (self.row, self.d_model), bf, dv)
        _lib.gqe_layer_prefill(self.dims, x, W_Q, W_K, W_V, W_s, W_r, bias, W_O, self.topk_idx,
                               self.p, self.w, self.Q, self.Qs, self.K, self.V, self.concat,
                               self.y, self.ws, stream)
        return self.y

    def dense(self, x, W_Q, W_K, W_V, W_O, stream=None):
        """The all-active GQA layer; returns its own y (float32)."""
        bf, dv = torch.bfloat16, self.device
        _expect(x, "x", (self.B, self.S, self.d_model), bf, dv)
        self._check_weights(W_Q, W_K, W_V)
        _expect(W_O, "W_O", (self.N * self.d, self.d_model), bf, dv)
        if self._dense is None:
            B, S, N, d = self.B, self.S, self.N, self.d
            self._dense = dict(Q=torch.empty(B, S, N, d, dtype=bf, device=dv),
                               K=torch.empty_like(self.K), V=torch.empty_like(self.V),
                               O=torch.empty(B, S, N, d, dtype=bf, device=dv),
                               y=torch.empty_like(self.y))
        t = self._dense
        _lib.gqe_dense_layer_prefill(self.dims, x, W_Q, W_K, W_V, W_O, t["Q"], t["K"], t["V"],
                                     t["O"], t["y"], self.ws, stream)
        return t["y"]

    def device_status(self, clear=True, stream=None) -> int:
        return _lib.gqe_get_device_status(self.ws, 1 if clear else 0, stream)
