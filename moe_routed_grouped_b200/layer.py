"""Torch-facing wrapper: owns the device buffers of one GQE prefill shape and
calls the C ABI.  Allocation and argument marshalling only; every step of the
computation runs in libgqe.so."""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib


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
        dev = torch.device(device)
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
        _lib.gqe_route(self.dims, x, W_r, bias, self.topk_idx, self.p, self.w, self.ws, stream)
        return self.topk_idx, self.p, self.w

    def attention(self, Q, Qs, K, V, stream=None):
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

    def dense(self, Q, K, V, out=None, stream=None):
        if out is None:
            if self._dense_out is None:
                self._dense_out = torch.empty(self.B, self.S, self.N, self.d, dtype=self.out_dtype,
                                              device=self.device)
            out = self._dense_out
        _lib.gqe_dense_gqa_prefill(self.dims, Q, K, V, out, self.ws, stream)
        return out

    def device_status(self, clear=True, stream=None) -> int:
        return _lib.gqe_get_device_status(self.ws, 1 if clear else 0, stream)
