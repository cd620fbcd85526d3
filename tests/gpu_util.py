"""Helpers for the GPU parity tests (input upload, tolerance checks)."""
import numpy as np
import torch

import oracle
from synth import normal_bf16

ATOL = 1e-2     # max-abs bound on float32 outputs
RTOL_L2 = 1e-3  # relative L2 bound on float32 outputs


def dev_bf16(bits):
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def check_close(got, ref, what, atol=ATOL, rtol_l2=RTOL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - ref)
    mx = float(err.max()) if err.size else 0.0
    nrm = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref) / nrm) if nrm > 0 else mx
    assert mx <= atol, f"{what}: max abs err {mx:.3e} > {atol}"
    assert rel <= rtol_l2, f"{what}: rel L2 err {rel:.3e} > {rtol_l2}"
    return mx, rel


def make_case(B, S, N, G, k, d, dm, seed, bias0=0.0, wr_std=None):
    M = N // G
    inp = dict(
        x=normal_bf16((B, S, dm), seed),
        W_r=normal_bf16((G, dm, M), seed + 1, std=wr_std or dm ** -0.5),
        Q=normal_bf16((B, S, N, d), seed + 2),
        Qs=normal_bf16((B, S, d), seed + 3),
        K=normal_bf16((B, S, G, d), seed + 4),
        V=normal_bf16((B, S, G, d), seed + 5),
    )
    inp["bias"] = None
    if bias0:
        b = np.zeros((G, M), np.float32)
        b[:, 0] = bias0
        inp["bias"] = b
    return inp


def upload(inp):
    out = {k: dev_bf16(v) for k, v in inp.items() if k != "bias"}
    out["bias"] = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).cuda()
    return out
