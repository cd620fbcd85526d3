"""Seeded synthetic inputs for GQE prefill.

This module is shared by the tests, the bench and the oracle.  It holds no
arithmetic of the method itself: it only turns (seed, element index) into
bf16 bit patterns and describes the workload shapes.

Generator (counter based, so any element can be produced independently):

* SplitMix64 finaliser applied to ``seed + (counter + 1) * 0x9E3779B97F4A7C15``
  (the published SplitMix64 mixing function, Steele/Lea/Flood 2014).
* Element ``n`` uses counters ``2n`` and ``2n + 1`` to build two uniforms
  ``u1 = ((a >> 11) + 1) / 2**53`` in (0, 1] and ``u2 = (b >> 11) / 2**53`` in
  [0, 1), and one Box-Muller normal ``sqrt(-2 ln u1) * cos(2 pi u2)`` in double.
* The double is scaled by ``std`` (and shifted by ``mean``), rounded to
  float32 (round-to-nearest-even) and then to bf16 (round-to-nearest-even on
  the upper 16 bits).  Both steps are part of the definition.

Seeds follow ``1000 * config_id + stream`` with streams x=0, W_r=1, Q=2, Qs=3,
K=4, V=5.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_X, STREAM_WR, STREAM_Q, STREAM_QS, STREAM_K, STREAM_V = range(6)


def splitmix64(counter: np.ndarray, seed: int) -> np.ndarray:
    """SplitMix64 output for each counter value (uint64 in, uint64 out)."""
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (counter.astype(np.uint64) + np.uint64(1)) * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def normal_f64(n: int, seed: int, offset: int = 0) -> np.ndarray:
    """``n`` standard normals (float64) for element indices offset..offset+n-1."""
    c = np.arange(offset, offset + n, dtype=np.uint64)
    a = splitmix64(np.uint64(2) * c, seed)
    b = splitmix64(np.uint64(2) * c + np.uint64(1), seed)
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (b >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); returns uint16 bit patterns."""
    bits = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((bits >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    out = ((bits + rnd) >> np.uint64(16)).astype(np.uint16)
    # keep NaN payloads quiet and non-zero
    nan = np.isnan(np.asarray(f, dtype=np.float32))
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(shape, seed: int, std: float = 1.0, mean: float = 0.0,
                chunk: int = 1 << 24) -> np.ndarray:
    """bf16 bit patterns (uint16 array of ``shape``) of N(mean, std^2) samples."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        v = normal_f64(e - s, seed, offset=s) * std + mean
        out[s:e] = f32_to_bf16_bits(v.astype(np.float32))
    return out.reshape(shape)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one GQE prefill workload."""
    cid: int
    name: str
    B: int
    S: int
    N: int
    G: int
    k: int
    d: int
    d_model: int
    bias0: float = 0.0  # additive router-logit bias on expert 0 of every group

    @property
    def M(self) -> int:
        return self.N // self.G

    @property
    def wr_std(self) -> float:
        return 1.0 / math.sqrt(self.d_model)

    def seed(self, stream: int) -> int:
        return 1000 * self.cid + stream

    def useful_flop_routed(self) -> float:
        return (self.G * self.k + 1) * self.B * 2.0 * self.d * self.S * (self.S + 1)

    def useful_flop_dense(self) -> float:
        return self.N * self.B * 2.0 * self.d * self.S * (self.S + 1)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(1, "tiny", B=1, S=128, N=16, G=8, k=1, d=64, d_model=256),
    "layer250m": Workload(2, "layer250m", B=8, S=2048, N=16, G=8, k=1, d=64, d_model=1024),
    "imbalanced32k": Workload(3, "imbalanced32k", B=1, S=32768, N=16, G=8, k=1, d=64,
                              d_model=1024, bias0=1.5),
    "wide131k": Workload(4, "wide131k", B=1, S=131072, N=32, G=8, k=2, d=128, d_model=4096),
    "million": Workload(5, "million", B=1, S=1048576, N=16, G=8, k=1, d=64, d_model=1024),
}


def make_inputs(w: Workload, streams=("x", "W_r", "Q", "Qs", "K", "V"),
                seed_base: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Generate the bf16 inputs (as uint16 bit arrays) of one workload.

    Layouts: x [B,S,d_model], W_r [G,d_model,M], Q [B,S,N,d], Qs [B,S,d],
    K/V [B,S,G,d].  ``bias`` [G,M] float32 is included when the workload biases
    expert 0.
    """
    sb = 1000 * w.cid if seed_base is None else seed_base
    shapes = {
        "x": ((w.B, w.S, w.d_model), STREAM_X, 1.0),
        "W_r": ((w.G, w.d_model, w.M), STREAM_WR, w.wr_std),
        "Q": ((w.B, w.S, w.N, w.d), STREAM_Q, 1.0),
        "Qs": ((w.B, w.S, w.d), STREAM_QS, 1.0),
        "K": ((w.B, w.S, w.G, w.d), STREAM_K, 1.0),
        "V": ((w.B, w.S, w.G, w.d), STREAM_V, 1.0),
    }
    out: Dict[str, np.ndarray] = {}
    for name in streams:
        shape, stream, std = shapes[name]
        out[name] = normal_bf16(shape, sb + stream, std=std)
    if w.bias0 != 0.0:
        b = np.zeros((w.G, w.M), dtype=np.float32)
        b[:, 0] = w.bias0
        out["bias"] = b
    return out
