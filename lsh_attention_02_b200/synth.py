"""Seeded synthetic inputs for LSH attention (shared query-key, values, rotations, dY).

This module holds random-number generation only: it contains none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed
from it without sharing any of the method's code.

Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes,
Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC 2011),
written here from its published round function (two 32x32->64 multiplies
per round, Weyl key schedule, ten rounds).  Uniforms are turned into
standard normals with the Box-Muller transform (Box and Muller, 1958).
Normals are produced in float64, rounded to float32, then (for bf16
workloads) rounded to bfloat16 with round-to-nearest-even.

Stream layout: every array is drawn from key = (seed, stream) with counter
(block, 0, 0, 0); each counter block yields four 32-bit words, i.e. four
uniforms or four normals.
"""
from __future__ import annotations

import dataclasses
import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint32(0x9E3779B9)
_W1 = np.uint32(0xBB67AE85)
_LO = np.uint64(0xFFFFFFFF)
_SH = np.uint64(32)

# sub-stream ids
STREAM_X, STREAM_V, STREAM_R, STREAM_DY = 0, 1, 2, 3
STREAM_CENTROID_X, STREAM_ASSIGN, STREAM_CENTROID_V = 4, 5, 6


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds on uint32 numpy arrays; returns four uint32 arrays."""
    c0 = np.asarray(c0, dtype=np.uint32)
    c1 = np.asarray(c1, dtype=np.uint32)
    c2 = np.asarray(c2, dtype=np.uint32)
    c3 = np.asarray(c3, dtype=np.uint32)
    k0 = np.uint32(k0)
    k1 = np.uint32(k1)
    with np.errstate(over="ignore"):
        for _ in range(10):
            p0 = _M0 * c0.astype(np.uint64)
            p1 = _M1 * c2.astype(np.uint64)
            hi0 = (p0 >> _SH).astype(np.uint32)
            lo0 = (p0 & _LO).astype(np.uint32)
            hi1 = (p1 >> _SH).astype(np.uint32)
            lo1 = (p1 & _LO).astype(np.uint32)
            c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
            k0 = np.uint32(k0 + _W0)
            k1 = np.uint32(k1 + _W1)
    return c0, c1, c2, c3


def random_u32(seed: int, stream: int, n: int) -> np.ndarray:
    """n uint32 words from key (seed, stream), counters 0..ceil(n/4)-1."""
    nblk = (n + 3) // 4
    ctr = np.arange(nblk, dtype=np.uint64)
    c0 = (ctr & _LO).astype(np.uint32)
    c1 = (ctr >> _SH).astype(np.uint32)
    z = np.zeros(nblk, dtype=np.uint32)
    r = philox4x32_10(c0, c1, z, z, seed & 0xFFFFFFFF, stream & 0xFFFFFFFF)
    return np.stack(r, axis=1).reshape(-1)[:n]


def uniform01(seed: int, stream: int, n: int) -> np.ndarray:
    """Uniforms in the open interval (0, 1) as float64: (u + 0.5) * 2^-32."""
    u = random_u32(seed, stream, n).astype(np.float64)
    return (u + 0.5) * (1.0 / 4294967296.0)


def normal(seed: int, stream: int, n: int) -> np.ndarray:
    """n standard normals (float64) via Box-Muller on consecutive uniform pairs."""
    m = n + (n & 1)
    u = uniform01(seed, stream, m).reshape(-1, 2)
    rad = np.sqrt(-2.0 * np.log(u[:, 0]))
    ang = 2.0 * np.pi * u[:, 1]
    z = np.stack([rad * np.cos(ang), rad * np.sin(ang)], axis=1).reshape(-1)
    return z[:n]


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))
    out = ((bits + bias) >> np.uint64(16)) << np.uint64(16)
    return out.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values already representable in bfloat16."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a32 = np.asarray(a, dtype=np.float32)
    if dtype == "bf16":
        return round_to_bf16(a32)
    if dtype == "f32":
        return a32
    raise ValueError(f"unknown dtype {dtype!r}")


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one LSH-attention workload."""
    name: str
    B: int
    H: int
    L: int
    d: int
    n_buckets: int
    n_hashes: int
    chunk: int
    causal: bool
    dtype: str            # "f32" or "bf16"
    backward: bool
    seed: int
    clustered: int = 0    # >0: number of Gaussian clusters per (b, h)
    sigma: float = 0.1    # within-cluster noise for clustered inputs

    @property
    def tokens(self) -> int:
        return self.B * self.L

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the method is exercised on (seed = 1000 + index).
WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 2, 1024, 64, 16, 1, 64, False, "f32", False, 1000),
    "bf16_causal_4k": Workload("bf16_causal_4k", 8, 8, 4096, 64, 64, 2, 64, True, "bf16", False, 1001),
    "long_64k": Workload("long_64k", 1, 8, 65536, 64, 1024, 4, 64, True, "bf16", True, 1002),
    "image_12k": Workload("image_12k", 8, 8, 12288, 64, 192, 8, 64, True, "bf16", True, 1003,
                          clustered=192),
    "half_million": Workload("half_million", 1, 2, 524288, 64, 8192, 2, 64, True, "bf16", False, 1004),
}


def _gaussian_tensor(w: Workload, stream: int) -> np.ndarray:
    n = w.B * w.H * w.L * w.d
    return normal(w.seed, stream, n).reshape(w.B, w.H, w.L, w.d)


def _clustered_tensor(w: Workload, centroid_stream: int, noise_stream: int) -> np.ndarray:
    """x = centroid[u] + sigma * noise, centroids and assignment drawn per (b, h)."""
    k = w.clustered
    bh = w.B * w.H
    cent = normal(w.seed, centroid_stream, bh * k * w.d).reshape(bh, k, w.d)
    u = random_u32(w.seed, STREAM_ASSIGN, bh * w.L).reshape(bh, w.L)
    assign = (u.astype(np.uint64) * np.uint64(k)) >> np.uint64(32)   # uniform over k, no modulo bias
    noise = normal(w.seed, noise_stream, bh * w.L * w.d).reshape(bh, w.L, w.d)
    out = np.take_along_axis(cent, assign.astype(np.int64)[:, :, None], axis=1) + w.sigma * noise
    return out.reshape(w.B, w.H, w.L, w.d)


def make_inputs(w: Workload, with_dy: bool | None = None) -> dict:
    """Seeded host arrays for one workload, already rounded to the storage dtype.

    Returns float32 numpy arrays (bf16-representable when dtype == "bf16"):
      x  [B, H, L, d]            shared query-key
      v  [B, H, L, d]            values
      R  [n_hashes, d, n_buckets/2]   random rotations, shared over batch and heads
      dy [B, H, L, d]            upstream gradient (only when requested)
    """
    if w.clustered:
        x = _clustered_tensor(w, STREAM_CENTROID_X, STREAM_X)
        v = _clustered_tensor(w, STREAM_CENTROID_V, STREAM_V)
    else:
        x = _gaussian_tensor(w, STREAM_X)
        v = _gaussian_tensor(w, STREAM_V)
    half = w.n_buckets // 2
    R = normal(w.seed, STREAM_R, w.n_hashes * w.d * half).reshape(w.n_hashes, w.d, half)
    out = {"x": _store(x, w.dtype), "v": _store(v, w.dtype), "R": _store(R, w.dtype)}
    if with_dy if with_dy is not None else w.backward:
        out["dy"] = _store(_gaussian_tensor(w, STREAM_DY), w.dtype)
    return out
