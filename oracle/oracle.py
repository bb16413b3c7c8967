"""Python access to the CPU oracle (test infrastructure only).

Only the test suite, the smoke check and the CPU-baseline leg of the
benchmark import this module.  The oracle library (lsh_oracle.c) is plain
double-precision C; this file only compiles it and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsh_oracle.c")
_LIB = os.path.join(_HERE, "liblsh_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_L = ctypes.c_long
_C = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle into liblsh_oracle.so next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = open_library(build())
    return _lib


def open_library(path: str):
    """Loads an oracle library and declares its entry points.  lib() opens the
    one built from lsh_oracle.c; the oracle tests' planted-mistake check opens
    altered copies of that source through this function."""
    L = ctypes.CDLL(path)
    L.oracle_hash.argtypes = [_D, _L, _C, _D, _C, _I32, _D]
    L.oracle_sort.argtypes = [_I32, _L, _I32]
    L.oracle_attn_round.argtypes = [_D, _D, _L, _C, _I32, _C, _C, _I32, _C, _D, _D]
    L.oracle_attn_slots.argtypes = [_D, _D, _L, _C, _I32, _C, _C, _I32, _C, _I64, _L, _D, _D]
    L.oracle_combine.argtypes = [_D, _D, _C, _L, _C, _D, _D]
    L.oracle_fwd_head.argtypes = [_D, _D, _L, _C, _D, _C, _C, _C, _C, _C, _C, _D, _D, _I32, _I32, _D]
    L.oracle_bwd_head.argtypes = [_D, _D, _D, _L, _C, _I32, _C, _C, _C, _I32, _C, _D, _D]
    L.oracle_fwd_batch.argtypes = [_D, _D, _L, _L, _C, _D, _C, _C, _C, _C, _C, _C, _D, _D, _I32, _I32, _D]
    L.oracle_fwd_perm_batch.argtypes = [_D, _D, _L, _L, _C, _I32, _C, _C, _C, _I32, _C, _D, _D]
    L.oracle_bwd_batch.argtypes = [_D, _D, _D, _L, _L, _C, _I32, _C, _C, _C, _I32, _C, _D, _D]
    L.oracle_local_fwd_batch.argtypes = [_D, _D, _L, _L, _C, _C, _C, _C, _C, _C, _D, _D]
    L.oracle_local_bwd_batch.argtypes = [_D, _D, _D, _L, _L, _C, _C, _C, _C, _C, _C, _D, _D]
    L.oracle_max_threads.argtypes = []
    return L


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t):
    return a.ctypes.data_as(t)


def _bucket(bucket, shape):
    """Optional bucket ids by position (the bucket-mask reading): int32 array or None."""
    if bucket is None:
        return None, None
    b = np.ascontiguousarray(bucket, dtype=np.int32)
    assert b.shape == tuple(shape), (b.shape, shape)
    return b, _p(b, _I32)


def _check(rc):
    if rc != 0:
        raise RuntimeError(f"oracle call failed (rc={rc})")


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def hash_round(x, Rr, n_buckets):
    """Buckets and near-tie margins of rows x [n, d] for one rotation Rr [d, n_buckets/2]."""
    x = _d(x); Rr = _d(Rr)
    n, d = x.shape
    b = np.empty(n, np.int32); mg = np.empty(n, np.float64)
    _check(lib().oracle_hash(_p(x, _D), n, d, _p(Rr, _D), int(n_buckets), _p(b, _I32), _p(mg, _D)))
    return b, mg


def sort_segment(bucket):
    """perm[s] = position at sorted slot s (stable by position)."""
    b = np.ascontiguousarray(bucket, dtype=np.int32)
    perm = np.empty_like(b)
    _check(lib().oracle_sort(_p(b, _I32), b.size, _p(perm, _I32)))
    return perm


def attn_round(x, v, perm, chunk, causal, bucket=None, self_penalty=False):
    """One round: o [L, d] and lse [L] in original order.  bucket [L] (by
    position) switches on the bucket mask; self_penalty the penalty reading."""
    x = _d(x); v = _d(v); perm = np.ascontiguousarray(perm, dtype=np.int32)
    L, d = x.shape
    b, bp = _bucket(bucket, (L,))
    o = np.empty((L, d)); lse = np.empty(L)
    _check(lib().oracle_attn_round(_p(x, _D), _p(v, _D), L, d, _p(perm, _I32), int(chunk), int(causal),
                                   bp, int(bool(self_penalty)), _p(o, _D), _p(lse, _D)))
    return o, lse


def attn_slots(x, v, perm, chunk, causal, slots, bucket=None, self_penalty=False):
    """One round for selected sorted slots: o [n, d], lse [n] in list order."""
    x = _d(x); v = _d(v); perm = np.ascontiguousarray(perm, dtype=np.int32)
    slots = np.ascontiguousarray(slots, dtype=np.int64)
    L, d = x.shape
    b, bp = _bucket(bucket, (L,))
    o = np.empty((slots.size, d)); lse = np.empty(slots.size)
    _check(lib().oracle_attn_slots(_p(x, _D), _p(v, _D), L, d, _p(perm, _I32), int(chunk), int(causal),
                                   bp, int(bool(self_penalty)), _p(slots, _I64), slots.size, _p(o, _D),
                                   _p(lse, _D)))
    return o, lse


def combine(o, lse):
    """Merge rounds: o [R, L, d], lse [R, L] -> y [L, d], LSE [L]."""
    o = _d(o); lse = _d(lse)
    R, L, d = o.shape
    y = np.empty((L, d)); big = np.empty(L)
    _check(lib().oracle_combine(_p(o, _D), _p(lse, _D), R, L, d, _p(y, _D), _p(big, _D)))
    return y, big


def fwd(x, v, R, n_buckets, chunk, causal, bucket_mask=False, self_penalty=False):
    """Full forward on [B, H, L, d] inputs with rotations R [n_hashes, d, n_buckets/2].

    Returns dict with y [B,H,L,d], lse/perm/bucket/margin [B,H,n_hashes,L]."""
    x = _d(x); v = _d(v); R = _d(R)
    B, H, L, d = x.shape
    nh = R.shape[0]
    y = np.empty_like(x)
    lse = np.empty((B, H, nh, L)); mg = np.empty((B, H, nh, L))
    perm = np.empty((B, H, nh, L), np.int32); bk = np.empty((B, H, nh, L), np.int32)
    _check(lib().oracle_fwd_batch(_p(x, _D), _p(v, _D), B * H, L, d, _p(R, _D), int(n_buckets), nh,
                                  int(chunk), int(causal), int(bool(bucket_mask)), int(bool(self_penalty)),
                                  _p(y, _D), _p(lse, _D), _p(perm, _I32),
                                  _p(bk, _I32), _p(mg, _D)))
    return {"y": y, "lse": lse, "perm": perm, "bucket": bk, "margin": mg}


def fwd_perm(x, v, perm, chunk, causal, bucket=None, self_penalty=False):
    """Forward with given permutations perm [B,H,n_hashes,L]: y [B,H,L,d], lse [B,H,n_hashes,L].
    bucket [B,H,n_hashes,L] (by position) switches on the bucket mask."""
    x = _d(x); v = _d(v); perm = np.ascontiguousarray(perm, dtype=np.int32)
    B, H, L, d = x.shape
    nh = perm.shape[2]
    b, bp = _bucket(bucket, perm.shape)
    y = np.empty_like(x); lse = np.empty((B, H, nh, L))
    _check(lib().oracle_fwd_perm_batch(_p(x, _D), _p(v, _D), B * H, L, d, _p(perm, _I32), nh,
                                       int(chunk), int(causal), bp, int(bool(self_penalty)), _p(y, _D),
                                       _p(lse, _D)))
    return y, lse


def bwd(x, v, dy, perm, chunk, causal, bucket=None, self_penalty=False):
    """Gradients (dx, dv) [B,H,L,d] of sum(y * dy) with permutations perm [B,H,n_hashes,L]."""
    x = _d(x); v = _d(v); dy = _d(dy); perm = np.ascontiguousarray(perm, dtype=np.int32)
    B, H, L, d = x.shape
    nh = perm.shape[2]
    b, bp = _bucket(bucket, perm.shape)
    dx = np.empty_like(x); dv = np.empty_like(x)
    _check(lib().oracle_bwd_batch(_p(x, _D), _p(v, _D), _p(dy, _D), B * H, L, d, _p(perm, _I32), nh,
                                  int(chunk), int(causal), bp, int(bool(self_penalty)), _p(dx, _D), _p(dv, _D)))
    return dx, dv


def local_fwd(x, v, chunk, causal, before=1, after=1, self_penalty=False):
    """Local (non-hashed) chunk attention on [B, H, L, d]: chunk c of the
    positions in their own order attends to chunks c - before .. c + after.
    Returns y [B, H, L, d] and lse [B, H, L]."""
    x = _d(x); v = _d(v)
    B, H, L, d = x.shape
    y = np.empty_like(x); lse = np.empty((B, H, L))
    _check(lib().oracle_local_fwd_batch(_p(x, _D), _p(v, _D), B * H, L, d, int(chunk), int(before), int(after),
                                        int(causal), int(bool(self_penalty)), _p(y, _D), _p(lse, _D)))
    return y, lse


def local_bwd(x, v, dy, chunk, causal, before=1, after=1, self_penalty=False):
    """Gradients (dx, dv) of sum(y * dy) for local chunk attention."""
    x = _d(x); v = _d(v); dy = _d(dy)
    B, H, L, d = x.shape
    dx = np.empty_like(x); dv = np.empty_like(x)
    _check(lib().oracle_local_bwd_batch(_p(x, _D), _p(v, _D), _p(dy, _D), B * H, L, d, int(chunk), int(before),
                                        int(after), int(causal), int(bool(self_penalty)), _p(dx, _D), _p(dv, _D)))
    return dx, dv


def rev_g(u, Wg, bg):
    """The reversible block's token-wise G(u) = tanh(u Wg + bg), float64."""
    return np.tanh(_d(u) @ _d(Wg) + _d(bg))


def rev_fwd(x1, x2, R, Wg, bg, n_buckets, chunk, causal, round_to=None):
    """Reversible block ("Reformer" paper note, Reversible Residual Layers):
    y1 = x1 + F(x2), y2 = x2 + G(y1), F = LSH attention with x2 as query-key and
    value.  round_to: a function applied to x2 before F (the rounding to the
    attention dtype), or None.  Returns y1, y2 and F's permutation."""
    xa = _d(x2) if round_to is None else _d(round_to(x2))
    f = fwd(xa, xa, R, n_buckets, chunk, causal)
    y1 = _d(x1) + f["y"]
    y2 = _d(x2) + rev_g(y1, Wg, bg)
    return y1, y2, f["perm"]


def rev_bwd(y1, y2, dy1, dy2, R, Wg, bg, n_buckets, chunk, causal, round_to=None):
    """Backward from the outputs: x2 = y2 - G(y1), x1 = y1 - F(x2);
    dx1 = dy1 + J_G(y1)^T dy2, dx2 = dy2 + J_F(x2)^T dx1 (F's two inputs are both
    x2, so its query-key and value gradients add).  Returns x1, x2, dx1, dx2."""
    y1 = _d(y1); y2 = _d(y2); dy1 = _d(dy1); dy2 = _d(dy2)
    g = rev_g(y1, Wg, bg)
    x2 = y2 - g
    dx1 = dy1 + ((dy2 * (1.0 - g * g)) @ _d(Wg).T)
    xa = x2 if round_to is None else _d(round_to(x2))
    f = fwd(xa, xa, R, n_buckets, chunk, causal)
    x1 = y1 - f["y"]
    # F's output gradient enters F in its dtype, as the rounding of x2 does
    dq, dv = bwd(xa, xa, dx1 if round_to is None else _d(round_to(dx1)), f["perm"], chunk, causal)
    return x1, x2, dx1, dy2 + dq + dv
