"""Python binding of the LSH attention C ABI (liblsh_attn.so).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are torch CUDA tensors (torch provides device memory and
streams); each function passes their device pointers and the current CUDA
stream to the C entry point of the same name.  The library is loaded on first
use; if it is missing that call raises ImportError -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsh_attn.so")

LSH_F32, LSH_BF16 = 0, 1
FLAG_BUCKET_MASK, FLAG_SELF_PENALTY = 1, 2      # lsh_attn_desc.flags bits
SELF_PENALTY_SCORE = -1.0e5

STATUS = {0: "LSH_OK", -1: "LSH_ERR_ARG", -2: "LSH_ERR_SHAPE", -3: "LSH_ERR_ALIGN",
          -4: "LSH_ERR_UNSUPPORTED", -5: "LSH_ERR_CUDA", -6: "LSH_ERR_TIMEOUT", -7: "LSH_ERR_WORKSPACE"}

EXPORTED = ("lsh_attn_make_rotations", "lsh_attn_workspace_size", "lsh_attn_hash", "lsh_attn_sort", "lsh_attn_sort_static", "lsh_attn_fwd_sorted", "lsh_attn_fwd",
            "lsh_attn_bwd", "lsh_attn_poll", "lsh_attn_selftest_timeout", "lsh_attn_trace_begin",
            "lsh_attn_trace_end", "lsh_attn_trace_stages", "lsh_attn_fused_forward",
            "lsh_attn_fused_forward_fits", "lsh_attn_last_near_ties",
            "lsh_attn_status_str", "lsh_attn_last_error", "lsh_attn_abi_version",
            "lsh_attn_local_workspace_size", "lsh_attn_local_fwd", "lsh_attn_local_bwd",
            "lsh_rev_workspace_size", "lsh_rev_fwd", "lsh_rev_bwd",
            "lsh_attn_step_host_scratch_size", "lsh_attn_step_host")

STAGES = ("hash", "sort", "norms", "attn_fwd", "combine", "bwd_prep", "attn_bwd", "bwd_final", "fused_fwd")


class LshAttnError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}" + (f" ({detail})" if detail else ""))


class Desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "L", "d", "n_buckets", "n_hashes", "chunk", "causal", "dtype", "flags")]


_lib = None


def load_library(path: str = LIB_PATH):
    """Loads liblsh_attn.so and declares its signatures (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m lsh_attention_02_b200.build`")
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    DP = ctypes.POINTER(Desc)
    S = ctypes.c_size_t
    L.lsh_attn_make_rotations.argtypes = [ctypes.c_uint64, DP, P]
    L.lsh_attn_workspace_size.argtypes = [DP, ctypes.c_int]
    L.lsh_attn_workspace_size.restype = S
    L.lsh_attn_hash.argtypes = [DP, P, P, P, P, S, P]
    L.lsh_attn_sort.argtypes = [DP, P, P, P, S, P]
    L.lsh_attn_sort_static.argtypes = [DP, P, P, P]
    L.lsh_attn_fwd_sorted.argtypes = [DP, P, P, P, P, P, P, S, P]
    L.lsh_attn_fwd.argtypes = [DP, P, P, P, P, P, P, P, S, P]
    L.lsh_attn_bwd.argtypes = [DP, P, P, P, P, P, P, P, P, P, P, S, P]
    L.lsh_attn_local_workspace_size.argtypes = [DP, ctypes.c_int32, ctypes.c_int]
    L.lsh_attn_local_workspace_size.restype = S
    L.lsh_attn_local_fwd.argtypes = [DP, ctypes.c_int32, P, P, P, P, P, S, P]
    L.lsh_attn_local_bwd.argtypes = [DP, ctypes.c_int32, P, P, P, P, P, P, P, P, S, P]
    L.lsh_rev_workspace_size.argtypes = [DP, ctypes.c_int]
    L.lsh_rev_workspace_size.restype = S
    L.lsh_rev_fwd.argtypes = [DP, P, P, P, P, P, P, P, P, S, P]
    L.lsh_rev_bwd.argtypes = [DP, P, P, P, P, P, P, P, P, P, P, P, P, S, P]
    L.lsh_attn_step_host_scratch_size.argtypes = [DP, ctypes.c_int32, ctypes.c_int]
    L.lsh_attn_step_host_scratch_size.restype = S
    L.lsh_attn_step_host.argtypes = [DP, ctypes.c_int32, P, P, P, P, P, P, P, P, P, S, ctypes.POINTER(P)]
    L.lsh_attn_poll.argtypes = [P, P]
    L.lsh_attn_selftest_timeout.argtypes = [P, ctypes.c_int64, P]
    L.lsh_attn_trace_begin.argtypes = [ctypes.c_int32]
    L.lsh_attn_trace_stages.argtypes = [ctypes.c_uint32]
    L.lsh_attn_fused_forward.argtypes = [ctypes.c_int32]
    L.lsh_attn_fused_forward_fits.argtypes = [DP]
    L.lsh_attn_fused_forward_fits.restype = ctypes.c_int32
    L.lsh_attn_trace_end.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32),
                                     ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
    L.lsh_attn_last_near_ties.argtypes = []
    L.lsh_attn_last_near_ties.restype = ctypes.c_int
    L.lsh_attn_status_str.argtypes = [ctypes.c_int]
    L.lsh_attn_status_str.restype = ctypes.c_char_p
    L.lsh_attn_last_error.argtypes = []
    L.lsh_attn_last_error.restype = ctypes.c_char_p
    L.lsh_attn_abi_version.argtypes = []
    L.lsh_attn_abi_version.restype = ctypes.c_int32
    for name in EXPORTED:
        getattr(L, name).restype = getattr(L, name).restype or ctypes.c_int
    _lib = L
    return L


def make_desc(B, H, L, d, n_buckets, n_hashes, chunk, causal, dtype, flags=0) -> Desc:
    if isinstance(dtype, torch.dtype):
        dtype = {torch.float32: LSH_F32, torch.bfloat16: LSH_BF16}[dtype]
    return Desc(B, H, L, d, n_buckets, n_hashes, chunk, int(bool(causal)), dtype, flags)


def desc_for(x: torch.Tensor, n_buckets: int, n_hashes: int, chunk: int, causal: bool, flags: int = 0):
    B, H, L, d = x.shape
    return make_desc(B, H, L, d, n_buckets, n_hashes, chunk, causal, x.dtype, flags)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(rc: int, where: str):
    if rc != 0:
        detail = load_library().lsh_attn_last_error().decode() if rc == -5 else ""
        raise LshAttnError(rc, where, detail)


def make_rotations(desc: Desc, seed: int) -> torch.Tensor:
    """Host tensor R [n_hashes, d, n_buckets/2] (float32 or bfloat16) drawn from
    `seed` by the library's generator."""
    shape = (desc.n_hashes, desc.d, desc.n_buckets // 2)
    dt = torch.bfloat16 if desc.dtype == LSH_BF16 else torch.float32
    R = torch.empty(shape, dtype=dt)
    _check(load_library().lsh_attn_make_rotations(ctypes.c_uint64(seed), ctypes.byref(desc), _ptr(R)),
           "lsh_attn_make_rotations")
    return R


def workspace_size(desc: Desc, for_backward: bool) -> int:
    return int(load_library().lsh_attn_workspace_size(ctypes.byref(desc), int(for_backward)))


def workspace(desc: Desc, for_backward: bool, device) -> torch.Tensor:
    n = workspace_size(desc, for_backward)
    if n == 0:
        raise LshAttnError(-1, "workspace_size", "invalid descriptor")
    return torch.empty(n, dtype=torch.uint8, device=device)


def _ws(desc, for_backward, ref, ws):
    return ws if ws is not None else workspace(desc, for_backward, ref.device)


def lsh_attn_hash(desc: Desc, qk, R, buckets, ws=None):
    ws = _ws(desc, False, qk, ws)
    _check(load_library().lsh_attn_hash(ctypes.byref(desc), _ptr(qk), _ptr(R), _ptr(buckets), _ptr(ws),
                                         ws.numel(), _stream(qk)), "lsh_attn_hash")
    return buckets


def lsh_attn_sort(desc: Desc, buckets, perm, ws=None):
    ws = _ws(desc, False, buckets, ws)
    _check(load_library().lsh_attn_sort(ctypes.byref(desc), _ptr(buckets), _ptr(perm), _ptr(ws), ws.numel(),
                                         _stream(buckets)), "lsh_attn_sort")
    return perm


def lsh_attn_sort_static(desc: Desc, buckets, perm):
    """Same result as lsh_attn_sort, with the library's fixed per-device
    scratch instead of a workspace (no allocation; calls on one device must
    not overlap in time)."""
    rc = load_library().lsh_attn_sort_static(ctypes.byref(desc), _ptr(buckets), _ptr(perm), _stream(buckets))
    if rc == -7:
        raise LshAttnError(rc, "lsh_attn_sort_static", load_library().lsh_attn_last_error().decode())
    _check(rc, "lsh_attn_sort_static")
    return perm


def lsh_attn_fwd_sorted(desc: Desc, qk, v, perm, out, lse, ws=None):
    ws = _ws(desc, False, qk, ws)
    _check(load_library().lsh_attn_fwd_sorted(ctypes.byref(desc), _ptr(qk), _ptr(v), _ptr(perm), _ptr(out),
                                               _ptr(lse), _ptr(ws), ws.numel(), _stream(qk)),
           "lsh_attn_fwd_sorted")
    return out, lse


def lsh_attn_fwd(desc: Desc, qk, v, R, out, lse, perm_out=None, ws=None):
    ws = _ws(desc, False, qk, ws)
    _check(load_library().lsh_attn_fwd(ctypes.byref(desc), _ptr(qk), _ptr(v), _ptr(R), _ptr(out), _ptr(lse),
                                        _ptr(perm_out), _ptr(ws), ws.numel(), _stream(qk)), "lsh_attn_fwd")
    return out, lse


def lsh_attn_bwd(desc: Desc, qk, v, R, out, lse, perm, dout, dqk, dv, ws=None):
    ws = _ws(desc, True, qk, ws)
    _check(load_library().lsh_attn_bwd(ctypes.byref(desc), _ptr(qk), _ptr(v), _ptr(R), _ptr(out), _ptr(lse),
                                        _ptr(perm), _ptr(dout), _ptr(dqk), _ptr(dv), _ptr(ws), ws.numel(),
                                        _stream(qk)), "lsh_attn_bwd")
    return dqk, dv


def local_workspace(desc: Desc, chunks_after: int, for_backward: bool, device) -> torch.Tensor:
    n = int(load_library().lsh_attn_local_workspace_size(ctypes.byref(desc), int(chunks_after), int(for_backward)))
    if n == 0:
        raise LshAttnError(-1, "lsh_attn_local_workspace_size", "invalid descriptor")
    return torch.empty(n, dtype=torch.uint8, device=device)


def lsh_attn_local_fwd(desc: Desc, chunks_after: int, qk, v, out, lse, ws=None):
    """Local chunk attention (no hashing): out [B,H,L,64], lse [B,H,1,L]."""
    ws = ws if ws is not None else local_workspace(desc, chunks_after, False, qk.device)
    _check(load_library().lsh_attn_local_fwd(ctypes.byref(desc), int(chunks_after), _ptr(qk), _ptr(v), _ptr(out),
                                              _ptr(lse), _ptr(ws), ws.numel(), _stream(qk)), "lsh_attn_local_fwd")
    return out, lse


def lsh_attn_local_bwd(desc: Desc, chunks_after: int, qk, v, out, lse, dout, dqk, dv, ws=None):
    ws = ws if ws is not None else local_workspace(desc, chunks_after, True, qk.device)
    _check(load_library().lsh_attn_local_bwd(ctypes.byref(desc), int(chunks_after), _ptr(qk), _ptr(v), _ptr(out),
                                              _ptr(lse), _ptr(dout), _ptr(dqk), _ptr(dv), _ptr(ws), ws.numel(),
                                              _stream(qk)), "lsh_attn_local_bwd")
    return dqk, dv


def rev_workspace(desc: Desc, for_backward: bool, device) -> torch.Tensor:
    n = int(load_library().lsh_rev_workspace_size(ctypes.byref(desc), int(for_backward)))
    if n == 0:
        raise LshAttnError(-1, "lsh_rev_workspace_size", "invalid descriptor")
    return torch.empty(n, dtype=torch.uint8, device=device)


def lsh_rev_fwd(desc: Desc, x1, x2, R, Wg, bg, y1, y2, ws=None):
    """Reversible block forward: y1 = x1 + LSHAttn(x2, x2), y2 = x2 + tanh(y1 Wg + bg); fp32 streams."""
    ws = ws if ws is not None else rev_workspace(desc, False, x1.device)
    _check(load_library().lsh_rev_fwd(ctypes.byref(desc), _ptr(x1), _ptr(x2), _ptr(R), _ptr(Wg), _ptr(bg),
                                       _ptr(y1), _ptr(y2), _ptr(ws), ws.numel(), _stream(x1)), "lsh_rev_fwd")
    return y1, y2


def lsh_rev_bwd(desc: Desc, y1, y2, dy1, dy2, R, Wg, bg, x1, x2, dx1, dx2, ws=None):
    """Reversible block backward from the outputs: recovers x1, x2 and writes dx1, dx2."""
    ws = ws if ws is not None else rev_workspace(desc, True, y1.device)
    _check(load_library().lsh_rev_bwd(ctypes.byref(desc), _ptr(y1), _ptr(y2), _ptr(dy1), _ptr(dy2), _ptr(R),
                                       _ptr(Wg), _ptr(bg), _ptr(x1), _ptr(x2), _ptr(dx1), _ptr(dx2), _ptr(ws),
                                       ws.numel(), _stream(y1)), "lsh_rev_bwd")
    return x1, x2, dx1, dx2


def step_host_scratch(desc: Desc, heads_per_chunk: int, with_backward: bool, device) -> torch.Tensor:
    n = int(load_library().lsh_attn_step_host_scratch_size(ctypes.byref(desc), int(heads_per_chunk),
                                                           int(with_backward)))
    if n == 0:
        raise LshAttnError(-1, "lsh_attn_step_host_scratch_size", "invalid descriptor")
    return torch.empty(n, dtype=torch.uint8, device=device)


def lsh_attn_step_host(desc: Desc, qk_h, v_h, R_h, dout_h, out_h, lse_h, dqk_h, dv_h, scratch, streams,
                       heads_per_chunk: int = 0):
    """Forward (+ backward when dout_h is given) on host tensors (pinned for overlap),
    pipelined per chunk of heads over three torch CUDA streams (compute, copy in,
    copy out); synchronise on streams[0]."""
    arr = (ctypes.c_void_p * 3)(*[s.cuda_stream for s in streams])
    _check(load_library().lsh_attn_step_host(ctypes.byref(desc), int(heads_per_chunk), _ptr(qk_h), _ptr(v_h),
                                              _ptr(R_h), _ptr(dout_h), _ptr(out_h), _ptr(lse_h), _ptr(dqk_h),
                                              _ptr(dv_h), _ptr(scratch), scratch.numel(), arr),
           "lsh_attn_step_host")


def lsh_attn_poll(ws: torch.Tensor) -> int:
    """Synchronises the current stream and returns the device status (0 or LSH_ERR_TIMEOUT)."""
    return int(load_library().lsh_attn_poll(_ptr(ws), _stream(ws)))


def lsh_attn_selftest_timeout(ws: torch.Tensor, budget_cycles: int):
    """Runs the bounded-wait self-test kernel on the current stream (see the header)."""
    _check(load_library().lsh_attn_selftest_timeout(_ptr(ws), int(budget_cycles), _stream(ws)),
           "lsh_attn_selftest_timeout")


def trace_begin(capacity: int = 4096):
    """Starts recording a CUDA event pair around every stage the library enqueues."""
    _check(load_library().lsh_attn_trace_begin(int(capacity)), "lsh_attn_trace_begin")


def trace_stages(names=None):
    """Restricts what a trace records to the named stages (None: every stage)."""
    mask = 0xFFFFFFFF if names is None else sum(1 << STAGES.index(n) for n in names)
    _check(load_library().lsh_attn_trace_stages(mask), "lsh_attn_trace_stages")


def fused_forward(mode=1):
    """Single-kernel forward of short segments, process-wide: 1 (or True; the
    default) where it fits and its segments fill the GPU's waves, 2 wherever it
    fits, 0 (or False) never."""
    mode = int(mode)
    _check(load_library().lsh_attn_fused_forward(mode), "lsh_attn_fused_forward")


def fused_forward_fits(desc) -> bool:
    """Whether a forward with this descriptor runs as the single kernel under the current setting."""
    return bool(load_library().lsh_attn_fused_forward_fits(ctypes.byref(desc)))


def trace_end() -> dict:
    """Stops recording; returns {stage: (total_ms, calls, kernels)}."""
    n = len(STAGES)
    ms = (ctypes.c_float * n)(); calls = (ctypes.c_int32 * n)(); ker = (ctypes.c_int32 * n)()
    _check(load_library().lsh_attn_trace_end(ms, calls, ker, n), "lsh_attn_trace_end")
    return {name: (float(ms[i]), int(calls[i]), int(ker[i])) for i, name in enumerate(STAGES)}


def outputs_like(desc: Desc, qk: torch.Tensor):
    """Fresh (out, lse, perm) buffers for a forward call."""
    B, H, L = desc.B, desc.H, desc.L
    out = torch.empty_like(qk)
    lse = torch.empty((B, H, desc.n_hashes, L), dtype=torch.float32, device=qk.device)
    perm = torch.empty((B, H, desc.n_hashes, L), dtype=torch.int32, device=qk.device)
    return out, lse, perm


class LSHAttention(torch.autograd.Function):
    """y = LSHAttention.apply(qk, v, R, n_buckets, chunk, causal[, flags]); gradients for qk and v."""

    @staticmethod
    def forward(ctx, qk, v, R, n_buckets, chunk, causal, flags=0):
        qk = qk.contiguous(); v = v.contiguous(); R = R.contiguous()
        desc = desc_for(qk, n_buckets, R.shape[0], chunk, causal, flags)
        out, lse, perm = outputs_like(desc, qk)
        lsh_attn_fwd(desc, qk, v, R, out, lse, perm)
        ctx.desc = desc
        ctx.save_for_backward(qk, v, R, out, lse, perm)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        qk, v, R, out, lse, perm = ctx.saved_tensors
        dqk = torch.empty_like(qk); dv = torch.empty_like(v)
        lsh_attn_bwd(ctx.desc, qk, v, R, out, lse, perm, dout.contiguous(), dqk, dv)
        return dqk, dv, None, None, None, None, None


def lsh_attention(qk, v, R, n_buckets, chunk=64, causal=False, flags=0):
    """Reformer LSH self-attention with shared query-key: returns (out, lse).

    qk, v: [B, H, L, 64] CUDA tensors (float32 or bfloat16); R: [n_hashes, 64, n_buckets/2];
    flags: FLAG_BUCKET_MASK | FLAG_SELF_PENALTY (0 = the default semantics)."""
    return LSHAttention.apply(qk, v, R, n_buckets, chunk, causal, flags)

