"""Helpers shared by the GPU parity tests: device upload, the library calls in
the order the benchmark makes them, and the error metrics with their bounds."""
from __future__ import annotations

import numpy as np
import torch

import lsh_attention_02_b200 as lsh

# Tolerances: fp32 path <= 1e-4 max-abs; bf16 inputs with fp32 accumulation
# <= 2e-2 max-abs and <= 1e-2 relative L2, for outputs and gradients.
TOL = {"f32": {"max_abs": 1e-4, "rel_l2": None}, "bf16": {"max_abs": 2e-2, "rel_l2": 1e-2}}
NEAR_TIE = 1e-6          # relative top-two gap below which an argmax flip is reported, not failed


def torch_dtype(dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


def to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Host float32 array (already representable in `dtype`) -> CUDA tensor, exactly."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(torch_dtype(dtype))


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def errors(got: np.ndarray, want: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64); want = np.asarray(want, dtype=np.float64)
    diff = got - want
    return {"max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
            "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-300))}


def assert_close(got, want, dtype: str, what: str):
    e = errors(got, want)
    tol = TOL[dtype]
    msg = f"{what}: max_abs={e['max_abs']:.3e} rel_l2={e['rel_l2']:.3e} (dtype {dtype})"
    assert e["max_abs"] <= tol["max_abs"], msg
    if tol["rel_l2"] is not None:
        assert e["rel_l2"] <= tol["rel_l2"], msg
    return e


def check_buckets(gpu_b: np.ndarray, ora_b: np.ndarray, margin: np.ndarray, what: str) -> int:
    """Bucket ids must agree except where the oracle's top-two gap is a near tie;
    returns the number of such flips (reported by the caller)."""
    diff = gpu_b.astype(np.int64) != ora_b.astype(np.int64)
    bad = diff & (margin >= NEAR_TIE)
    assert not bad.any(), f"{what}: {int(bad.sum())} bucket mismatches away from near ties " \
                          f"(first at {np.argwhere(bad)[0].tolist()}, margin {margin[bad].min():.3e})"
    return int(diff.sum())


def check_perm_is_stable_sort(perm: np.ndarray, buckets: np.ndarray, what: str):
    """perm[..., s] must equal the stable argsort of buckets[...] (bit-exact)."""
    flat_p = perm.reshape(-1, perm.shape[-1]); flat_b = buckets.reshape(-1, buckets.shape[-1])
    for k in range(flat_p.shape[0]):
        want = np.argsort(flat_b[k], kind="stable")
        if not np.array_equal(flat_p[k], want):
            first = int(np.nonzero(flat_p[k] != want)[0][0])
            raise AssertionError(f"{what}: segment {k} differs from the stable sort at slot {first}")


class Run:
    """One forward (and optionally backward) through the C ABI, as the benchmark calls it."""

    def __init__(self, inp: dict, n_buckets: int, chunk: int, causal: bool, dtype: str, flags: int = 0):
        self.dtype = dtype
        self.x = to_dev(inp["x"], dtype)
        self.v = to_dev(inp["v"], dtype)
        self.R = to_dev(inp["R"], dtype)
        self.desc = lsh.desc_for(self.x, n_buckets, inp["R"].shape[0], chunk, causal, flags)
        self.out, self.lse, self.perm = lsh.outputs_like(self.desc, self.x)
        self.ws = lsh.workspace(self.desc, False, self.x.device)
        lsh.lsh_attn_fwd(self.desc, self.x, self.v, self.R, self.out, self.lse, self.perm, self.ws)
        B, H, L = self.desc.B, self.desc.H, self.desc.L
        self.buckets = torch.empty((B, H, self.desc.n_hashes, L), dtype=torch.int16, device=self.x.device)
        lsh.lsh_attn_hash(self.desc, self.x, self.R, self.buckets, self.ws)
        assert lsh.lsh_attn_poll(self.ws) == 0
        if "dy" in inp:
            self.dy = to_dev(inp["dy"], dtype)
            self.dx = torch.empty_like(self.x); self.dv = torch.empty_like(self.v)
            wsb = lsh.workspace(self.desc, True, self.x.device)
            lsh.lsh_attn_bwd(self.desc, self.x, self.v, self.R, self.out, self.lse, self.perm, self.dy,
                             self.dx, self.dv, wsb)
            assert lsh.lsh_attn_poll(wsb) == 0
        torch.cuda.synchronize()

    def host_buckets(self) -> np.ndarray:
        return self.buckets.cpu().numpy().view(np.uint16).astype(np.int64)
