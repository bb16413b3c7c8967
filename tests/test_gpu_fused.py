"""The single-kernel forward of short segments (hash, sort, attention and the
round merge in one cluster per head) against the staged kernels and the CPU
oracle.

Both paths compute the same products with the same tie rule and the same
merge arithmetic, so their bucket ids, permutations, logsumexps and outputs
are compared bit for bit; the oracle comparison uses the tolerances of the
other parity tests (bf16: 2e-2 max-abs, 1e-2 relative L2)."""
import numpy as np
import pytest
import torch

import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import synth
from oracle import oracle
from tests.gpu_util import Run, assert_close, check_buckets, check_perm_is_stable_sort, to_host

pytestmark = pytest.mark.gpu


def small(**kw):
    return synth.WORKLOADS["bf16_causal_4k"].replace(**kw)


def run_both(w, inp, flags=0, mode=2):
    """The forward with the single kernel (setting `mode`; 2: wherever it fits,
    so that small shapes reach it), then with the staged kernels."""
    try:
        lsh.fused_forward(mode)
        fused = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype, flags)
        assert lsh.fused_forward_fits(fused.desc)
        lsh.fused_forward(0)
        staged = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype, flags)
        assert not lsh.fused_forward_fits(staged.desc)
    finally:
        lsh.fused_forward(1)
    return fused, staged


# (L, n_buckets, n_hashes, causal, flags): one chunk; a last tile of one chunk;
# the largest segment; 2 and 128 buckets (16 and 64 rotation columns) and an
# odd column count; 1, 3 and 8 rounds (cluster sizes); both optional readings
CASES = [
    (64, 16, 2, True, 0), (192, 8, 2, False, 0), (4096, 64, 2, True, 0), (4032, 32, 3, True, 0),
    (1024, 2, 2, True, 0), (1024, 128, 2, False, 0), (704, 34, 2, True, 0), (512, 16, 1, True, 0),
    (512, 16, 8, False, 0), (960, 64, 2, True, lsh.FLAG_BUCKET_MASK), (960, 64, 2, False, lsh.FLAG_SELF_PENALTY),
    (1152, 128, 3, True, lsh.FLAG_BUCKET_MASK | lsh.FLAG_SELF_PENALTY),
]


@pytest.mark.parametrize("L,nb,nh,causal,flags", CASES)
def test_fused_equals_staged(L, nb, nh, causal, flags):
    w = small(B=2, H=2, L=L, n_buckets=nb, n_hashes=nh, causal=causal, backward=False)
    inp = synth.make_inputs(w)
    fused, staged = run_both(w, inp, flags)
    # the fused kernel's permutation is the stable sort of the hash kernel's bucket ids
    check_perm_is_stable_sort(fused.perm.cpu().numpy(), fused.host_buckets(), "fused perm")
    assert torch.equal(fused.perm, staged.perm), "permutation"
    assert torch.equal(fused.lse, staged.lse), "per-round logsumexp"
    assert torch.equal(fused.out, staged.out), "merged output"


@pytest.mark.parametrize("L,nb,nh,causal,flags", [(4096, 64, 2, True, 0), (960, 64, 2, False, 0),
                                                  (1024, 16, 3, True, lsh.FLAG_BUCKET_MASK)])
def test_fused_forward_then_backward_against_oracle(L, nb, nh, causal, flags):
    """Buckets and permutation of the fused forward against the oracle's hash
    and stable sort, outputs and lse against the oracle with that permutation,
    and the backward run from the fused forward's permutation, lse and output."""
    w = small(B=1, H=3, L=L, n_buckets=nb, n_hashes=nh, causal=causal, backward=True)
    inp = synth.make_inputs(w)
    inp["dy"] = (inp["dy"] / 4.0).astype(np.float32)           # exact: a power of two
    try:
        lsh.fused_forward(2)
        run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype, flags)
        assert lsh.fused_forward_fits(run.desc)
    finally:
        lsh.fused_forward(1)
    gb = run.host_buckets()
    gperm = run.perm.cpu().numpy()
    check_perm_is_stable_sort(gperm, gb, "fused perm")
    flips = 0
    for h in range(w.H):
        ref = oracle.fwd(inp["x"][:, h:h + 1], inp["v"][:, h:h + 1], inp["R"], nb, w.chunk, causal)
        flips += check_buckets(gb[0, h], ref["bucket"][0, 0], ref["margin"][0, 0], f"fused ({h})")
        if flips == 0:
            np.testing.assert_array_equal(gperm[0, h], ref["perm"][0, 0])
    bk = gb if flags & lsh.FLAG_BUCKET_MASK else None
    y, lr = oracle.fwd_perm(inp["x"], inp["v"], gperm, w.chunk, causal, bucket=bk)
    assert_close(to_host(run.out), y, "bf16", "out")
    assert_close(run.lse.cpu().numpy(), lr, "bf16", "lse")
    dx, dv = oracle.bwd(inp["x"], inp["v"], inp["dy"], gperm, w.chunk, causal, bucket=bk)
    assert_close(to_host(run.dx), dx, "bf16", "dqk")
    assert_close(to_host(run.dv), dv, "bf16", "dv")
    print(f"[near-tie] fused L={L}: {flips} argmax flips")


def test_fused_forward_full_workload_equals_staged():
    """The 4K-token forward workload (8 x 8 heads, 64 buckets, 2 rounds) in the
    launch configuration the benchmark times: both paths bit for bit."""
    w = synth.WORKLOADS["bf16_causal_4k"]
    inp = synth.make_inputs(w)
    fused, staged = run_both(w, inp, mode=1)             # the default setting takes it (128 segments)
    assert torch.equal(fused.perm, staged.perm)
    assert torch.equal(fused.lse, staged.lse)
    assert torch.equal(fused.out, staged.out)


def test_fused_forward_without_permutation_output_then_recomputing_backward():
    """The single kernel writes the permutation into the workspace when the
    caller passes none; the outputs equal those of the call that asks for it,
    and a backward that recomputes the permutation from R gives the gradients
    of the backward that is handed it (same buckets, so the same bits up to
    the fp32 reductions' order)."""
    w = small(B=2, H=2, L=2048, n_buckets=64, n_hashes=2, causal=True, backward=True)
    inp = synth.make_inputs(w)
    try:
        lsh.fused_forward(2)
        run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
        assert lsh.fused_forward_fits(run.desc)
        out2, lse2 = torch.empty_like(run.out), torch.empty_like(run.lse)
        lsh.lsh_attn_fwd(run.desc, run.x, run.v, run.R, out2, lse2, None)
        torch.cuda.synchronize()
    finally:
        lsh.fused_forward(1)
    assert torch.equal(out2, run.out) and torch.equal(lse2, run.lse)
    dx2, dv2 = torch.empty_like(run.x), torch.empty_like(run.v)
    lsh.lsh_attn_bwd(run.desc, run.x, run.v, run.R, run.out, run.lse, None, run.dy, dx2, dv2)
    torch.cuda.synchronize()
    assert_close(to_host(dx2), to_host(run.dx), "bf16", "dqk, permutation recomputed")
    assert_close(to_host(dv2), to_host(run.dv), "bf16", "dv, permutation recomputed")
