"""Exact properties of the method checked on the CUDA path, at sizes and
bucket counts the element-by-element parity cases also use.

* "LSH Attention", hash equation h(x) = argmax [xR ; -xR]: a power-of-two
  scale of x scales every product and every partial sum exactly, in bf16 and
  in fp32, so the bucket ids must not change at all; negating x exchanges the
  halves of [xR ; -xR] (products and sums negate exactly), so without a near
  tie every bucket moves by n_buckets / 2.
* "LSH Attention", output equation: the weights depend on x alone, so doubling
  v doubles every per-round output and the merged output exactly (a
  power-of-two scale commutes with every rounding), and leaves lse and the
  permutation unchanged.  Checked through the staged kernels and the single
  kernel of short segments.
"""
import numpy as np
import pytest
import torch

import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import synth
from oracle import oracle
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

NEAR = 1e-5        # rows whose oracle top-two gap is below this may resolve a tie differently


def _hash(desc, x, R, shape):
    bk = torch.empty(shape, dtype=torch.int16, device="cuda")
    lsh.lsh_attn_hash(desc, x, R, bk)
    return bk.cpu().numpy().view(np.uint16).astype(np.int64)


@pytest.mark.parametrize("dtype,nb,nh", [("bf16", 64, 2), ("bf16", 1024, 2), ("bf16", 100, 1), ("bf16", 8192, 1),
                                         ("f32", 16, 2), ("f32", 8192, 1)])
def test_hash_scale_and_negation(dtype, nb, nh):
    L = 1024 if nb < 8192 else 256
    w = synth.WORKLOADS["bf16_causal_4k"].replace(B=1, H=2, L=L, n_buckets=nb, n_hashes=nh, dtype=dtype)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], dtype); R = to_dev(inp["R"], dtype)
    desc = lsh.desc_for(x, nb, nh, 64, True)
    shape = (1, 2, nh, L)
    b0 = _hash(desc, x, R, shape)
    for c in (4.0, 0.125):
        np.testing.assert_array_equal(_hash(desc, x * c, R, shape), b0, err_msg=f"scale {c}")
    bn = _hash(desc, -x, R, shape)
    moved = (b0 + nb // 2) % nb
    near = np.zeros(shape, dtype=bool)
    for h in range(2):
        for r in range(nh):
            _, mg = oracle.hash_round(inp["x"][0, h], inp["R"][r], nb)
            near[0, h, r] = mg < NEAR
    bad = (bn != moved) & ~near
    assert not bad.any(), f"{int(bad.sum())} rows do not move by nb/2 under negation"
    print(f"[negation] nb={nb} {dtype}: {int(((bn != moved) & near).sum())} near-tie rows differ, "
          f"{int(near.sum())} near-tie rows in {near.size}")


@pytest.mark.parametrize("mode", [0, 2])
@pytest.mark.parametrize("causal,flags", [(True, 0), (False, 0), (True, lsh.FLAG_BUCKET_MASK | lsh.FLAG_SELF_PENALTY)])
def test_output_doubles_with_values(mode, causal, flags):
    """mode 0: the staged kernels; mode 2: the single kernel of short segments;
    flags: the bucket mask and the self penalty."""
    w = synth.WORKLOADS["bf16_causal_4k"].replace(B=1, H=2, L=2048, causal=causal)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], "bf16"); v = to_dev(inp["v"], "bf16"); R = to_dev(inp["R"], "bf16")
    desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, causal, flags)
    try:
        lsh.fused_forward(mode)
        assert lsh.fused_forward_fits(desc) == (mode == 2)
        res = []
        for vv in (v, v * 2):
            out, lse, perm = lsh.outputs_like(desc, x)
            lsh.lsh_attn_fwd(desc, x, vv, R, out, lse, perm)
            res.append((out, lse, perm))
        torch.cuda.synchronize()
    finally:
        lsh.fused_forward(1)
    (o1, l1, p1), (o2, l2, p2) = res
    assert torch.equal(o2, o1 * 2)
    assert torch.equal(l2, l1)
    assert torch.equal(p2, p1)


@pytest.mark.parametrize("after", [0, 1])
def test_local_output_doubles_with_values(after):
    """Local chunk attention (no hashing), with and without the following chunk."""
    L = 1024
    w = synth.WORKLOADS["long_64k"].replace(B=1, H=2, L=L, n_hashes=1, causal=after == 0)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], "bf16"); v = to_dev(inp["v"], "bf16")
    desc = lsh.make_desc(1, 2, L, 64, 2, 1, 64, after == 0, dtype=torch.bfloat16)
    res = []
    for vv in (v, v * 2):
        out = torch.empty_like(x)
        lse = torch.empty((1, 2, 1, L), dtype=torch.float32, device="cuda")
        lsh.lsh_attn_local_fwd(desc, after, x, vv, out, lse)
        res.append((out, lse))
    torch.cuda.synchronize()
    (o1, l1), (o2, l2) = res
    assert torch.equal(o2, o1 * 2)
    assert torch.equal(l2, l1)


@pytest.mark.parametrize("mode", [0, 2])
def test_heads_are_independent(mode):
    """Each (batch, head) slice is its own problem: the forward of a 2 x 2
    problem equals the forward of every slice alone, bit for bit (merged
    output, per-round lse and permutation), through the staged kernels (mode
    0) and the single kernel (mode 2)."""
    w = synth.WORKLOADS["bf16_causal_4k"].replace(B=2, H=2, L=1024)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], "bf16"); v = to_dev(inp["v"], "bf16"); R = to_dev(inp["R"], "bf16")
    desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, w.causal)
    try:
        lsh.fused_forward(mode)
        out, lse, perm = lsh.outputs_like(desc, x)
        lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm)
        for b in range(2):
            for h in range(2):
                xs = x[b:b + 1, h:h + 1].contiguous(); vs = v[b:b + 1, h:h + 1].contiguous()
                ds = lsh.desc_for(xs, w.n_buckets, w.n_hashes, w.chunk, w.causal)
                assert lsh.fused_forward_fits(ds) == (mode == 2)
                o1, l1, p1 = lsh.outputs_like(ds, xs)
                lsh.lsh_attn_fwd(ds, xs, vs, R, o1, l1, p1)
                torch.cuda.synchronize()
                assert torch.equal(o1[0, 0], out[b, h]), (b, h)
                assert torch.equal(l1[0, 0], lse[b, h]), (b, h)
                assert torch.equal(p1[0, 0], perm[b, h]), (b, h)
    finally:
        lsh.fused_forward(1)
