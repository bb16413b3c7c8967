"""GPU parity: the CUDA library through its C ABI against the CPU oracle on the
same seeded inputs.

Bucket ids and permutations are compared bit for bit (an argmax flip is
allowed only where the oracle's top-two gap is below 1e-6 relative, and is
counted and printed).  To keep a flip from spreading, attention outputs and
gradients are compared with the GPU's own permutation injected into the
oracle.  Floating-point bounds: fp32 1e-4 max-abs; bf16 2e-2 max-abs and
1e-2 relative L2.
"""
import numpy as np
import pytest
import torch

import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import synth
from oracle import oracle
from tests.gpu_util import (NEAR_TIE, Run, assert_close, check_buckets, check_perm_is_stable_sort, errors,
                            to_dev, to_host, torch_dtype)

pytestmark = pytest.mark.gpu

def small(name, **kw):
    return synth.WORKLOADS[name].replace(**kw)


def _flip_report(tag, flips, total):
    print(f"[near-tie] {tag}: {flips} argmax flips out of {total} row-rounds")


def full_check(w: synth.Workload, heads=None, inp=None):
    """Runs fwd (+bwd) on the GPU for workload w and checks (b, h) slices `heads`
    (all when None) against the oracle."""
    inp = synth.make_inputs(w) if inp is None else inp
    run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    B, H, L = w.B, w.H, w.L
    sel = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    gb = run.host_buckets()
    gperm = run.perm.cpu().numpy()
    out, lse = to_host(run.out), run.lse.cpu().numpy().astype(np.float64)
    check_perm_is_stable_sort(gperm, gb, f"{w.name} perm")
    flips = 0
    for b, h in sel:
        xs, vs = inp["x"][b:b + 1, h:h + 1], inp["v"][b:b + 1, h:h + 1]
        ref = oracle.fwd(xs, vs, inp["R"], w.n_buckets, w.chunk, w.causal)
        flips += check_buckets(gb[b, h], ref["bucket"][0, 0], ref["margin"][0, 0], f"{w.name} ({b},{h})")
        if flips == 0:
            np.testing.assert_array_equal(gperm[b, h], ref["perm"][0, 0])
        y, lr = oracle.fwd_perm(xs, vs, gperm[b:b + 1, h:h + 1], w.chunk, w.causal)
        assert_close(out[b, h], y[0, 0], w.dtype, f"{w.name} ({b},{h}) out")
        assert_close(lse[b, h], lr[0, 0], "f32" if w.dtype == "f32" else "bf16", f"{w.name} ({b},{h}) lse")
        if w.backward:
            dx, dv = oracle.bwd(xs, vs, inp["dy"][b:b + 1, h:h + 1], gperm[b:b + 1, h:h + 1], w.chunk, w.causal)
            assert_close(to_host(run.dx[b, h]), dx[0, 0], w.dtype, f"{w.name} ({b},{h}) dqk")
            assert_close(to_host(run.dv[b, h]), dv[0, 0], w.dtype, f"{w.name} ({b},{h}) dv")
    _flip_report(w.name, flips, len(sel) * w.n_hashes * L)
    return run


# ------------------------------------------------------------------ stage: hash
@pytest.mark.parametrize("dtype,nb,nh", [("f32", 16, 1), ("bf16", 64, 2), ("bf16", 1024, 3), ("bf16", 192, 2),
                                         ("bf16", 128, 2), ("bf16", 2, 2), ("f32", 8192, 1), ("bf16", 8192, 2),
                                         ("bf16", 6, 2), ("bf16", 100, 1), ("bf16", 200, 2), ("f32", 6, 2)])
def test_hash_bit_exact_up_to_near_ties(dtype, nb, nh):
    """Bucket counts whose half is a multiple of 128, 96 or 64 use whole N-tiles;
    the others (2, 6, 100, 200) pad the last tile with zero rotation columns."""
    w = small("bf16_causal_4k", B=2, H=2, L=1024 if nb < 8192 else 256, n_buckets=nb, n_hashes=nh, dtype=dtype)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], dtype); R = to_dev(inp["R"], dtype)
    desc = lsh.desc_for(x, nb, nh, 64, True)
    bk = torch.empty((2, 2, nh, w.L), dtype=torch.int16, device="cuda")
    lsh.lsh_attn_hash(desc, x, R, bk)
    gb = bk.cpu().numpy().view(np.uint16).astype(np.int64)
    flips = 0
    for b in range(2):
        for h in range(2):
            for r in range(nh):
                ob, mg = oracle.hash_round(inp["x"][b, h], inp["R"][r], nb)
                flips += check_buckets(gb[b, h, r], ob, mg, f"hash nb={nb} ({b},{h},{r})")
    _flip_report(f"hash {dtype} nb={nb}", flips, 4 * nh * w.L)


def test_hash_extreme_magnitudes_and_exact_ties():
    """Rows by blocks of 128 (whole warps alike): zero rows, signed one-hot rows
    (the projection is a row of R exactly, so equal bf16 entries make exact ties
    that must go to the lowest index), and Gaussian rows scaled by 2^-110, 2^-60
    and 2^40; one block mixes 2^-110 rows with plain ones.  Zero and one-hot rows
    must match bit for bit; the others up to near ties."""
    nb, nh, L = 1024, 2, 1024
    w = small("bf16_causal_4k", B=1, H=2, L=L, n_buckets=nb, n_hashes=nh)
    inp = synth.make_inputs(w)
    x = inp["x"].astype(np.float64).copy()
    exact = np.zeros((2, L), dtype=bool)
    for h in range(2):
        for i in range(L):
            blk = i // 128
            onehot = np.zeros(64)
            onehot[(i * 7 + h) % 64] = 1.0
            if blk == 0:
                x[0, h, i] = 0.0
            elif blk == 1:
                x[0, h, i] = onehot * 2.0 ** (i % 3 - 1)
            elif blk == 2:
                x[0, h, i] *= 2.0 ** -110
            elif blk == 3:
                x[0, h, i] *= 2.0 ** -60
            elif blk == 4:
                x[0, h, i] *= 2.0 ** 40
            elif blk == 5:
                x[0, h, i] = onehot * 2.0 ** -110
            elif blk == 6:
                x[0, h, i] *= 2.0 ** -110 if i % 2 == 0 else 1.0
            else:
                x[0, h, i] = -onehot
            exact[h, i] = blk in (0, 1, 5, 7)
    xd = to_dev(x.astype(np.float32), "bf16"); R = to_dev(inp["R"], "bf16")
    desc = lsh.desc_for(xd, nb, nh, 64, True)
    bk = torch.empty((1, 2, nh, L), dtype=torch.int16, device="cuda")
    lsh.lsh_attn_hash(desc, xd, R, bk)
    gb = bk.cpu().numpy().view(np.uint16).astype(np.int64)
    flips = 0
    for h in range(2):
        for r in range(nh):
            ob, mg = oracle.hash_round(x[0, h].astype(np.float32), inp["R"][r], nb)
            e = exact[h]
            np.testing.assert_array_equal(gb[0, h, r][e], ob[e], err_msg=f"exact rows h={h} r={r}")
            flips += check_buckets(gb[0, h, r][~e], ob[~e], mg[~e], f"scaled rows h={h} r={r}")
    _flip_report("hash extreme magnitudes", flips, 2 * nh * L)


# ------------------------------------------------------------------ stage: sort
@pytest.mark.parametrize("L,nb,dist", [(1, 2, "uniform"), (64, 2, "uniform"), (2048, 16, "uniform"),
                                       (2112, 1024, "uniform"), (12288, 192, "skewed"), (4096, 65536, "uniform"),
                                       (65536, 1024, "one_bucket"), (10240, 8192, "skewed"),
                                       (4160, 256, "descending")])
def test_sort_bit_exact(L, nb, dist):
    rng = np.random.default_rng(L + nb)
    S = 3
    if dist == "uniform":
        b = rng.integers(0, nb, size=(S, L))
    elif dist == "skewed":
        b = np.minimum((rng.pareto(1.2, size=(S, L)) * 3).astype(np.int64), nb - 1)
    elif dist == "one_bucket":
        b = np.full((S, L), nb // 3)
    else:
        b = np.tile(np.arange(L)[::-1] % nb, (S, 1))
    bk = torch.from_numpy(b.astype(np.uint16).view(np.int16).reshape(1, S, 1, L)).cuda()
    perm = torch.empty((1, S, 1, L), dtype=torch.int32, device="cuda")
    desc = lsh.make_desc(1, S, L, 64, nb, 1, 1, False, lsh.LSH_BF16)
    lsh.lsh_attn_sort(desc, bk, perm)
    got = perm.cpu().numpy().reshape(S, L)
    for s in range(S):
        np.testing.assert_array_equal(got[s], oracle.sort_segment(b[s]))


# ------------------------------------------------------------------ stage: attention with a given permutation
@pytest.mark.parametrize("dtype,causal,L,m,nh", [("f32", False, 1024, 64, 1), ("f32", True, 512, 32, 3),
                                                 ("bf16", True, 1024, 64, 2), ("bf16", False, 2048, 64, 4),
                                                 ("bf16", True, 960, 64, 2), ("f32", True, 48, 1, 2),
                                                 ("bf16", True, 64, 64, 1), ("f32", False, 128, 128, 2),
                                                 ("bf16", False, 576, 64, 3), ("bf16", True, 192, 64, 2)])
def test_attention_given_perm(dtype, causal, L, m, nh):
    """L = 960, 576, 192 and 64 leave the last 128-slot tile of the tensor-core
    kernels with one chunk only."""
    w = small("bf16_causal_4k", B=1, H=3, L=L, n_buckets=16, n_hashes=nh, chunk=m, causal=causal, dtype=dtype)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(L + nh)
    perm = np.stack([[rng.permutation(L) for _ in range(nh)] for _ in range(3)])[None].astype(np.int32)
    x, v = to_dev(inp["x"], dtype), to_dev(inp["v"], dtype)
    desc = lsh.desc_for(x, 16, nh, m, causal)
    out, lse, _ = lsh.outputs_like(desc, x)
    lsh.lsh_attn_fwd_sorted(desc, x, v, torch.from_numpy(perm).cuda(), out, lse)
    y, lr = oracle.fwd_perm(inp["x"], inp["v"], perm, m, causal)
    assert_close(to_host(out), y, dtype, "out")
    assert_close(lse.cpu().numpy(), lr, "f32" if dtype == "f32" else "bf16", "lse")


# ------------------------------------------------------------------ whole path, small cases
@pytest.mark.parametrize("dtype,causal,nb,nh,L", [("f32", False, 16, 1, 1024), ("f32", True, 16, 2, 512),
                                                  ("bf16", True, 64, 2, 1024), ("bf16", False, 128, 3, 1152),
                                                  ("bf16", True, 1024, 4, 2048), ("bf16", True, 2, 2, 256),
                                                  ("bf16", True, 256, 3, 1408), ("bf16", True, 64, 2, 960),
                                                  ("bf16", False, 6, 2, 704), ("f32", True, 6, 2, 320)])
def test_forward_backward_small(dtype, causal, nb, nh, L):
    w = small("long_64k", B=2, H=2, L=L, n_buckets=nb, n_hashes=nh, causal=causal, dtype=dtype, backward=True)
    full_check(w)


def test_clustered_inputs_small():
    w = small("image_12k", B=1, H=2, L=1536)
    full_check(w)


@pytest.mark.parametrize("causal", [True, False])
def test_wide_rows_forward_backward(causal):
    """Rows with |x| of 300 to 2000 next to ordinary rows (|x| about 8), so that
    warps of the forward kernel hold both: for such rows the bound tau |x| on
    the scores is loose enough that the softmax first finds the exact row
    maximum.  Outputs and both gradients against the oracle.

    Key-role gradients scale with the query rows' norms: with dY ~ N(0, 1) they
    reach |dx| ~ 66 here, where one bf16 rounding step (0.0625 in [8, 16))
    already exceeds the 2e-2 absolute bound.  dY is therefore scaled by 1/32
    (gradients are linear in dY, and the relative-L2 bound is scale-free)."""
    w = small("long_64k", B=1, H=2, L=2048, n_buckets=64, n_hashes=2, causal=causal, backward=True)
    inp = synth.make_inputs(w)
    inp["dy"] = (inp["dy"] / 32.0).astype(np.float32)           # exact: a power of two
    rng = np.random.default_rng(11)
    x = inp["x"].astype(np.float64)
    wide = rng.random(x.shape[:3]) < 0.4
    target = rng.uniform(300.0, 2000.0, size=x.shape[:3])
    scale = np.where(wide, target / np.linalg.norm(x, axis=-1), 1.0)
    inp["x"] = synth.round_to_bf16((x * scale[..., None]).astype(np.float32))
    norms = np.linalg.norm(inp["x"].astype(np.float64), axis=-1)
    assert (norms > 277).mean() > 0.3 and (norms < 20).mean() > 0.3
    full_check(w, inp=inp)


def test_edge_cases():
    """Zero rows (key 0), duplicated rows, causal first token = its own value."""
    w = small("long_64k", B=1, H=2, L=256, n_buckets=8, n_hashes=2, backward=True)
    inp = synth.make_inputs(w)
    inp["x"][0, 0, 5] = 0.0
    inp["x"][0, 1, 10] = inp["x"][0, 1, 11]
    run = Run(inp, w.n_buckets, w.chunk, True, "bf16")
    out = to_host(run.out)
    np.testing.assert_array_equal(out[0, :, 0], inp["v"][0, :, 0])   # causal position 0 sees only itself
    y, _ = oracle.fwd_perm(inp["x"], inp["v"], run.perm.cpu().numpy(), w.chunk, True)
    assert_close(out, y, "bf16", "out")
    dx, dv = oracle.bwd(inp["x"], inp["v"], inp["dy"], run.perm.cpu().numpy(), w.chunk, True)
    assert_close(to_host(run.dx), dx, "bf16", "dqk")
    assert_close(to_host(run.dv), dv, "bf16", "dv")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_recomputes_permutation_when_not_given(dtype):
    """lsh_attn_bwd with perm = NULL hashes and sorts again from qk and R in its
    own workspace: the gradients match the oracle and the perm-given call."""
    w = small("long_64k", B=1, H=2, L=1024, n_buckets=64, n_hashes=2, causal=True, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    dx = torch.empty_like(run.x); dv = torch.empty_like(run.v)
    wsb = lsh.workspace(run.desc, True, run.x.device)
    lsh.lsh_attn_bwd(run.desc, run.x, run.v, run.R, run.out, run.lse, None, run.dy, dx, dv, wsb)
    assert lsh.lsh_attn_poll(wsb) == 0
    assert_close(to_host(dx), to_host(run.dx), dtype, "dqk recomputed vs given perm")
    assert_close(to_host(dv), to_host(run.dv), dtype, "dv recomputed vs given perm")
    gperm = run.perm.cpu().numpy()
    odx, odv = oracle.bwd(inp["x"], inp["v"], inp["dy"], gperm, w.chunk, w.causal)
    assert_close(to_host(dx), odx, dtype, "dqk recomputed vs oracle")
    assert_close(to_host(dv), odv, dtype, "dv recomputed vs oracle")


@pytest.mark.parametrize("dtype,L", [("bf16", 1024), ("bf16", 960), ("f32", 512)])
def test_permutation_entries_out_of_range_are_reported(dtype, L):
    """A permutation entry outside [0, L) is treated as an empty slot by the
    forward and backward kernels (nothing is read or written at it) and
    lsh_attn_poll reports LSH_ERR_ARG; every other output stays finite and the
    next call with a valid permutation is exact again."""
    nh = 2
    w = small("long_64k", B=1, H=2, L=L, n_buckets=64, n_hashes=nh, causal=True, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(3)
    perm = np.stack([[rng.permutation(L) for _ in range(nh)] for _ in range(2)])[None].astype(np.int32)
    bad = perm.copy()
    lost = {(0, 1, bad[0, 0, 1, 5]), (1, 0, bad[0, 1, 0, 70])}
    bad[0, 0, 1, 5] = L + 3
    bad[0, 1, 0, 70] = -7
    x, v, dy = to_dev(inp["x"], dtype), to_dev(inp["v"], dtype), to_dev(inp["dy"], dtype)
    desc = lsh.desc_for(x, w.n_buckets, nh, w.chunk, w.causal)
    out, lse, _ = lsh.outputs_like(desc, x)
    lse.fill_(0.0)
    out.zero_()
    ws = lsh.workspace(desc, False, x.device)
    lsh.lsh_attn_fwd_sorted(desc, x, v, torch.from_numpy(bad).cuda(), out, lse, ws)
    assert lsh.lsh_attn_poll(ws) == -1                   # LSH_ERR_ARG
    lse_h = lse.cpu().numpy()
    for h, r, pos in lost:
        lse_h[0, h, r, pos] = 0.0                        # never written
    assert np.isfinite(lse_h).all()
    dx = torch.empty_like(x); dvv = torch.empty_like(v)
    wsb = lsh.workspace(desc, True, x.device)
    lsh.lsh_attn_bwd(desc, x, v, None, out, lse, torch.from_numpy(bad).cuda(), dy, dx, dvv, wsb)
    assert lsh.lsh_attn_poll(wsb) == -1
    lsh.lsh_attn_fwd_sorted(desc, x, v, torch.from_numpy(perm).cuda(), out, lse, ws)
    assert lsh.lsh_attn_poll(ws) == 0
    y, lr = oracle.fwd_perm(inp["x"], inp["v"], perm, w.chunk, w.causal)
    assert_close(to_host(out), y, dtype, "out after a bad call")


def test_backward_run_to_run_drift_is_one_rounding_step():
    """The backward adds every round's gradient rows into fp32 accumulators with
    atomic vector reductions, so their summation order is not fixed.  Two runs on
    the same inputs may differ by the fp32 reassociation of those sums (about
    1e-6 here) and by the final rounding to bf16: elementwise at most one bf16
    step (2^-7 of the larger magnitude) plus 2^-16 absolute."""
    w = small("long_64k", B=1, H=2, L=8192, backward=True)
    inp = synth.make_inputs(w)
    a = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    b = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    assert torch.equal(a.perm, b.perm) and torch.equal(a.out, b.out)
    for name, u, t in [("dqk", a.dx, b.dx), ("dv", a.dv, b.dv)]:
        u, t = to_host(u), to_host(t)
        bound = 2.0 ** -7 * np.maximum(np.abs(u), np.abs(t)) + 2.0 ** -16
        assert (np.abs(u - t) <= bound).all(), name
        print(f"[drift] {name}: {(u != t).mean():.2e} of elements differ between two runs, "
              f"largest difference {np.abs(u - t).max():.2e}")


# ------------------------------------------------------------------ optional readings (flags)
@pytest.mark.parametrize("dtype,causal,flags,nb,L", [
    ("bf16", True, lsh.FLAG_BUCKET_MASK, 64, 1024), ("bf16", False, lsh.FLAG_BUCKET_MASK, 64, 1024),
    ("bf16", True, lsh.FLAG_SELF_PENALTY, 64, 1024), ("bf16", False, lsh.FLAG_SELF_PENALTY, 64, 1024),
    ("bf16", False, 3, 256, 960), ("bf16", True, 3, 1024, 2048), ("bf16", True, lsh.FLAG_BUCKET_MASK, 2, 576),
    ("f32", True, lsh.FLAG_BUCKET_MASK, 16, 512), ("f32", False, 3, 16, 512), ("f32", True, lsh.FLAG_SELF_PENALTY, 16, 256),
])
def test_flags_forward_backward(dtype, causal, flags, nb, L):
    """Bucket mask ("LSH Attention", strict N_LSH) and self penalty
    ("Implementation Reading", same-token question): outputs, lse and both
    gradients against the oracle's readings, with the GPU's permutation and
    bucket ids.  Many queries have no same-bucket key in their window, so the
    lone-query paths run often.  With sparse buckets attention concentrates on
    few keys and |dv| reaches 7, where bf16 output rounding alone costs 0.016 of
    the 2e-2 absolute bound; dY is scaled by 1/4 (gradients are linear in it, the
    relative bound is scale-free)."""
    w = small("long_64k", B=1, H=2, L=L, n_buckets=nb, n_hashes=2, causal=causal, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    inp["dy"] = (inp["dy"] / 4.0).astype(np.float32)           # exact: a power of two
    run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype, flags)
    gb = run.host_buckets()
    gperm = run.perm.cpu().numpy()
    check_perm_is_stable_sort(gperm, gb, "flags perm")
    flips = 0
    for h in range(2):
        ref = oracle.fwd(inp["x"][:, h:h + 1], inp["v"][:, h:h + 1], inp["R"], nb, w.chunk, causal)
        flips += check_buckets(gb[0, h], ref["bucket"][0, 0], ref["margin"][0, 0], f"flags ({h})")
    bk = gb if flags & lsh.FLAG_BUCKET_MASK else None
    pen = bool(flags & lsh.FLAG_SELF_PENALTY)
    y, lr = oracle.fwd_perm(inp["x"], inp["v"], gperm, w.chunk, causal, bucket=bk, self_penalty=pen)
    lone = np.isclose(lr, lsh.SELF_PENALTY_SCORE) if pen else np.zeros_like(lr, dtype=bool)
    print(f"[flags {flags}] {int(lone.sum())} penalised lone (row, round) pairs of {lr.size}")
    assert_close(to_host(run.out), y, dtype, "out")
    assert_close(run.lse.cpu().numpy(), lr, "f32" if dtype == "f32" else "bf16", "lse")
    dx, dv = oracle.bwd(inp["x"], inp["v"], inp["dy"], gperm, w.chunk, causal, bucket=bk, self_penalty=pen)
    assert_close(to_host(run.dx), dx, dtype, "dqk")
    assert_close(to_host(run.dv), dv, dtype, "dv")
    _flip_report(f"flags {flags}", flips, 2 * 2 * L)


# ------------------------------------------------------------------ local (non-hashed) chunk attention
@pytest.mark.parametrize("dtype,causal,after,L,chunk,flags", [
    ("bf16", False, 1, 1024, 64, 0), ("bf16", True, 1, 1024, 64, 0), ("bf16", False, 0, 960, 64, 0),
    ("bf16", False, 1, 576, 64, lsh.FLAG_SELF_PENALTY), ("bf16", True, 0, 2048, 64, lsh.FLAG_SELF_PENALTY),
    ("f32", False, 1, 512, 32, 0), ("f32", True, 0, 256, 64, lsh.FLAG_SELF_PENALTY), ("f32", False, 1, 96, 16, 0),
])
def test_local_attention_forward_backward(dtype, causal, after, L, chunk, flags):
    """Local chunk attention ("The Reformer - Pushing the limits of language
    modeling", Approach / What changed): chunk c of the unsorted positions
    attends to chunks c - 1, c and (chunks_after = 1) c + 1.  Output, the
    window's lse and both gradients against the oracle."""
    w = small("long_64k", B=1, H=2, L=L, chunk=chunk, n_hashes=1, causal=causal, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    x, v, dy = to_dev(inp["x"], dtype), to_dev(inp["v"], dtype), to_dev(inp["dy"], dtype)
    desc = lsh.make_desc(1, 2, L, 64, 2, 1, chunk, causal, dtype=torch_dtype(dtype), flags=flags)
    out = torch.empty_like(x)
    lse = torch.empty((1, 2, 1, L), dtype=torch.float32, device="cuda")
    wsf = lsh.local_workspace(desc, after, False, x.device)
    lsh.lsh_attn_local_fwd(desc, after, x, v, out, lse, wsf)
    dx = torch.empty_like(x); dv = torch.empty_like(v)
    wsb = lsh.local_workspace(desc, after, True, x.device)
    lsh.lsh_attn_local_bwd(desc, after, x, v, out, lse, dy, dx, dv, wsb)
    assert lsh.lsh_attn_poll(wsf) == 0 and lsh.lsh_attn_poll(wsb) == 0
    pen = bool(flags & lsh.FLAG_SELF_PENALTY)
    y, lr = oracle.local_fwd(inp["x"], inp["v"], chunk, causal, 1, after, self_penalty=pen)
    assert_close(to_host(out), y, dtype, "local out")
    assert_close(lse.cpu().numpy()[:, :, 0], lr, "f32" if dtype == "f32" else "bf16", "local lse")
    odx, odv = oracle.local_bwd(inp["x"], inp["v"], inp["dy"], chunk, causal, 1, after, self_penalty=pen)
    assert_close(to_host(dx), odx, dtype, "local dqk")
    assert_close(to_host(dv), odv, dtype, "local dv")


# ------------------------------------------------------------------ reversible residual block
@pytest.mark.parametrize("dtype,causal,L", [("bf16", True, 1024), ("bf16", False, 576), ("f32", True, 512)])
def test_reversible_block(dtype, causal, L):
    """Reversible block ("Reformer", Reversible Residual Layers) with LSH
    attention as F and G = tanh(u Wg + bg): outputs against the oracle; the
    backward, run from the GPU's outputs, recovers the inputs (fp32 streams) and
    its input gradients match the oracle's backward from the same outputs."""
    nb, nh = 64, 2
    w = small("long_64k", B=1, H=2, L=L, n_buckets=nb, n_hashes=nh, causal=causal, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(5)
    x1 = inp["v"].astype(np.float32); x2 = inp["x"].astype(np.float32)
    Wg = (rng.standard_normal((64, 64)) / 8).astype(np.float32); bg = (0.1 * rng.standard_normal(64)).astype(np.float32)
    dy1 = inp["dy"].astype(np.float32); dy2 = rng.standard_normal(x1.shape).astype(np.float32)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()

    R = to_dev(inp["R"], dtype)
    desc = lsh.make_desc(1, 2, L, 64, nb, nh, 64, causal, torch_dtype(dtype))
    X1, X2, W, Bg = dev(x1), dev(x2), dev(Wg), dev(bg)
    Y1 = torch.empty_like(X1); Y2 = torch.empty_like(X1)
    wsf = lsh.rev_workspace(desc, False, X1.device)
    lsh.lsh_rev_fwd(desc, X1, X2, R, W, Bg, Y1, Y2, wsf)
    rnd = synth.round_to_bf16 if dtype == "bf16" else None
    y1, y2, _ = oracle.rev_fwd(x1, x2, inp["R"], Wg, bg, nb, 64, causal, round_to=rnd)
    assert_close(to_host(Y1), y1, dtype, "y1")
    assert_close(to_host(Y2), y2, dtype, "y2")
    R1, R2, DX1, DX2 = (torch.empty_like(X1) for _ in range(4))
    wsb = lsh.rev_workspace(desc, True, X1.device)
    lsh.lsh_rev_bwd(desc, Y1, Y2, dev(dy1), dev(dy2), R, W, Bg, R1, R2, DX1, DX2, wsb)
    assert lsh.lsh_attn_poll(wsf) == 0 and lsh.lsh_attn_poll(wsb) == 0
    np.testing.assert_allclose(to_host(R2), x2, rtol=0, atol=2e-6)      # fp32 rounding of the residual adds
    np.testing.assert_allclose(to_host(R1), x1, rtol=0, atol=2e-6)
    _, _, odx1, odx2 = oracle.rev_bwd(to_host(Y1), to_host(Y2), dy1, dy2, inp["R"], Wg, bg, nb, 64, causal,
                                      round_to=rnd)
    assert_close(to_host(DX1), odx1, dtype, "dx1")
    assert_close(to_host(DX2), odx2, dtype, "dx2")


# ------------------------------------------------------------------ host-buffer pipeline
@pytest.mark.parametrize("dtype,heads_per_chunk,bwd", [("bf16", 1, True), ("bf16", 3, True), ("bf16", 0, False),
                                                       ("f32", 2, True)])
def test_host_pipeline_matches_device_calls(dtype, heads_per_chunk, bwd):
    """lsh_attn_step_host (host buffers, chunks of heads through two device slots
    on three streams) gives what lsh_attn_fwd + lsh_attn_bwd give on device
    buffers: the forward bit for bit (same kernels, same inputs), the gradients
    within the bf16 bound (their fp32 sums are reassociated), and the oracle's
    values."""
    w = small("long_64k", B=2, H=3, L=1024, n_buckets=64, n_hashes=2, dtype=dtype, backward=True)
    inp = synth.make_inputs(w)
    run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    tdt = torch_dtype(dtype)
    host = {k: torch.from_numpy(inp[k]).to(tdt).pin_memory() for k in ("x", "v", "R", "dy")}
    out_h = torch.empty_like(host["x"]).pin_memory()
    lse_h = torch.empty(tuple(run.lse.shape), dtype=torch.float32).pin_memory()
    dqk_h = torch.empty_like(host["x"]).pin_memory(); dv_h = torch.empty_like(host["x"]).pin_memory()
    streams = [torch.cuda.Stream() for _ in range(3)]
    scratch = lsh.step_host_scratch(run.desc, heads_per_chunk, bwd, run.x.device)
    lsh.lsh_attn_step_host(run.desc, host["x"], host["v"], host["R"], host["dy"] if bwd else None, out_h, lse_h,
                           dqk_h if bwd else None, dv_h if bwd else None, scratch, streams, heads_per_chunk)
    streams[0].synchronize()
    assert lsh.lsh_attn_poll(scratch) == 0
    assert torch.equal(out_h, run.out.cpu()) and torch.equal(lse_h, run.lse.cpu())
    if bwd:
        assert_close(to_host(dqk_h), to_host(run.dx), dtype, "dqk host vs device")
        assert_close(to_host(dv_h), to_host(run.dv), dtype, "dv host vs device")
        gperm = run.perm.cpu().numpy()
        dx, dv = oracle.bwd(inp["x"], inp["v"], inp["dy"], gperm, w.chunk, w.causal)
        assert_close(to_host(dqk_h), dx, dtype, "dqk host vs oracle")
        assert_close(to_host(dv_h), dv, dtype, "dv host vs oracle")


# ------------------------------------------------------------------ the five workloads
def test_workload_tiny_f32():
    full_check(synth.WORKLOADS["tiny_f32"])


def test_workload_bf16_causal_4k():
    full_check(synth.WORKLOADS["bf16_causal_4k"], heads=[(0, 0), (3, 5), (7, 7)])


def test_workload_long_64k_one_head():
    full_check(synth.WORKLOADS["long_64k"], heads=[(0, 3)])


def test_workload_image_12k_two_heads():
    full_check(synth.WORKLOADS["image_12k"], heads=[(0, 0), (5, 6)])


def test_workload_half_million_sampled():
    """L = 524288: every permutation is checked against numpy's stable argsort
    of the GPU buckets; bucket ids and outputs on sampled rows and slots."""
    w = synth.WORKLOADS["half_million"]
    inp = synth.make_inputs(w)
    run = Run(inp, w.n_buckets, w.chunk, w.causal, w.dtype)
    gb = run.host_buckets()
    gperm = run.perm.cpu().numpy()
    check_perm_is_stable_sort(gperm, gb, "half_million perm")
    rng = np.random.default_rng(5)
    out = to_host(run.out)
    lse = run.lse.cpu().numpy().astype(np.float64)
    flips = 0
    for h in range(w.H):
        rows = np.sort(rng.choice(w.L, size=1024, replace=False))
        for r in range(w.n_hashes):
            ob, mg = oracle.hash_round(inp["x"][0, h, rows], inp["R"][r], w.n_buckets)
            flips += check_buckets(gb[0, h, r, rows], ob, mg, f"half_million h={h} r={r}")
        # merged output at sampled positions: every round's slot of that position
        pos = rows[:256]
        o_r, l_r = [], []
        for r in range(w.n_hashes):
            inv = np.empty(w.L, np.int64); inv[gperm[0, h, r]] = np.arange(w.L)
            o, l = oracle.attn_slots(inp["x"][0, h], inp["v"][0, h], gperm[0, h, r], w.chunk, w.causal, inv[pos])
            o_r.append(o); l_r.append(l)
            assert_close(lse[0, h, r, pos], l, "bf16", f"half_million lse h={h} r={r}")
        o_r, l_r = np.stack(o_r), np.stack(l_r)
        wts = np.exp(l_r - l_r.max(0)); wts /= wts.sum(0)
        y = (wts[:, :, None] * o_r).sum(0)
        assert_close(out[0, h, pos], y, "bf16", f"half_million out h={h}")
    _flip_report("half_million sampled", flips, w.H * w.n_hashes * 1024)


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_reports_timeout():
    """A device wait that nothing completes gives up after its budget and the
    status word reports it; the context stays usable."""
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    assert lsh.lsh_attn_poll(ws) == 0
    lsh.lsh_attn_selftest_timeout(ws, 2_000_000)          # about a millisecond
    assert lsh.lsh_attn_poll(ws) == -6                     # LSH_ERR_TIMEOUT
    assert lsh.lsh_attn_poll(ws) == 0                      # cleared by the poll
    w = small("long_64k", B=1, H=1, L=256, backward=False)
    run = Run(synth.make_inputs(w), w.n_buckets, w.chunk, w.causal, w.dtype)
    assert torch.isfinite(run.out.float()).all()


# ------------------------------------------------------------------ near-tie bookkeeping
_NEAR_TIE_SCRIPT = r"""
import json, sys
import numpy as np, torch
sys.path.insert(0, {root!r})
import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import build, synth
import os
trace = build.LIB.replace(".so", "_trace.so")
lsh.load_library(trace if os.path.exists(trace) else build.build(phase_trace=True))
w = synth.WORKLOADS["bf16_causal_4k"].replace(B=1, H=2, L=1024, n_buckets=64, n_hashes=2)
inp = synth.make_inputs(w)
inp["x"][0, 0, :5] = 0.0
inp["x"][0, 1, 100:105] = 0.0
x = torch.from_numpy(inp["x"]).cuda().to(torch.bfloat16)
R = torch.from_numpy(inp["R"]).cuda().to(torch.bfloat16)
desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, w.causal)
bk = torch.empty((1, 2, 2, w.L), dtype=torch.int16, device="cuda")
lsh.lsh_attn_hash(desc, x, R, bk)
print(json.dumps({{"count": lsh.load_library().lsh_attn_last_near_ties()}}))
"""


def test_near_tie_count_in_tuning_build():
    """The tuning build counts (row, round) pairs whose top-two gap is below
    1e-6: every zero row is an exact tie in each round; the other rows count
    only if the oracle also sees them within a small relative gap."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _NEAR_TIE_SCRIPT.format(root=root)], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    count = json.loads(r.stdout.strip().splitlines()[-1])["count"]
    w = synth.WORKLOADS["bf16_causal_4k"].replace(B=1, H=2, L=1024, n_buckets=64, n_hashes=2)
    inp = synth.make_inputs(w)
    inp["x"][0, 0, :5] = 0.0
    inp["x"][0, 1, 100:105] = 0.0
    close = 0
    for h in range(2):
        for rr in range(2):
            _, mg = oracle.hash_round(inp["x"][0, h], inp["R"][rr], w.n_buckets)
            close += int((mg < 1e-4).sum())
    assert 20 <= count <= close, (count, close)
    assert lsh.load_library().lsh_attn_last_near_ties() == -1     # the regular build does not count


def test_trace_records_only_selected_stages():
    """With a stage mask the trace puts events around the selected stages alone
    (the bench times its dominant kernel this way); the results are unchanged."""
    w = small("bf16_causal_4k", B=1, H=2, L=1024, n_buckets=64, n_hashes=2)
    inp = synth.make_inputs(w)
    x = to_dev(inp["x"], "bf16"); v = to_dev(inp["v"], "bf16"); R = to_dev(inp["R"], "bf16")
    desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, w.causal)
    out, lse, perm = lsh.outputs_like(desc, x)
    ws = lsh.workspace(desc, False, x.device)
    lsh.fused_forward(0)                         # the staged kernels, one stage each
    try:
        lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm, ws)
        ref = out.clone()
        try:
            lsh.trace_stages(["attn_fwd"])
            lsh.trace_begin(16)
            lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm, ws)
            st = lsh.trace_end()
        finally:
            lsh.trace_stages(None)
        assert st["attn_fwd"][1] == 1 and st["attn_fwd"][0] > 0
        assert all(st[k][1] == 0 for k in st if k != "attn_fwd")
        assert torch.equal(out, ref)
        lsh.trace_begin(16)
        lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm, ws)
        st = lsh.trace_end()
        assert st["hash"][1] == 1 and st["sort"][1] == 1 and st["combine"][1] == 1
    finally:
        lsh.fused_forward(1)
    # the single kernel (wherever it fits: this shape has 4 segments): one stage of its own, same output
    try:
        lsh.fused_forward(2)
        lsh.trace_begin(16)
        lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm, ws)
        st = lsh.trace_end()
    finally:
        lsh.fused_forward(1)
    assert st["fused_fwd"][1] == 1 and all(st[k][1] == 0 for k in st if k != "fused_fwd")
    assert torch.equal(out, ref)
