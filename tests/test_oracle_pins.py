"""Pins that tie the CPU oracle to the method and to mathematics, not to itself.

Each test checks the oracle against something it does not compute itself:
textbook dense attention, a hand-derived worked example, library routines
(numpy argmax / stable argsort), invariants, a brute-force candidate
enumeration and central finite differences.  Page references are to the
paper note "Reformer" (eightmm.github.io) by section.
"""
import math

import numpy as np
import pytest

from oracle import oracle
from lsh_attention_02_b200 import synth


def _rng(seed):
    return np.random.default_rng(seed)


def dense_shared_qk(x, v, causal):
    """Textbook softmax attention with Q = K (keys unit-normalised), self masked
    unless it is the only candidate, optional causal mask; numpy, float64.
    ("LSH Attention": dense formula A = Q K^T / sqrt(d_k); "Shared Query-Key Space")"""
    L, d = x.shape
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    s = (x @ k.T) / math.sqrt(d)
    allowed = ~np.eye(L, dtype=bool)
    if causal:
        allowed &= np.tril(np.ones((L, L), dtype=bool))
    empty = ~allowed.any(axis=1)
    allowed[empty, empty.nonzero()[0]] = True
    s = np.where(allowed, s, -np.inf)
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    lse = (mx[:, 0] + np.log(e.sum(axis=1)))
    return (e / e.sum(axis=1, keepdims=True)) @ v, lse


# ---------------------------------------------------------------- P1
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_buckets", [2, 8, 32])
def test_one_chunk_equals_dense(causal, n_buckets):
    """n_hashes = 1 and one chunk spanning L: LSH attention is dense attention."""
    rng = _rng(1 + n_buckets + causal)
    L, d = 48, 16
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((1, d, n_buckets // 2))
    out = oracle.fwd(x, v, R, n_buckets, chunk=L, causal=causal)
    yd, lsed = dense_shared_qk(x[0, 0], v[0, 0], causal)
    np.testing.assert_allclose(out["y"][0, 0], yd, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"][0, 0, 0], lsed, rtol=0, atol=1e-12)


def test_worked_example_by_hand():
    """Three tokens, d = 2, one chunk, non-causal; values derived by hand.

    x0 = (2,0), x1 = (0,3), x2 = (1,0)  ->  keys k0 = (1,0), k1 = (0,1), k2 = (1,0),
    tau = 1/sqrt(2).  Query 0 sees {1, 2}: scores 0 and 2 tau;
    query 1 sees {0, 2}: scores 0 and 0; query 2 sees {0, 1}: scores tau and 0.
    """
    x = np.array([[2.0, 0.0], [0.0, 3.0], [1.0, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0], [5.0, 7.0]])
    R = np.array([[[1.0], [0.0]]])  # any rotation: one chunk covers every slot
    out = oracle.fwd(x[None, None], v[None, None], R, 2, chunk=3, causal=False)
    t = 1 / math.sqrt(2)
    e = math.exp(2 * t)
    y0 = (v[1] + e * v[2]) / (1 + e)
    y1 = (v[0] + v[2]) / 2
    e2 = math.exp(t)
    y2 = (e2 * v[0] + v[1]) / (1 + e2)
    np.testing.assert_allclose(out["y"][0, 0], np.stack([y0, y1, y2]), atol=1e-14)
    np.testing.assert_allclose(out["lse"][0, 0, 0],
                               [math.log(1 + e), math.log(2), math.log(1 + e2)], atol=1e-14)


# ---------------------------------------------------------------- P2
@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(causal):
    """softmax weights sum to 1 per row and per round, round weights sum to 1:
    with constant values every output equals that constant."""
    rng = _rng(7)
    B, H, L, d, nb, nh, m = 1, 2, 96, 8, 8, 3, 16
    x = rng.standard_normal((B, H, L, d))
    v = np.full((B, H, L, d), 0.75)
    R = rng.standard_normal((nh, d, nb // 2))
    out = oracle.fwd(x, v, R, nb, m, causal)
    np.testing.assert_allclose(out["y"], 0.75, atol=1e-13)


# ---------------------------------------------------------------- P3
def test_hash_matches_numpy_argmax():
    """bucket = argmax over [xR; -xR], first index on ties (numpy.argmax)."""
    rng = _rng(3)
    x = rng.standard_normal((500, 16)); R = rng.standard_normal((16, 12))
    b, mg = oracle.hash_round(x, R, 24)
    u = np.concatenate([x @ R, -(x @ R)], axis=1)
    np.testing.assert_array_equal(b, np.argmax(u, axis=1))
    us = np.sort(u, axis=1)
    np.testing.assert_allclose(mg, (us[:, -1] - us[:, -2]) / np.abs(us[:, -1]), rtol=1e-12)


def test_hash_exact_tie_takes_lowest_index():
    """A zero row ties every entry of [xR; -xR]: bucket 0."""
    b, _ = oracle.hash_round(np.zeros((2, 4)), _rng(0).standard_normal((4, 3)), 6)
    np.testing.assert_array_equal(b, [0, 0])


def test_sort_is_stable_argsort():
    """perm = stable argsort of bucket ids (positions increase inside a bucket)."""
    rng = _rng(4)
    for L, nb in [(1, 2), (17, 4), (1000, 16), (4096, 1024)]:
        bucket = rng.integers(0, nb, size=L).astype(np.int32)
        perm = oracle.sort_segment(bucket)
        np.testing.assert_array_equal(perm, np.argsort(bucket, kind="stable"))


# ---------------------------------------------------------------- P4
@pytest.mark.parametrize("causal", [False, True])
def test_identical_rounds_reproduce_single_round(causal):
    rng = _rng(11)
    B, H, L, d, nb, m = 2, 1, 128, 16, 16, 32
    x = rng.standard_normal((B, H, L, d)); v = rng.standard_normal((B, H, L, d))
    R1 = rng.standard_normal((1, d, nb // 2))
    one = oracle.fwd(x, v, R1, nb, m, causal)
    three = oracle.fwd(x, v, np.repeat(R1, 3, axis=0), nb, m, causal)
    np.testing.assert_allclose(three["y"], one["y"], atol=1e-13)
    for r in range(3):
        np.testing.assert_allclose(three["lse"][:, :, r], one["lse"][:, :, 0], atol=1e-13)
        np.testing.assert_array_equal(three["perm"][:, :, r], one["perm"][:, :, 0])


# ---------------------------------------------------------------- P5
@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_differences(causal):
    """Gradient of sum(y * G) w.r.t. x and v against central differences,
    permutations held fixed (the hash is piecewise constant)."""
    rng = _rng(5 + causal)
    B, H, L, d, nb, nh, m = 1, 1, 16, 8, 4, 2, 4
    x = rng.standard_normal((B, H, L, d)); v = rng.standard_normal((B, H, L, d))
    G = rng.standard_normal((B, H, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    perm = oracle.fwd(x, v, R, nb, m, causal)["perm"]
    dx, dv = oracle.bwd(x, v, G, perm, m, causal)

    def loss(xx, vv):
        y, _ = oracle.fwd_perm(xx, vv, perm, m, causal)
        return float((y * G).sum())

    h = 1e-6
    for arr, grad, is_x in [(x, dx, True), (v, dv, False)]:
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = arr.copy(); a[idx] += h
            b = arr.copy(); b[idx] -= h
            lp = loss(a, v) if is_x else loss(x, a)
            lm = loss(b, v) if is_x else loss(x, b)
            num[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=0, atol=2e-8)


def test_self_only_row_gradient():
    """Causal position 0 only sees itself: y0 = v0, so dy0 flows only into dv0."""
    rng = _rng(9)
    L, d, m = 8, 4, 4
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    G = np.zeros((1, 1, L, d)); G[0, 0, 0] = rng.standard_normal(d)
    perm = oracle.fwd(x, v, rng.standard_normal((1, d, 2)), 4, m, True)["perm"]
    dx, dv = oracle.bwd(x, v, G, perm, m, True)
    np.testing.assert_allclose(dv[0, 0, 0], G[0, 0, 0], atol=1e-14)
    np.testing.assert_allclose(dv[0, 0, 1:], 0, atol=1e-14)
    np.testing.assert_allclose(dx, 0, atol=1e-14)


# ---------------------------------------------------------------- P6
def brute_force(x, v, buckets, m, causal):
    """Candidates enumerated from (bucket, position) ranks, no chunk buffers:
    rank(i) = #{j : (b_j, j) < (b_i, i)}, chunk(i) = rank(i) // m; j is a candidate
    of i iff chunk(j) in {chunk(i), chunk(i) - 1}, j != i and (not causal or j <= i);
    self alone if that set is empty.  Rounds merged by softmax over lse."""
    nh, L = buckets.shape
    d = x.shape[1]
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    zs, vs = [[] for _ in range(L)], [[] for _ in range(L)]
    for r in range(nh):
        b = buckets[r]
        rank = np.array([sum(1 for j in range(L) if (b[j], j) < (b[i], i)) for i in range(L)])
        ch = rank // m
        for i in range(L):
            c = [j for j in range(L) if j != i and ch[j] in (ch[i], ch[i] - 1) and (not causal or j <= i)]
            if not c:
                c = [i]
            z = np.array([x[i] @ k[j] / math.sqrt(d) for j in c])
            lse = np.log(np.exp(z - z.max()).sum()) + z.max()
            o = (np.exp(z - lse)[:, None] * v[c]).sum(0)
            zs[i].append(lse); vs[i].append(o)
    y = np.zeros((L, d))
    for i in range(L):
        lse = np.array(zs[i]); w = np.exp(lse - lse.max()); w /= w.sum()
        y[i] = (w[:, None] * np.array(vs[i])).sum(0)
    return y


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,m,nb,nh", [(24, 4, 4, 2), (40, 8, 8, 3), (12, 12, 4, 1), (9, 1, 4, 2)])
def test_chunked_equals_brute_force(causal, L, m, nb, nh):
    rng = _rng(L * 7 + m + causal)
    d = 6
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    out = oracle.fwd(x, v, R, nb, m, causal)
    y = brute_force(x[0, 0], v[0, 0], out["bucket"][0, 0], m, causal)
    np.testing.assert_allclose(out["y"][0, 0], y, atol=1e-12)


# ---------------------------------------------------------------- P7
def test_two_buckets_is_sign_hash_and_causal_first_token():
    rng = _rng(12)
    B, H, L, d, m = 2, 2, 64, 8, 8
    x = rng.standard_normal((B, H, L, d)); v = rng.standard_normal((B, H, L, d))
    R = rng.standard_normal((2, d, 1))
    out = oracle.fwd(x, v, R, 2, m, True)
    for r in range(2):
        sign0 = (x @ R[r])[..., 0] >= 0
        np.testing.assert_array_equal(out["bucket"][:, :, r] == 0, sign0)
    np.testing.assert_allclose(out["y"][:, :, 0], v[:, :, 0], atol=1e-14)


# ---------------------------------------------------------------- P8
def test_near_tie_margin_reported():
    """A row built to sit almost on the boundary of two buckets has a margin < 1e-6."""
    R = np.array([[1.0, 0.0], [0.0, 1.0]])
    x = np.array([[1.0, 1.0 - 1e-9], [1.0, 0.5]])
    b, mg = oracle.hash_round(x, R, 4)
    assert b[0] == 0 and mg[0] < 1e-6
    assert b[1] == 0 and abs(mg[1] - 0.5) < 1e-12


def test_zero_norm_key_contributes_zero_score():
    """|x_j| = 0 gives k_j = 0: score 0 for every query that sees j (reading of the
    normalisation step at the origin); the row of x_j itself attends with scores 0."""
    L, d = 4, 2
    x = np.array([[1.0, 0.0], [0.0, 0.0], [0.0, 2.0], [1.0, 1.0]])
    v = np.arange(L * d, dtype=float).reshape(L, d)
    out = oracle.fwd(x[None, None], v[None, None], np.ones((1, d, 1)), 2, chunk=L, causal=False)
    # query 1 (zero row): all scores 0 -> mean of the others
    np.testing.assert_allclose(out["y"][0, 0, 1], v[[0, 2, 3]].mean(0), atol=1e-14)
    # query 0 = (1,0): key 1 is 0, key 2 = (0,1), key 3 = (1,1)/sqrt(2):
    # scores 0, 0 and (1/sqrt(2)) * (1/sqrt(2)) = 1/2
    w = np.array([1.0, 1.0, math.exp(0.5)])
    np.testing.assert_allclose(out["y"][0, 0, 0], (w[:, None] * v[[1, 2, 3]]).sum(0) / w.sum(), atol=1e-14)


# ---------------------------------------------------------------- inputs
def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0e-3], dtype=np.float32)
    out = synth.round_to_bf16(vals)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    assert out[0] == 1.0 and out[1] == 1.0
    # 1 + 1.5 * 2^-8 rounds up to 1 + 2^-7
    assert out[2] == np.float32(1.0078125)
    assert out[3] == -2.5
    assert (synth.bf16_bits(out).astype(np.uint32) << 16).view(np.float32)[4] == out[4]


def test_philox_known_answer():
    """Philox4x32-10 with zero counter and key: the published known-answer output."""
    r = synth.philox4x32_10([0], [0], [0], [0], 0, 0)
    assert [int(a[0]) for a in r] == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]


def test_normals_moments():
    z = synth.normal(1234, 0, 200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
