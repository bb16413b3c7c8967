"""Pins of the oracle's two optional readings, against things it does not
compute itself (numpy dense attention, a hand-derived example, a brute-force
candidate enumeration, central finite differences).

* Bucket mask: the strict candidate set of "Reformer" (paper note), section
  "LSH Attention", N_LSH(i) = {j : h(q_i) = h(k_j)}, applied inside the
  chunk window of "Sorting and Chunking".
* Self penalty: the other answer to the same-token question of section
  "Implementation Reading": the query's own position is always a candidate
  with the fixed score -1e5, so it carries weight only when nothing else is
  left (and a round where that happens is weighted out of the merge when
  another round has real candidates).
"""
import math

import numpy as np
import pytest

from oracle import oracle

PENALTY = -1.0e5


def _rng(seed):
    return np.random.default_rng(seed)


def numpy_buckets(x, R, nb):
    """argmax over [xR; -xR] (numpy, first index on ties)."""
    p = x @ R
    return np.argmax(np.concatenate([p, -p], axis=-1), axis=-1)


def dense_same_bucket(x, v, b, causal, penalty):
    """Dense shared-QK attention (unit keys) restricted to same-bucket keys;
    the query's own position: removed unless nothing is left (penalty False)
    or always present with score PENALTY (penalty True)."""
    L, d = x.shape
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    s = (x @ k.T) / math.sqrt(d)
    allowed = (b[:, None] == b[None, :]) & ~np.eye(L, dtype=bool)
    if causal:
        allowed &= np.tril(np.ones((L, L), dtype=bool))
    if penalty:
        s[np.arange(L), np.arange(L)] = PENALTY
        allowed[np.arange(L), np.arange(L)] = True
    else:
        empty = ~allowed.any(axis=1)
        allowed[empty, empty.nonzero()[0]] = True
    s = np.where(allowed, s, -np.inf)
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    return (e / e.sum(axis=1, keepdims=True)) @ v, mx[:, 0] + np.log(e.sum(axis=1))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("penalty", [False, True])
@pytest.mark.parametrize("nb", [2, 6, 16])
def test_bucket_mask_one_chunk_equals_dense_restricted_to_the_bucket(causal, penalty, nb):
    """n_hashes = 1, one chunk spanning L: with the bucket mask, LSH attention is
    dense attention over the keys that share the query's bucket."""
    rng = _rng(nb * 4 + 2 * causal + penalty)
    L, d = 40, 8
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((1, d, nb // 2))
    out = oracle.fwd(x, v, R, nb, chunk=L, causal=causal, bucket_mask=True, self_penalty=penalty)
    b = numpy_buckets(x[0, 0], R[0], nb)
    np.testing.assert_array_equal(out["bucket"][0, 0, 0], b)
    yd, lsed = dense_same_bucket(x[0, 0], v[0, 0], b, causal, penalty)
    np.testing.assert_allclose(out["y"][0, 0], yd, rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["lse"][0, 0, 0], lsed, rtol=0, atol=1e-9)


def test_self_penalty_worked_example_by_hand():
    """Three tokens, d = 2, one chunk, causal, self penalty; by hand:
    x0 = (2,0), x1 = (0,3), x2 = (1,0); keys k0 = (1,0), k1 = (0,1), k2 = (1,0);
    tau = 1/sqrt(2).  Query 0 has no earlier key: its own entry (score -1e5) is
    the only candidate, so y0 = v0 and lse0 = -1e5.  Query 1 sees key 0 (score
    0) and itself (-1e5, weight exp(-1e5) = 0 in double): y1 = v0, lse1 = 0.
    Query 2 sees keys 0 (score tau) and 1 (score 0): y2 = (e^tau v0 + v1) / (e^tau + 1)."""
    x = np.array([[2.0, 0.0], [0.0, 3.0], [1.0, 0.0]])
    v = np.array([[1.0, 0.0], [0.0, 1.0], [5.0, 7.0]])
    R = np.array([[[1.0], [0.0]]])
    perm = np.arange(3, dtype=np.int32)[None, None, None]
    y, lse = oracle.fwd_perm(x[None, None], v[None, None], perm, 3, True, self_penalty=True)
    t = 1 / math.sqrt(2)
    e = math.exp(t)
    np.testing.assert_array_equal(y[0, 0, 0], v[0])
    np.testing.assert_array_equal(y[0, 0, 1], v[0])
    np.testing.assert_allclose(y[0, 0, 2], (e * v[0] + v[1]) / (e + 1), atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], [PENALTY, 0.0, math.log(e + 1)], atol=1e-14)
    # the exact-set reading differs only where the query is alone: lse0 = tau |x0| = 2 tau
    y2, lse2 = oracle.fwd_perm(x[None, None], v[None, None], perm, 3, True)
    np.testing.assert_allclose(lse2[0, 0, 0], [2 * t, 0.0, math.log(e + 1)], atol=1e-14)
    np.testing.assert_allclose(y2[0, 0], y[0, 0], atol=1e-14)
    del R


def test_self_penalty_round_is_weighted_out_of_the_merge():
    """Two rounds, position 0 causal: in both it is alone, so both rounds give
    v0 with lse -1e5 and the merge keeps v0.  A later position that is alone in
    one round only takes its output from the other round (weight exp(-1e5 - lse)
    = 0), while the exact-set reading mixes in v_i with weight softmax(tau|x_i|, lse)."""
    rng = _rng(21)
    L, d, m = 8, 4, 2
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    # round 0: identity order; round 1: chunk 0 holds positions 5 and 6, so 5 has no
    # earlier key there, and chunk 1 holds 0 and 1 (window {5, 6, 0, 1}: 0 is alone too)
    p0 = np.arange(L)
    p1 = np.array([5, 6, 0, 1, 2, 3, 4, 7])
    perm = np.stack([p0, p1]).astype(np.int32)[None, None]
    y, lse = oracle.fwd_perm(x, v, perm, m, True, self_penalty=True)
    # both rounds alone: weights 1/2 each, computed next to lse = -1e5 (1e-11 relative)
    np.testing.assert_allclose(y[0, 0, 0], v[0, 0, 0], rtol=1e-10, atol=0)
    assert lse[0, 0, 1, 5] == PENALTY
    o0, l0 = oracle.attn_round(x[0, 0], v[0, 0], p0, m, True, self_penalty=True)
    np.testing.assert_allclose(y[0, 0, 5], o0[5], atol=1e-14)
    ye, lsee = oracle.fwd_perm(x, v, perm, m, True)
    w = 1.0 / (1.0 + math.exp(lsee[0, 0, 0, 5] - lsee[0, 0, 1, 5]))      # weight of round 1 (alone)
    np.testing.assert_allclose(ye[0, 0, 5], (1 - w) * o0[5] + w * v[0, 0, 5], atol=1e-12)


def brute_force(x, v, buckets, m, causal, mask, penalty):
    """Candidates from (bucket, position) ranks without chunk buffers, for both
    readings: j (!= i) is a candidate of i iff chunk(j) in {chunk(i),
    chunk(i) - 1}, (not causal or j <= i) and (not mask or b_j == b_i); the
    query itself: score PENALTY, always present (penalty), else present with
    its own score only when nothing else is.  Rounds merged by softmax of lse."""
    nh, L = buckets.shape
    d = x.shape[1]
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    lses, outs = [[] for _ in range(L)], [[] for _ in range(L)]
    for r in range(nh):
        b = buckets[r]
        rank = np.array([sum(1 for j in range(L) if (b[j], j) < (b[i], i)) for i in range(L)])
        ch = rank // m
        for i in range(L):
            c = [j for j in range(L) if j != i and ch[j] in (ch[i], ch[i] - 1) and (not causal or j <= i)
                 and (not mask or b[j] == b[i])]
            z = [x[i] @ k[j] / math.sqrt(d) for j in c]
            if penalty:
                c.append(i); z.append(PENALTY)
            elif not c:
                c.append(i); z.append(x[i] @ k[i] / math.sqrt(d))
            z = np.array(z)
            lse = np.log(np.exp(z - z.max()).sum()) + z.max()
            lses[i].append(lse)
            outs[i].append((np.exp(z - lse)[:, None] * v[c]).sum(0))
    y = np.zeros((L, d))
    for i in range(L):
        lse = np.array(lses[i]); w = np.exp(lse - lse.max()); w /= w.sum()
        y[i] = (w[:, None] * np.array(outs[i])).sum(0)
    return y


@pytest.mark.parametrize("mask,penalty", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,m,nb,nh", [(24, 4, 4, 2), (40, 8, 8, 3), (9, 1, 4, 2)])
def test_chunked_equals_brute_force_with_flags(mask, penalty, causal, L, m, nb, nh):
    rng = _rng(L * 11 + m + 3 * causal + 5 * mask + 7 * penalty)
    d = 6
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    out = oracle.fwd(x, v, R, nb, m, causal, bucket_mask=mask, self_penalty=penalty)
    y = brute_force(x[0, 0], v[0, 0], out["bucket"][0, 0], m, causal, mask, penalty)
    np.testing.assert_allclose(out["y"][0, 0], y, atol=1e-12)


@pytest.mark.parametrize("mask,penalty", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_with_flags_matches_central_differences(mask, penalty, causal):
    """Gradient of sum(y * G) w.r.t. x and v against central differences with the
    permutations and bucket ids held fixed."""
    rng = _rng(31 + 2 * causal + 4 * mask + 8 * penalty)
    B, H, L, d, nb, nh, m = 1, 1, 16, 8, 4, 2, 4
    x = rng.standard_normal((B, H, L, d)); v = rng.standard_normal((B, H, L, d))
    G = rng.standard_normal((B, H, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    f = oracle.fwd(x, v, R, nb, m, causal, bucket_mask=mask, self_penalty=penalty)
    perm, bk = f["perm"], (f["bucket"] if mask else None)
    dx, dv = oracle.bwd(x, v, G, perm, m, causal, bucket=bk, self_penalty=penalty)

    def loss(xx, vv):
        y, _ = oracle.fwd_perm(xx, vv, perm, m, causal, bucket=bk, self_penalty=penalty)
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


def test_flags_off_match_the_default_reading():
    """bucket=None and self_penalty=False are the default reading exactly."""
    rng = _rng(41)
    x = rng.standard_normal((1, 2, 32, 8)); v = rng.standard_normal((1, 2, 32, 8))
    R = rng.standard_normal((2, 8, 4))
    a = oracle.fwd(x, v, R, 8, 8, True)
    b = oracle.fwd(x, v, R, 8, 8, True, bucket_mask=False, self_penalty=False)
    np.testing.assert_array_equal(a["y"], b["y"])
