"""Pins of the oracle's local (non-hashed) chunk attention: positions in their
own order, chunk c attends to chunks c - before .. c + after ("The Reformer -
Pushing the limits of language modeling", section "Approach / What changed":
local self-attention over chunks with a preceding and a following overlap),
with the keys, self rule and causal mask of the LSH path ("Reformer" paper
note, "Shared Query-Key Space" and "Implementation Reading").

Checked against numpy dense attention, a brute-force window enumeration,
central finite differences and the LSH path with the identity permutation.
"""
import math

import numpy as np
import pytest

from oracle import oracle

from tests.test_oracle_pins import dense_shared_qk


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("causal", [False, True])
def test_window_spanning_everything_is_dense(causal):
    """before = after = number of chunks: every chunk sees every other, so local
    attention is dense shared-QK attention with the self rule."""
    rng = _rng(3 + causal)
    L, d, m = 48, 8, 8
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    y, lse = oracle.local_fwd(x, v, m, causal, before=L // m, after=L // m)
    yd, lsed = dense_shared_qk(x[0, 0], v[0, 0], causal)
    np.testing.assert_allclose(y[0, 0], yd, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lsed, atol=1e-12)


def brute_force_local(x, v, m, before, after, causal):
    """j (!= i) is a candidate of i iff chunk(i) - before <= chunk(j) <= chunk(i) + after
    and (not causal or j <= i); i itself only when nothing else is."""
    L, d = x.shape
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    y = np.zeros((L, d)); lse = np.zeros(L)
    for i in range(L):
        c = [j for j in range(L) if j != i and -before <= j // m - i // m <= after and (not causal or j <= i)]
        if not c:
            c = [i]
        z = np.array([x[i] @ k[j] / math.sqrt(d) for j in c])
        lse[i] = np.log(np.exp(z - z.max()).sum()) + z.max()
        y[i] = (np.exp(z - lse[i])[:, None] * v[c]).sum(0)
    return y, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,m,before,after", [(32, 4, 1, 1), (30, 6, 1, 0), (24, 4, 2, 1), (9, 1, 1, 1), (16, 16, 1, 1)])
def test_local_equals_brute_force(causal, L, m, before, after):
    rng = _rng(L + m + 10 * before + 100 * after + causal)
    d = 6
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    y, lse = oracle.local_fwd(x, v, m, causal, before=before, after=after)
    yb, lb = brute_force_local(x[0, 0], v[0, 0], m, before, after, causal)
    np.testing.assert_allclose(y[0, 0], yb, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], lb, atol=1e-12)


def test_causal_window_ignores_the_following_chunk():
    """With the causal mask every key of a following chunk is in the future, so
    after = 1 and after = 0 agree exactly."""
    rng = _rng(8)
    x = rng.standard_normal((1, 2, 64, 8)); v = rng.standard_normal((1, 2, 64, 8))
    a = oracle.local_fwd(x, v, 8, True, before=1, after=1)
    b = oracle.local_fwd(x, v, 8, True, before=1, after=0)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_preceding_window_is_lsh_attention_with_identity_order():
    """before = 1, after = 0 is the LSH window on sorted slots; with the identity
    permutation and one round the two oracle paths must agree."""
    rng = _rng(9)
    B, H, L, d, m = 1, 2, 40, 8, 8
    x = rng.standard_normal((B, H, L, d)); v = rng.standard_normal((B, H, L, d))
    ident = np.broadcast_to(np.arange(L, dtype=np.int32), (B, H, 1, L)).copy()
    for causal in (False, True):
        y, lse = oracle.local_fwd(x, v, m, causal, before=1, after=0)
        y2, lse2 = oracle.fwd_perm(x, v, ident, m, causal)
        np.testing.assert_allclose(y, y2, atol=1e-13)
        np.testing.assert_allclose(lse, lse2[:, :, 0], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("penalty", [False, True])
def test_local_backward_matches_central_differences(causal, penalty):
    rng = _rng(50 + causal + 2 * penalty)
    L, d, m = 16, 6, 4
    x = rng.standard_normal((1, 1, L, d)); v = rng.standard_normal((1, 1, L, d))
    G = rng.standard_normal((1, 1, L, d))
    dx, dv = oracle.local_bwd(x, v, G, m, causal, 1, 1, self_penalty=penalty)

    def loss(xx, vv):
        y, _ = oracle.local_fwd(xx, vv, m, causal, 1, 1, self_penalty=penalty)
        return float((y * G).sum())

    h = 1e-6
    for arr, grad, is_x in [(x, dx, True), (v, dv, False)]:
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = arr.copy(); a[idx] += h
            b = arr.copy(); b[idx] -= h
            num[idx] = ((loss(a, v) if is_x else loss(x, a)) - (loss(b, v) if is_x else loss(x, b))) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=0, atol=2e-8)


def test_window_of_three_is_the_merge_of_two_disjoint_windows():
    """The split the kernels use: chunks {c-1, c} (the LSH window, identity order)
    and chunk {c+1} alone (the previous chunk of the reversed order) are disjoint,
    so merging them by their logsumexps is the three-chunk window exactly.  The
    second part is built here by brute force in numpy."""
    rng = _rng(13)
    L, d, m = 32, 8, 4
    x = rng.standard_normal((L, d)); v = rng.standard_normal((L, d))
    y3, l3 = oracle.local_fwd(x[None, None], v[None, None], m, False, 1, 1)
    ya, la = oracle.local_fwd(x[None, None], v[None, None], m, False, 1, 0)
    k = x / np.linalg.norm(x, axis=1, keepdims=True)
    yb = np.zeros((L, d)); lb = np.full(L, -np.inf)
    for i in range(L):
        c = [j for j in range(L) if j // m == i // m + 1]
        if c:
            z = np.array([x[i] @ k[j] / math.sqrt(d) for j in c])
            lb[i] = np.log(np.exp(z - z.max()).sum()) + z.max()
            yb[i] = (np.exp(z - lb[i])[:, None] * v[c]).sum(0)
    big = np.logaddexp(la[0, 0], lb)
    y = np.exp(la[0, 0] - big)[:, None] * ya[0, 0] + np.exp(lb - big)[:, None] * yb
    np.testing.assert_allclose(y3[0, 0], y, atol=1e-12)
    np.testing.assert_allclose(l3[0, 0], big, atol=1e-12)
