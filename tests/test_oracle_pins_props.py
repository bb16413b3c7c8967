"""Exact properties of the method that pin the CPU oracle at sizes beyond the
brute-force and finite-difference pins (several rounds, several chunks).

Each property follows from the definitions in the paper note "Reformer"
(eightmm.github.io), not from the oracle's own code:

* "LSH Attention", hash equation h(x) = argmax [xR ; -xR]: the bucket depends
  only on the direction of x (a positive scale multiplies every projection by
  the same factor), and negating x exchanges the two halves of [xR ; -xR].
* "LSH Attention", output equation, and "Multiple Hash Rounds": the output is
  a convex combination of value rows whose weights depend on x alone, so it is
  linear in v, and the weights of every query sum to one over all rounds and
  candidates; hence sum_j dL/dv_j = sum_i dL/dy_i.
* "Shared Query-Key Space" (unit keys): scaling every x by c leaves the keys'
  directions unchanged and multiplies every score by c, so the derivative of
  the loss along x itself is the scaled-score derivative.
"""
import numpy as np
import pytest

from oracle import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _case(seed, B=2, H=2, L=256, d=16, nb=16, nh=3):
    rng = _rng(seed)
    x = rng.standard_normal((B, H, L, d))
    v = rng.standard_normal((B, H, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    return rng, x, v, R, nb


# ---------------------------------------------------------------- hash geometry
@pytest.mark.parametrize("c", [4.0, 0.25])
def test_hash_depends_on_direction_only(c):
    """bucket(c x) = bucket(x) for c > 0.  A power of two scales every product
    and every partial sum exactly, so even exact ties stay where they are."""
    rng = _rng(21)
    x = rng.standard_normal((700, 24)); R = rng.standard_normal((24, 32))
    x[:5] = 0.0                                    # all-zero rows: the tie rule
    b, _ = oracle.hash_round(x, R, 64)
    bc, _ = oracle.hash_round(c * x, R, 64)
    np.testing.assert_array_equal(bc, b)


@pytest.mark.parametrize("nb", [2, 8, 64])
def test_hash_negation_swaps_halves(nb):
    """[(-x)R ; -(-x)R] is [xR ; -xR] with its halves exchanged, so without an
    exact tie bucket(-x) = (bucket(x) + nb/2) mod nb."""
    rng = _rng(22 + nb)
    x = rng.standard_normal((600, 16)); R = rng.standard_normal((16, nb // 2))
    b, mg = oracle.hash_round(x, R, nb)
    bn, _ = oracle.hash_round(-x, R, nb)
    assert (mg > 0).all()
    np.testing.assert_array_equal(bn, (b + nb // 2) % nb)


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("causal", [False, True])
def test_output_is_linear_in_values(causal):
    """The weights depend on x alone, so y(a v1 + b v2) = a y(v1) + b y(v2);
    the lse does not depend on v at all."""
    rng, x, v1, R, nb = _case(31 + causal)
    v2 = rng.standard_normal(v1.shape)
    a, b = 0.75, -1.5
    o1 = oracle.fwd(x, v1, R, nb, 32, causal)
    o2 = oracle.fwd(x, v2, R, nb, 32, causal)
    o12 = oracle.fwd(x, a * v1 + b * v2, R, nb, 32, causal)
    np.testing.assert_allclose(o12["y"], a * o1["y"] + b * o2["y"], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(o12["lse"], o1["lse"])
    np.testing.assert_array_equal(o12["perm"], o1["perm"])


@pytest.mark.parametrize("causal", [False, True])
def test_heads_are_independent(causal):
    """Each (batch, head) slice is its own problem: the batched forward equals
    the forward of every slice alone, bit for bit."""
    _, x, v, R, nb = _case(41 + causal)
    full = oracle.fwd(x, v, R, nb, 32, causal)
    for bb in range(x.shape[0]):
        for h in range(x.shape[1]):
            one = oracle.fwd(x[bb:bb + 1, h:h + 1], v[bb:bb + 1, h:h + 1], R, nb, 32, causal)
            for k in ("y", "lse", "perm", "bucket"):
                np.testing.assert_array_equal(full[k][bb, h], one[k][0, 0])


def test_combine_closed_forms():
    """Round merge, weights softmax_r(lse_r): equal lse gives the mean of the
    rounds; lse differing by ln 2 gives weights 2/3 and 1/3; the merged lse is
    log(sum_r exp(lse_r))."""
    rng = _rng(51)
    o = rng.standard_normal((2, 10, 8))
    lse = np.full((2, 10), 3.5)
    y, big = oracle.combine(o, lse)
    np.testing.assert_allclose(y, o.mean(axis=0), rtol=0, atol=1e-14)
    np.testing.assert_allclose(big, 3.5 + np.log(2.0), rtol=0, atol=1e-14)
    lse2 = np.stack([np.full(10, 1.0 + np.log(2.0)), np.full(10, 1.0)])
    y2, big2 = oracle.combine(o, lse2)
    np.testing.assert_allclose(y2, (2.0 * o[0] + o[1]) / 3.0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(big2, 1.0 + np.log(3.0), rtol=0, atol=1e-14)


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("causal,flags", [(False, {}), (True, {}), (True, {"self_penalty": True}),
                                          (False, {"bucket_mask": True})])
def test_value_gradient_sums_to_output_gradient(causal, flags):
    """dL/dv_j = sum_i P_ij dL/dy_i with sum_j P_ij = 1 over all rounds and
    candidates (a query with no other candidate keeps itself, weight 1), so the
    rows of dv sum to the rows of dy, per (batch, head)."""
    rng, x, v, R, nb = _case(61 + causal + 2 * len(flags))
    dy = rng.standard_normal(x.shape)
    fw = oracle.fwd(x, v, R, nb, 32, causal, **flags)
    bucket = fw["bucket"] if flags.get("bucket_mask") else None
    _, dv = oracle.bwd(x, v, dy, fw["perm"], 32, causal, bucket=bucket,
                       self_penalty=flags.get("self_penalty", False))
    np.testing.assert_allclose(dv.sum(axis=2), dy.sum(axis=2), rtol=0, atol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_along_x_matches_score_scaling(causal):
    """L(c) = sum(y(c x) * G): keys are unit vectors, so every score scales by
    c and the buckets do not change; dL/dc at c = 1 equals sum(dx * x)."""
    rng, x, v, R, nb = _case(71 + causal, B=1, H=2, L=192)
    G = rng.standard_normal(x.shape)
    perm = oracle.fwd(x, v, R, nb, 32, causal)["perm"]
    dx, _ = oracle.bwd(x, v, G, perm, 32, causal)
    h = 1e-5
    lp = float((oracle.fwd(x * (1 + h), v, R, nb, 32, causal)["y"] * G).sum())
    lm = float((oracle.fwd(x * (1 - h), v, R, nb, 32, causal)["y"] * G).sum())
    for c in (1 + h, 1 - h):                       # the scaled inputs hash the same
        np.testing.assert_array_equal(oracle.fwd(x * c, v, R, nb, 32, causal)["perm"], perm)
    num = (lp - lm) / (2 * h)
    ana = float((dx * x).sum())
    assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (num, ana)
