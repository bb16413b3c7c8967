"""Pins of the oracle's reversible residual block ("Reformer" paper note,
section "Reversible Residual Layers": y1 = x1 + F(x2), y2 = x2 + G(y1) and its
inverse), checked against the inverse itself, central finite differences of the
whole block, and G's closed-form derivative."""
import numpy as np
import pytest

from oracle import oracle


def _setup(seed, L=16, d=8, nb=4, nh=2):
    rng = np.random.default_rng(seed)
    x1 = rng.standard_normal((1, 1, L, d)); x2 = rng.standard_normal((1, 1, L, d))
    R = rng.standard_normal((nh, d, nb // 2))
    Wg = rng.standard_normal((d, d)) / np.sqrt(d); bg = rng.standard_normal(d) * 0.1
    return x1, x2, R, Wg, bg, nb


@pytest.mark.parametrize("causal", [False, True])
def test_inverse_recovers_the_inputs(causal):
    x1, x2, R, Wg, bg, nb = _setup(1 + causal)
    y1, y2, _ = oracle.rev_fwd(x1, x2, R, Wg, bg, nb, 4, causal)
    r1, r2, _, _ = oracle.rev_bwd(y1, y2, np.zeros_like(y1), np.zeros_like(y2), R, Wg, bg, nb, 4, causal)
    np.testing.assert_allclose(r2, x2, atol=1e-13)
    np.testing.assert_allclose(r1, x1, atol=1e-13)


def test_g_derivative_closed_form():
    """d tanh(u W + b)/du against central differences."""
    rng = np.random.default_rng(3)
    d = 6
    u = rng.standard_normal(d); W = rng.standard_normal((d, d)); b = rng.standard_normal(d)
    G = rng.standard_normal(d)
    g = oracle.rev_g(u, W, b)
    grad = (G * (1 - g * g)) @ W.T
    h = 1e-6
    num = np.array([(oracle.rev_g(u + h * e, W, b) @ G - oracle.rev_g(u - h * e, W, b) @ G) / (2 * h)
                    for e in np.eye(d)])
    np.testing.assert_allclose(grad, num, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_block_gradient_matches_central_differences(causal):
    """Gradient of sum(y1 * D1 + y2 * D2) w.r.t. x1 and x2, with F's permutation
    held fixed (the hash is piecewise constant), against central differences."""
    x1, x2, R, Wg, bg, nb = _setup(7 + causal)
    rng = np.random.default_rng(11)
    D1 = rng.standard_normal(x1.shape); D2 = rng.standard_normal(x2.shape)
    y1, y2, perm = oracle.rev_fwd(x1, x2, R, Wg, bg, nb, 4, causal)
    _, _, dx1, dx2 = oracle.rev_bwd(y1, y2, D1, D2, R, Wg, bg, nb, 4, causal)

    def loss(a1, a2):
        f, _ = oracle.fwd_perm(a2, a2, perm, 4, causal)
        b1 = a1 + f
        b2 = a2 + oracle.rev_g(b1, Wg, bg)
        return float((b1 * D1).sum() + (b2 * D2).sum())

    h = 1e-6
    for which, grad in [(0, dx1), (1, dx2)]:
        num = np.zeros_like(x1)
        for idx in np.ndindex(x1.shape):
            a = [x1.copy(), x2.copy()]; b = [x1.copy(), x2.copy()]
            a[which][idx] += h; b[which][idx] -= h
            num[idx] = (loss(*a) - loss(*b)) / (2 * h)
        np.testing.assert_allclose(grad, num, atol=3e-8)
