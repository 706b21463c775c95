"""Pins for the RMSNorm oracle: a hand-computed row, scale invariance, unit mean square, and the
backward against central finite differences."""
import numpy as np

from oracle import rmsnorm as rn


def test_hand_row():
    # x = (3, 4): mean square 12.5, r = 1/sqrt(12.5 + 0.5) = 1/sqrt(13); g = (2, -1)
    Xn, r = rn.rmsnorm_fwd(np.array([[3.0, 4.0]]), np.array([2.0, -1.0]), 0.5, mirror=False)
    assert np.isclose(r[0], 1 / np.sqrt(13.0), rtol=1e-15)
    assert np.allclose(Xn[0], [6 / np.sqrt(13.0), -4 / np.sqrt(13.0)], rtol=1e-15)


def test_scale_invariance_and_unit_mean_square():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((5, 64))
    g = np.ones(64)
    a, _ = rn.rmsnorm_fwd(X, g, 0.0, mirror=False)
    b, _ = rn.rmsnorm_fwd(7.5 * X, g, 0.0, mirror=False)
    assert np.allclose(a, b, rtol=1e-13)
    assert np.allclose(np.mean(a * a, axis=1), 1.0, rtol=1e-13)


def test_backward_finite_differences():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((3, 40))
    g = rng.standard_normal(40)
    d = rng.standard_normal((3, 40))
    eps = 1e-3
    _, r = rn.rmsnorm_fwd(X, g, eps, mirror=False)
    dX = rn.rmsnorm_bwd(X, g, r, d)
    h = 1e-6
    for _ in range(12):
        i, j = rng.integers(0, 3), rng.integers(0, 40)
        Xp, Xm = X.copy(), X.copy()
        Xp[i, j] += h
        Xm[i, j] -= h
        fp = np.sum(d * rn.rmsnorm_fwd(Xp, g, eps, mirror=False)[0])
        fm = np.sum(d * rn.rmsnorm_fwd(Xm, g, eps, mirror=False)[0])
        assert abs((fp - fm) / (2 * h) - dX[i, j]) <= 1e-7 * max(1.0, abs(dX[i, j]))
