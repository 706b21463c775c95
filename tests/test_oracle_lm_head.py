"""Pins for the lm_head cross-entropy oracle: a scalar brute-force loop, the zero-weight closed form,
finite differences of the summed loss, and the zero row sums of D."""
import math

import numpy as np

from oracle import lm_head as lh


def _data(M=4, V=9, K=6, seed=0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((V, K)), rng.standard_normal((M, K)), rng.integers(0, V, M)


def test_brute_force_loop():
    W, X, lab = _data()
    lab[2] = -100                                             # ignored token
    loss, dX, D = lh.lm_head_ce(W, X, lab, grad_scale=0.5, mirror=False)
    V, K = W.shape
    for t in range(X.shape[0]):
        z = [sum(X[t, k] * W[v, k] for k in range(K)) for v in range(V)]
        if lab[t] < 0:
            assert loss[t] == 0 and np.all(dX[t] == 0)
            continue
        s = sum(math.exp(zi) for zi in z)
        assert math.isclose(loss[t], math.log(s) - z[lab[t]], rel_tol=1e-12)
        d = [0.5 * (math.exp(zi) / s - (1.0 if v == lab[t] else 0.0)) for v, zi in enumerate(z)]
        for k in range(K):
            assert math.isclose(dX[t, k], sum(d[v] * W[v, k] for v in range(V)), rel_tol=1e-10, abs_tol=1e-14)


def test_zero_weights_give_log_v():
    W, X, lab = _data(V=37)
    loss, dX, _ = lh.lm_head_ce(np.zeros_like(W), X, lab)
    assert np.allclose(loss, math.log(37), rtol=1e-15)
    assert np.all(dX == 0)


def test_finite_differences_and_row_sums():
    W, X, lab = _data(M=3, V=11, K=5, seed=3)
    loss, dX, D = lh.lm_head_ce(W, X, lab, grad_scale=1.0, mirror=False)
    assert np.allclose(D.sum(axis=1), 0.0, atol=1e-14)
    h = 1e-6
    for t in range(3):
        for k in range(5):
            Xp, Xm = X.copy(), X.copy()
            Xp[t, k] += h
            Xm[t, k] -= h
            fd = (lh.lm_head_ce(W, Xp, lab, mirror=False)[0].sum() - lh.lm_head_ce(W, Xm, lab, mirror=False)[0].sum()) / (2 * h)
            assert abs(fd - dX[t, k]) <= 1e-7 * max(1.0, abs(dX[t, k]))
