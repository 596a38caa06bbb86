"""Pins of the oracle's low-rank-plus-diagonal quadratic (the conditioning-study workload)
against what the mathematics fixes: the dense Hessian, exact per-probe curvature on a
dyadic grid, and the estimator's mean by exhaustive enumeration."""
import itertools

import numpy as np

import oracle
from oracle import core


def _dense_H(D, lam, V):
    M = D.size
    return np.diag(D.astype(np.float64)) + sum(l / M * np.outer(v, v) for l, v in zip(lam, V))


def test_loss_equals_half_theta_H_theta():
    r = np.random.default_rng(0)
    M = 40
    D = (10 ** r.uniform(-3, 3, M)).astype(np.float32)
    th = r.standard_normal(M).astype(np.float32)
    lam = [500.0, 20.0, 3.0]
    V = oracle.lowrank.directions(7, 3, M)
    H = _dense_H(D, lam, V)
    t = th.astype(np.float64)
    assert np.isclose(oracle.lowrank.loss(th, D, lam, V), 0.5 * t @ H @ t, rtol=1e-12)
    # rank 0 is the diagonal quadratic
    assert oracle.lowrank.loss(th, D, [], oracle.lowrank.directions(7, 0, M)) == core.quad_loss(th, D)


def test_directions_are_the_generators_probes():
    M = 1000
    V = oracle.lowrank.directions(11, 4, M)
    for k in range(4):
        assert np.array_equal(V[k], core.probe_signs(11, 0, k, M).astype(np.float64))
        assert V[k] @ V[k] == M
    G = V @ V.T
    assert np.abs(G - np.diag(np.diag(G))).max() < 5 * np.sqrt(M)  # nearly orthogonal


def test_curvature_per_probe_is_exact_on_a_dyadic_grid():
    """(L+ + L- - 2 L0) / eps^2 = z^T H z = tr(D) + sum_k lam_k (v_k . z)^2 / M exactly when
    every quantity is a short dyadic number (M = 64, eps = 2^-6)."""
    r = np.random.default_rng(1)
    M, eps = 64, 2.0 ** -6
    D = (2.0 ** r.integers(-3, 4, M)).astype(np.float32)
    th = (r.integers(-64, 65, M) / 64.0).astype(np.float32)
    lam = [64.0, 16.0]
    V = oracle.lowrank.directions(3, 2, M)
    L0 = oracle.lowrank.loss(th, D, lam, V)
    seen = set()
    for i in range(12):
        z = core.probe_signs(5, 0, i, M).astype(np.float64)
        Lp = oracle.lowrank.loss(core.perturb(th, 5, 0, i, +1, eps), D, lam, V)
        Lm = oracle.lowrank.loss(core.perturb(th, 5, 0, i, -1, eps), D, lam, V)
        c = (Lp + Lm - 2 * L0) / eps ** 2
        expect = float(D.astype(np.float64).sum()) + sum(l * (v @ z) ** 2 / M for l, v in zip(lam, V))
        assert c == expect
        g = (Lp - Lm) / (2 * eps)
        assert g == z @ _dense_H(D, lam, V) @ th.astype(np.float64)
        seen.add(c)
    assert len(seen) > 3  # the curvature differs across probes (it cannot on the diagonal)


def test_estimator_mean_is_H_theta_by_enumeration():
    """Over all 2^M sign vectors, the mean of g(z) z with g from the oracle's central loss
    difference equals H theta (E[z z^T] = I; the difference is exact for a quadratic on a
    dyadic grid)."""
    r = np.random.default_rng(2)
    M, eps = 8, 2.0 ** -5  # lam_k / M dyadic too
    D = (2.0 ** r.integers(-2, 3, M)).astype(np.float32)
    th = (r.integers(-32, 33, M) / 32.0).astype(np.float32)
    lam = [32.0, 4.0]
    V = oracle.lowrank.directions(9, 2, M)
    acc = np.zeros(M)
    for bits in itertools.product((1.0, -1.0), repeat=M):
        z = np.array(bits, np.float32)
        Lp = oracle.lowrank.loss(th + np.float32(eps) * z, D, lam, V)
        Lm = oracle.lowrank.loss(th - np.float32(eps) * z, D, lam, V)
        acc += (Lp - Lm) / (2 * eps) * z
    H = _dense_H(D, lam, V)
    assert np.allclose(acc / 2 ** M, H @ th.astype(np.float64), rtol=1e-12, atol=1e-12)
