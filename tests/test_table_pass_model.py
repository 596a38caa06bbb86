"""A numpy model of the table-based loss pass (zero_order_forward_b200/csrc/zo_loss.cu):
per 4-element vector the 16 sums (x_0 + x_1) + (x_2 + x_3), x_q in {t_a, t_b}, and per probe
the entry its 4 sign bits select, summed over the vectors; L- = T - L+ from the common sum
T = sum (t_a + t_b).  For the diagonal quadratic's terms and for the low-rank quadratic's dot
product terms, the model equals the oracle's direct per-probe evaluation to fp64 rounding,
so the restructuring itself computes the method's losses."""
import numpy as np

import oracle
import synth
from oracle import core


def _tables(ta, tb):
    """[vectors][16] entry n: element q of the vector takes tb if bit q of n is set."""
    ta = ta.reshape(-1, 4)
    tb = tb.reshape(-1, 4)
    tab = np.empty((ta.shape[0], 16))
    for n in range(16):
        x = [tb[:, q] if (n >> q) & 1 else ta[:, q] for q in range(4)]
        tab[:, n] = (x[0] + x[1]) + (x[2] + x[3])
    return tab


def _model_losses(ta, tb, bits):
    """bits [n][M] (1 where z = -1): (L+[n], L-[n]) by table lookups."""
    M = ta.size
    pad = (-M) % 4  # elements past the end contribute nothing
    ta = np.concatenate([ta, np.zeros(pad)])
    tb = np.concatenate([tb, np.zeros(pad)])
    bits = np.concatenate([bits, np.zeros((bits.shape[0], pad), np.int64)], axis=1)
    tab = _tables(ta, tb)
    nib = (bits.reshape(bits.shape[0], -1, 4) << np.arange(4)).sum(axis=2)  # [n][vectors]
    Lp = np.array([np.sum(tab[np.arange(tab.shape[0]), nib[i]]) for i in range(bits.shape[0])])
    T = np.sum(ta + tb)
    return Lp, T - Lp


def test_diagonal_terms_model_equals_direct_losses():
    M, n, seed, step, eps = 2 * 2048 + 37, 12, 5, 2, np.float32(1e-3)
    th, D = synth.quad_problem(M, seed=7)
    Pa = (th + eps).astype(np.float32).astype(np.float64)
    Pb = (th - eps).astype(np.float32).astype(np.float64)
    hd = 0.5 * D.astype(np.float64)
    ta, tb = hd * Pa * Pa, hd * Pb * Pb
    bits = np.stack([(core.probe_signs(seed, step, i, M) < 0).astype(np.int64) for i in range(n)])
    Lp, Lm = _model_losses(ta, tb, bits)
    for i in range(n):
        rp = core.quad_loss(core.perturb(th, seed, step, i, +1, float(eps)), D)
        rm = core.quad_loss(core.perturb(th, seed, step, i, -1, float(eps)), D)
        assert abs(Lp[i] - rp) <= 1e-12 * rp and abs(Lm[i] - rm) <= 1e-12 * rm


def test_dot_product_terms_model_equals_direct_dots():
    M, n, seed, step, eps = 2048 + 9, 6, 3, 1, np.float32(1e-3)
    th, D, lam, vseed = synth.lowrank_problem(M, seed=4, rank=2)
    V = oracle.lowrank.directions(vseed, 2, M)
    Pa = (th + eps).astype(np.float32).astype(np.float64)
    Pb = (th - eps).astype(np.float32).astype(np.float64)
    bits = np.stack([(core.probe_signs(seed, step, i, M) < 0).astype(np.int64) for i in range(n)])
    for k in range(2):
        dp, dm = _model_losses(V[k] * Pa, V[k] * Pb, bits)
        for i in range(n):
            Pp = core.perturb(th, seed, step, i, +1, float(eps)).astype(np.float64)
            Pm = core.perturb(th, seed, step, i, -1, float(eps)).astype(np.float64)
            scale = np.sum(np.abs(Pp))  # the dots cancel: compare on the scale of the terms
            assert abs(dp[i] - V[k] @ Pp) <= 1e-13 * scale
            assert abs(dm[i] - V[k] @ Pm) <= 1e-13 * scale
