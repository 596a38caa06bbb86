"""Loss of the low-rank-plus-diagonal quadratic, the workload of the conditioning study.

TEST INFRASTRUCTURE (see oracle/__init__.py).  On the diagonal quadratic every Rademacher
probe sees the same curvature, z^T D z = tr(D), so 1.5-SPSA's per-probe weights are all
equal there.  The preconditioner of "Stanford's 1.5-SPSA Trains OPT-30B Without
Backpropagation" (section "Probe-Space Preconditioning") exists for losses whose curvature
differs from direction to direction; this workload adds r <= 8 stiff rank-one terms:

  L(theta) = 1/2 sum_j D_j theta_j^2 + 1/2 sum_k (lam_k / M) (v_k . theta)^2,

so H = diag(D) + sum_k (lam_k / M) v_k v_k^T and z^T H z = tr(D) + sum_k lam_k (v_k . z)^2 / M
varies from probe to probe.  The directions v_k in {-1, +1}^M are the probe generator's
probes k = 0 .. r-1 at step 0 under their own seed `vseed` (each has norm^2 = M, so lam_k is
the eigenvalue that v_k adds).  Everything in fp64.
"""
import numpy as np

from . import core


def directions(vseed, rank, M):
    """V [rank][M] as float64 +/-1 (probes 0..rank-1 of step 0 under vseed)."""
    if not 0 <= rank <= 8:
        raise ValueError("rank must be in 0..8")
    return np.stack([core.probe_signs(vseed, 0, k, M).astype(np.float64) for k in range(rank)]) \
        if rank else np.zeros((0, M))


def loss(P, D, lam, V):
    """1/2 sum_j D_j P_j^2 + 1/2 sum_k (lam_k / M) (V_k . P)^2 for float32 P and D."""
    P = np.asarray(P, np.float32)
    M = P.size
    diag = core.quad_loss(P, D)
    Pd = P.astype(np.float64)
    dots = V @ Pd
    return diag + 0.5 * float(np.sum(np.asarray(lam, np.float64) / M * dots * dots))
