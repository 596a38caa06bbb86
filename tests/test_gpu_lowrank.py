"""The conditioning-study quadratic on the GPU against the oracle: the loss (clean,
perturbed, both signs from one pass; ragged tails), and full 1SPSA / 1.5-SPSA steps.
Every sum is fp64 on both sides, in different orders: 1e-11 relative on losses."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import core

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,rank", [(4096 * 3 + 77, 4), (50001, 1), (1 << 16, 3), (5, 2)])
def test_lowrank_loss_matches_oracle(zo, M, rank):
    th_np, D_np, lam, vseed = synth.lowrank_problem(M, seed=M, rank=rank)
    V = oracle.lowrank.directions(vseed, rank, M)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=9)
    out = torch.zeros(5, dtype=torch.float64, device="cuda")
    zo.zo_lowrank_loss(ctx, D, lam, vseed, out[0:1])
    zo.zo_perturb(ctx, -1, 1e-3, 6)
    zo.zo_lowrank_loss(ctx, D, lam, vseed, out[1:2])
    zo.zo_restore(ctx)
    zo.zo_perturb(ctx, +1, 1e-3, 6)
    zo.zo_lowrank_loss(ctx, D, lam, vseed, out[2:3])
    zo.zo_restore(ctx)
    zo.zo_lowrank_loss_pair(ctx, D, lam, vseed, 6, 1e-3, out[3:4], out[4:5])
    assert zo.zo_sync(ctx) == 0
    got = out.cpu().numpy()
    e32 = float(np.float32(1e-3))
    ref0 = oracle.lowrank.loss(th_np, D_np, lam, V)
    refm = oracle.lowrank.loss(core.perturb(th_np, 9, 0, 6, -1, e32), D_np, lam, V)
    refp = oracle.lowrank.loss(core.perturb(th_np, 9, 0, 6, +1, e32), D_np, lam, V)
    assert np.allclose(got[:3], [ref0, refm, refp], rtol=1e-11, atol=0)
    assert got[3] == got[2] and got[4] == got[1]  # one pass per pair, same order as single
    ctx.close()


@pytest.mark.parametrize("preconditioned", [True, False])
def test_lowrank_full_step_matches_oracle(zo, preconditioned):
    M, n, eps, lr, lam_d = 1 << 15, 16, 1e-3, 2e-4, 1e-3
    th_np, D_np, lam, vseed = synth.lowrank_problem(M, seed=2)
    V = oracle.lowrank.directions(vseed, len(lam), M)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=4)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_lowrank_step(ctx, D, lam, vseed, n, eps, lr, lam_d, preconditioned, losses)
    assert zo.zo_sync(ctx) == 0
    loss = lambda P: oracle.lowrank.loss(P, D_np, lam, V)  # noqa: E731
    nxt, rec = oracle.step.spsa_step(th_np, loss, n, eps, lr, lam_d, 4, 0,
                                     preconditioned=preconditioned, update="mirror")
    L = losses.cpu().numpy()
    if preconditioned:
        assert abs(L[0] - rec["L0"]) <= 1e-11 * rec["L0"]
    assert np.allclose(L[1:n + 1], rec["Lp"], rtol=1e-11, atol=0)
    assert np.allclose(L[n + 1:], rec["Lm"], rtol=1e-11, atol=0)
    # the GPU's coefficients through the oracle's fixed-order update: bit-exact
    g, c, w, a = zo.zo_get_precond(ctx, n)
    mirror = core.update_mirror(th_np, a, 4, 0)
    assert (th.cpu().numpy().view(np.uint32) == mirror.view(np.uint32)).all()
    # and those coefficients against the oracle's from its own losses (1e-11 relative on
    # losses; the curvature's cancellation (L+ + L- - 2 L0) magnifies it by L / (c eps^2))
    if preconditioned:
        rel = 1e-11 * np.abs(rec["Lp"]).max() / (np.abs(rec["c"]) * (2 * eps) ** 2 / 4) * 8
        assert np.allclose(c, rec["c"], rtol=max(rel.max(), 1e-9))
        assert len(np.unique(np.round(c, 3))) > 1  # curvature differs across probes here
    assert zo.zo_get_step(ctx) == 1
    ctx.close()


def test_lowrank_rejects_bad_rank(zo):
    th = torch.zeros(64, device="cuda")
    D = torch.ones(64, device="cuda")
    ctx = zo.zo_create(th)
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    with pytest.raises(ValueError):
        zo.zo_lowrank_loss(ctx, D, [], 1, out)
    with pytest.raises(ValueError):
        zo.zo_lowrank_loss(ctx, D, [1.0] * 5, 1, out)
    ctx.close()


@pytest.mark.parametrize("M,rank,n", [((1 << 20) + 17, 4, 64), (50001, 1, 20), (4096 * 3 + 77, 3, 5),
                                      (1 << 16, 2, 70)])
def test_lowrank_step_losses_equal_one_probe_passes(zo, M, rank, n):
    """zo_lowrank_step's losses (one table pass for the diagonal part and one per direction for
    the dot products, per 64 probes) equal the one-probe low-rank passes to fp64 rounding, with
    the clean loss, for 1..4 directions and every pass size."""
    th_np, D_np, lam, vseed = synth.lowrank_problem(M, seed=M + n, rank=rank)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=12)
    zo.zo_set_step(ctx, 3)
    ref = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_lowrank_loss(ctx, D, lam, vseed, ref[0:1])
    for i in range(n):
        zo.zo_lowrank_loss_pair(ctx, D, lam, vseed, i, 1e-3, ref[1 + i:2 + i],
                                ref[1 + n + i:2 + n + i])
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_lowrank_step(ctx, D, lam, vseed, n, 1e-3, 0.0, 1e-3, True, losses)  # lr 0: theta kept
    assert zo.zo_sync(ctx) == 0
    got, want = losses.cpu().numpy(), ref.cpu().numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=0), np.abs(got / want - 1).max()
    assert np.array_equal(th.cpu().numpy(), th_np)  # lr = 0 leaves theta unchanged
    ctx.close()
