"""zo_mlp_losses: every loss of one MLP step from one staged-parameter launch (plus its batch
sum) equals, bit for bit, the perturb / zo_mlp_loss / restore evaluation of the same probe,
sign and step; the clean loss equals zo_mlp_loss at theta.  The batch is cut into slices of
8 samples per block, so ragged batches and shapes are covered."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _per_probe(zo, ctx, X, y, batch, n_in, n_hidden, n_out, n, eps, scale):
    zo.zo_set_live_buffer(ctx, True)
    out = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_mlp_loss(ctx, X, y, batch, n_in, n_hidden, n_out, scale, out[0:1])
    for i in range(n):
        for s, off in ((+1, 1), (-1, 1 + n)):
            zo.zo_perturb(ctx, s, eps, i)
            zo.zo_mlp_loss(ctx, X, y, batch, n_in, n_hidden, n_out, scale, out[off + i:off + i + 1])
            zo.zo_restore(ctx)
    return out.cpu().numpy()


@pytest.mark.parametrize("batch,n_in,n_hidden,n_out,n,step", [
    (64, 64, 256, 10, 16, 0),     # the MLP workload's shape
    (13, 64, 256, 10, 3, 5),      # a batch that is not a multiple of the slice
    (1, 17, 33, 5, 1, 2),         # small odd shape (M not a multiple of 16)
    (70, 100, 300, 7, 9, 11),     # hidden units beyond one block of threads
])
def test_batched_mlp_losses_equal_per_probe_losses(zo, batch, n_in, n_hidden, n_out, n, step):
    M = synth.mlp_param_count(n_in, n_hidden, n_out)
    P = synth.mlp_params(3, n_in=n_in, n_hidden=n_hidden, n_out=n_out)
    teacher = synth.mlp_params(4, tag="teacher", n_in=n_in, n_hidden=n_hidden, n_out=n_out)
    X_np, y_np = synth.mlp_batch(7, step, teacher, n_in=n_in, n_hidden=n_hidden, n_out=n_out,
                                 batch=batch)
    X, y = torch.from_numpy(X_np).cuda(), torch.from_numpy(y_np).cuda()
    th = torch.from_numpy(P).cuda()
    ctx = zo.zo_create(th, seed=21)
    zo.zo_set_step(ctx, step)
    eps, scale = 1e-3, 1.0 / batch
    lp = torch.full((n,), -5.0, dtype=torch.float64, device="cuda")
    lm = torch.full((n,), -5.0, dtype=torch.float64, device="cuda")
    l0 = torch.full((1,), -5.0, dtype=torch.float64, device="cuda")
    zo.zo_mlp_losses(ctx, X, y, batch, n_in, n_hidden, n_out, n, eps, scale, lp, lm, l0)
    got = np.concatenate([l0.cpu().numpy(), lp.cpu().numpy(), lm.cpu().numpy()])
    ref = _per_probe(zo, ctx, X, y, batch, n_in, n_hidden, n_out, n, eps, scale)
    assert zo.zo_sync(ctx) == 0
    assert np.array_equal(got, ref), np.abs(got - ref).max()
    # without the clean loss: the probes' losses are the same values, *loss_clean untouched
    lp2 = torch.zeros_like(lp)
    lm2 = torch.zeros_like(lm)
    zo.zo_mlp_losses(ctx, X, y, batch, n_in, n_hidden, n_out, n, eps, scale, lp2, lm2)
    assert torch.equal(lp2, lp) and torch.equal(lm2, lm)
    assert th.numel() == M
    ctx.close()


def test_batched_mlp_losses_reject_bad_calls(zo):
    P = synth.mlp_params(0)
    th = torch.from_numpy(P).cuda()
    X = torch.zeros((64, 64), device="cuda")
    y = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.zeros(40, dtype=torch.float64, device="cuda")
    ctx = zo.zo_create(th, seed=1)
    with pytest.raises(zo.ZoError) as ei:  # shape does not match M
        zo.zo_mlp_losses(ctx, X, y, 64, 64, 128, 10, 4, 1e-3, 1.0, out[0:4], out[4:8])
    assert ei.value.status == zo.ZO_ERR_INVALID
    zo.zo_set_live_buffer(ctx, True)
    zo.zo_perturb(ctx, +1, 1e-3, 0)
    with pytest.raises(zo.ZoError) as ei:  # needs the clean state
        zo.zo_mlp_losses(ctx, X, y, 64, 64, 256, 10, 4, 1e-3, 1.0, out[0:4], out[4:8])
    assert ei.value.status == zo.ZO_ERR_STATE
    zo.zo_restore(ctx)
    ctx.close()
    big = torch.zeros(synth.mlp_param_count(64, 1000, 1), device="cuda")  # M = 66,001
    cb = zo.zo_create(big, seed=1)
    with pytest.raises(zo.ZoError) as ei:  # beyond the staged-parameter limit
        zo.zo_mlp_losses(cb, X, y, 64, 64, 1000, 1, 4, 1e-3, 1.0, out[0:4], out[4:8])
    assert ei.value.status == zo.ZO_ERR_UNSUPPORTED
    cb.close()
