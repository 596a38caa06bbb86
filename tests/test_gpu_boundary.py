"""The boundary calls that move data between the host and the step, and the measurement hooks:

  - zo_set_loss_location(ctx, 0): zo_step from host losses gives the same theta' (bit for
    bit) as from the same losses on the device;
  - zo_model_step_host: tokens and labels copied from host memory, losses copied back, the
    same losses and theta' as zo_model_step on device buffers;
  - zo_kernel_times / zo_launch_count: the recorded launches and their algorithmic work are
    the ones a decoder forward issues, counted independently from its configuration.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TINY = dict(n_layers=2, d_model=128, n_heads=2, d_ffn=512, vocab=1000, max_pos=128,
            class_ids=(3, 7))


def _bits_equal(a, b):
    return torch.equal(a.view(torch.int16 if a.dtype == torch.bfloat16 else torch.int32),
                       b.view(torch.int16 if b.dtype == torch.bfloat16 else torch.int32))


@pytest.mark.parametrize("preconditioned", [True, False])
def test_host_losses_step_equals_device_losses_step(zo, preconditioned):
    M, n = 40013, 24
    th_np, _ = synth.quad_problem(M, seed=21)
    lp, lm, L0 = synth.losses(n, seed=4)
    a = torch.from_numpy(th_np).cuda()
    b = a.clone()
    ca, cb = zo.zo_create(a, seed=5), zo.zo_create(b, seed=5)
    dev = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float64)).cuda()  # noqa: E731
    zo.zo_step(ca, dev(lp), dev(lm), n, dev([L0]) if preconditioned else None, 1e-2, 1e-3, 1e-3)
    zo.zo_set_loss_location(cb, False)
    host_l0 = np.array([L0]) if preconditioned else None
    zo.zo_step(cb, np.ascontiguousarray(lp), np.ascontiguousarray(lm), n, host_l0, 1e-2, 1e-3, 1e-3)
    assert zo.zo_sync(ca) == 0 and zo.zo_sync(cb) == 0
    assert zo.zo_get_step(ca) == zo.zo_get_step(cb) == 1
    assert _bits_equal(a, b)
    assert not torch.equal(a, torch.from_numpy(th_np).cuda())  # the step did move theta
    ga, gb = zo.zo_get_precond(ca, n), zo.zo_get_precond(cb, n)
    for x, y in zip(ga, gb):
        assert np.array_equal(x, y)
    # back to device losses on the same context
    zo.zo_set_loss_location(cb, True)
    zo.zo_step(cb, dev(lp), dev(lm), n, dev([L0]), 1e-2, 1e-3, 1e-3)
    assert zo.zo_sync(cb) == 0 and zo.zo_get_step(cb) == 2
    ca.close()
    cb.close()


def test_model_step_host_equals_device_step(zo):
    cfg = TINY
    B, S, k, n = 2, 64, 2, 4
    bits = synth.opt_params(cfg, seed=3, varied=True)
    toks, labs = zip(*(synth.opt_batch(cfg, B, S, seed=3, step=j) for j in range(k)))
    tokens, labels = np.stack(toks), np.stack(labs)
    thetas, losses = [], []
    for host in (False, True):
        th = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        ctx = zo.zo_create(th, seed=3)
        model = zo.zo_model_create(ctx, cfg, B * S)
        if host:
            L = np.zeros(2 * n + 1)
            pin_t = torch.from_numpy(tokens).pin_memory()
            pin_l = torch.from_numpy(labels).pin_memory()
            zo.zo_model_step_host(model, pin_t, pin_l, B, S, k, n, 1e-3, 1e-2, 1e-3, True, L)
        else:
            dl = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
            zo.zo_model_step(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                             B, S, k, n, 1e-3, 1e-2, 1e-3, True, dl)
            L = dl.cpu().numpy()
        assert zo.zo_sync(ctx) == 0 and zo.zo_get_step(ctx) == 1
        thetas.append(th)
        losses.append(L)
        model.close()
        ctx.close()
    assert np.array_equal(losses[0], losses[1])
    assert _bits_equal(thetas[0], thetas[1])


def test_kernel_times_count_the_forward_launches(zo):
    """One full-layer forward (pruning off) of a perturbed tiny OPT decoder issues, per layer,
    one window perturbation, 4 projection GEMMs and one attention; the recorded work is the
    algorithmic flops / bytes of those launches."""
    cfg = dict(TINY, n_layers=3)
    B, S = 2, 96
    d, f, H, Lyr = cfg["d_model"], cfg["d_ffn"], cfg["n_heads"], cfg["n_layers"]
    bits = synth.opt_params(cfg, seed=2)
    th = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(th, seed=2)
    model = zo.zo_model_create(ctx, cfg, B * S)
    zo.zo_model_set_pruning(model, False)
    tokens, labels = synth.opt_batch(cfg, B, S, seed=2)
    dtok, dlab = torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda()
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    n0 = zo.zo_launch_count(ctx)
    zo.zo_enable_kernel_timing(ctx, True)
    zo.zo_perturb(ctx, +1, 1e-3, 0)
    zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out)
    zo.zo_restore(ctx)
    kt, dropped = zo.zo_kernel_times(ctx)
    zo.zo_enable_kernel_timing(ctx, False)
    n1 = zo.zo_launch_count(ctx)
    T = B * S
    layer_params = 3 * d * d + 3 * d + d * d + d + 2 * d * f + f + d + 4 * d
    assert dropped == 0
    assert kt["gemm"]["launches"] == 4 * Lyr
    assert kt["gemm"]["work"] == Lyr * 2.0 * T * (3 * d * d + d * d + 2 * f * d)
    assert kt["attention"]["launches"] == Lyr
    hd = d // H
    assert kt["attention"]["work"] == Lyr * 4.0 * hd * B * H * S * (S + 1) / 2
    assert kt["perturb"]["launches"] == Lyr
    assert kt["perturb"]["work"] == Lyr * 2.0 * 2 * layer_params
    assert kt["update"]["launches"] == 0
    assert all(kt[c]["ms"] > 0 for c in ("gemm", "attention", "perturb"))
    # embedding, per layer (perturb, 2 LayerNorms, 4 GEMMs, attention), head
    assert n1 - n0 == 1 + 8 * Lyr + 1
    # timing off: nothing is recorded
    zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out)
    kt2, _ = zo.zo_kernel_times(ctx)
    assert all(v["launches"] == 0 for v in kt2.values())
    assert zo.zo_sync(ctx) == 0
    model.close()
    ctx.close()
