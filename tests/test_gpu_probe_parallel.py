"""The probe-parallel step on the CUDA path: two ranks (processes, gloo for the loss exchange)
share the one GPU; each holds a replica of theta, evaluates its share of the probes (and, in
the batch-shared mode, of the clean batch) through libzo, and applies the same step.

Splitting probe evaluation across devices needs no gradient communication ("Stanford's
1.5-SPSA Trains OPT-30B Without Backpropagation", section "Probe-Space Preconditioning"):
after the all-gather of the losses the replicas stay bit-identical.  Checked against the
single-process zo_model_step (same kernels on the same inputs, so the same loss bits) and,
for the batch-shared clean loss, against the oracle's preconditioner and fixed-order update
fed with the gathered losses.  The ranks' kernels never wait on one another: the only
exchange is gloo's, on the host, between launches.
"""
import os
import socket

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

CFG = dict(n_layers=2, d_model=128, n_heads=2, d_ffn=512, vocab=1000, max_pos=128, class_ids=(3, 7))
B, S, K, N, EPS, LR, LAM, SEED = 3, 64, 2, 6, 1e-3, 1e-2, 1e-3, 4


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs():
    bits = synth.opt_params(CFG, seed=SEED, varied=True)
    toks, labs = zip(*(synth.opt_batch(CFG, B, S, seed=SEED, step=j) for j in range(K)))
    return bits, np.stack(toks), np.stack(labs)


def _rank(rank, world, port, out_dir, clean_shared):
    import datetime

    import torch.distributed as dist

    import zero_order_forward_b200 as zo
    from zero_order_forward_b200 import dist as zdist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        bits, tokens, labels = _inputs()
        theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        ctx = zo.zo_create(theta, seed=SEED)
        model = zo.zo_model_create(ctx, CFG, B * S)
        dtok, dlab = torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda()
        scratch = torch.zeros(1, dtype=torch.float64, device="cuda")
        scale = 1.0 / (K * B)
        b0, nb = zdist.batch_share(B, rank, world) if clean_shared else (0, B)

        def loss_at(sign, probe, out):  # out: a CPU tensor (gloo exchanges host memory)
            zo.zo_perturb(ctx, sign, EPS, probe)
            for j in range(K):
                zo.zo_model_loss(model, dtok[j], dlab[j], B, S, scale, scratch, j > 0)
            zo.zo_restore(ctx)
            out.copy_(scratch.cpu())

        def clean(out):
            scratch.zero_()
            for j in range(K if nb else 0):
                zo.zo_model_loss(model, dtok[j, b0:b0 + nb], dlab[j, b0:b0 + nb], nb, S, scale,
                                 scratch, j > 0)
            out.copy_(scratch.cpu())

        def apply_step(Lp, Lm, L0):
            zo.zo_step(ctx, Lp.cuda(), Lm.cuda(), N, L0.cuda(), LR, EPS, LAM)

        L0, Lp, Lm = zdist.probe_parallel_step(N, loss_at, clean, apply_step, "cpu",
                                               clean_shared=clean_shared)
        assert zo.zo_sync(ctx) == 0
        np.savez(os.path.join(out_dir, f"r{rank}.npz"),
                 theta=theta.view(torch.int16).cpu().numpy().view(np.uint16),
                 L=np.concatenate([L0.numpy(), Lp.numpy(), Lm.numpy()]))
        model.close()
        ctx.close()
    finally:
        dist.destroy_process_group()


def _single_process(zo):
    bits, tokens, labels = _inputs()
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=SEED)
    model = zo.zo_model_create(ctx, CFG, B * S)
    losses = torch.zeros(2 * N + 1, dtype=torch.float64, device="cuda")
    zo.zo_model_step(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                     B, S, K, N, EPS, LR, LAM, True, losses)
    assert zo.zo_sync(ctx) == 0
    out = theta.view(torch.int16).cpu().numpy().view(np.uint16), losses.cpu().numpy()
    model.close()
    ctx.close()
    return out


@pytest.mark.parametrize("clean_shared", [False, True])
def test_two_ranks_on_the_cuda_path_match_one(zo, tmp_path, clean_shared):
    import torch.multiprocessing as mp

    from oracle import core
    world = 2
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path), clean_shared),
                       nprocs=world, start_method="spawn", join=True)
    r = [np.load(os.path.join(tmp_path, f"r{i}.npz")) for i in range(world)]
    assert np.array_equal(r[0]["theta"], r[1]["theta"])  # bit-identical replicas
    assert np.array_equal(r[0]["L"], r[1]["L"])
    th1, L1 = _single_process(zo)
    L = r[0]["L"]
    # every perturbed loss is the same kernels' result on the same inputs
    assert np.array_equal(L[1:], L1[1:])
    if not clean_shared:
        assert np.array_equal(L, L1)
        assert np.array_equal(r[0]["theta"], th1)
    else:
        # the clean loss is the rank-order sum of two batch shares: the same value up to
        # the fp64 rounding of the regrouped sum
        assert abs(L[0] - L1[0]) <= 1e-14 * abs(L1[0])
    # teacher forcing: the oracle's preconditioner and fixed-order update from the gathered
    # losses give the replicas' theta bit for bit
    e32 = float(np.float32(EPS))
    pc = core.precond(L[1:1 + N], L[1 + N:], L[0], e32, float(np.float32(LR)),
                      float(np.float32(LAM)), float(np.float32(0.1)))
    bits, _, _ = _inputs()
    nxt = core.update_mirror(bits, pc["a"].astype(np.float32), SEED, 0)
    assert np.array_equal(r[0]["theta"], nxt)
