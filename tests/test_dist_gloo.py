"""Host-side logic of the probe-parallel and element-parallel steps on 2 and 3 CPU ranks
(gloo): the probe partition, the element slices, the loss exchange and bit-identical
replicas or slices.  The per-probe loss and the update
are the oracle's here (CPU); on GPUs the same driver calls the CUDA library over NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from zero_order_forward_b200 import dist as zdist


def test_partition_covers_every_probe_once():
    for n in (1, 2, 5, 16, 64, 161):
        for world in (1, 2, 3, 8):
            for block in (1, 8):
                seen = sorted(i for r in range(world)
                              for i in zdist.rank_probes(n, r, world, block))
                assert seen == list(range(n))
                idx = zdist.global_order(n, world, block=block)
                assert idx.shape == (world, zdist.slots(n, world, block))
                assert sorted(idx[idx >= 0].tolist()) == list(range(n))
                for r in range(world):  # blocks are whole octets except the last
                    for first, count in zdist.rank_units(n, r, world, block):
                        assert first % block == 0 and 1 <= count <= block


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


M, N_PERT, EPS, LR, LAM, SEED = 3000, 7, 1e-3, 1e-5, 1e-3, 5


def _worker(rank, world, port, out_dir, block=1):
    import torch.distributed as dist

    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        theta, D = synth.quad_problem(M, seed=1)
        state = {"theta": theta}
        e32 = float(np.float32(EPS))

        def loss_at(sign, probe, out):
            P = oracle.core.perturb(state["theta"], SEED, 0, probe, sign, e32)
            out[0] = oracle.core.quad_loss(P, D)

        def clean(out):
            out[0] = oracle.core.quad_loss(state["theta"], D)

        def apply_step(Lp, Lm, L0):
            pc = oracle.core.precond(Lp.numpy(), Lm.numpy(), float(L0[0]), e32,
                                     float(np.float32(LR)), float(np.float32(LAM)),
                                     float(np.float32(0.1)))
            state["theta"] = oracle.core.update_mirror(state["theta"], pc["a"].astype(np.float32),
                                                       SEED, 0)

        def block_at(first, count, out_p, out_m):  # a block's losses written at once
            for t in range(count):
                loss_at(+1, first + t, out_p[t:t + 1])
                loss_at(-1, first + t, out_m[t:t + 1])

        L0, Lp, Lm = zdist.probe_parallel_step(N_PERT, loss_at, clean, apply_step, "cpu",
                                               block=block,
                                               block_at=block_at if block > 1 else None)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), theta=state["theta"], L0=L0.numpy(),
                 Lp=Lp.numpy(), Lm=Lm.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,block", [(2, 1), (3, 1), (2, 4)])
def test_probe_parallel_step_matches_single_rank(tmp_path, world, block):
    import oracle
    import synth
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), block), nprocs=world,
                       join=True, start_method="spawn")
    theta, D = synth.quad_problem(M, seed=1)
    nxt, rec = oracle.step.spsa_step(theta, lambda P: oracle.core.quad_loss(P, D), N_PERT, EPS,
                                     LR, LAM, SEED, 0, update="mirror")
    outs = [np.load(tmp_path / f"r{r}.npz") for r in range(world)]
    for o in outs:
        assert np.array_equal(o["Lp"], rec["Lp"]) and np.array_equal(o["Lm"], rec["Lm"])
        assert o["L0"][0] == rec["L0"]
        assert o["theta"].tobytes() == nxt.tobytes()  # bit-identical replicas


def test_shard_ranges_tile_the_vector():
    for M in (16, 17, 3000, 1 << 20, (1 << 24) + 5):
        for world in (1, 2, 3, 8):
            ranges = [zdist.shard_range(M, r, world) for r in range(world)]
            assert sum(c for _, c in ranges) == M
            pos = 0
            for first, count in ranges:
                assert first == pos and count >= 0
                assert count == 0 or first % 16 == 0  # empty slices only past the end
                pos += count


def _element_worker(rank, world, port, out_dir):
    import torch.distributed as dist

    import oracle
    import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        theta, D = synth.quad_problem(M, seed=1)
        first, count = zdist.shard_range(M, rank, world)
        th, Ds = theta[first:first + count].copy(), D[first:first + count]
        e32 = float(np.float32(EPS))
        state = {}

        def partial_losses(out):  # this slice's terms, signs of the global element index
            out[0] = oracle.core.quad_loss(th, Ds)
            for i in range(N_PERT):
                for s, off in ((+1, 1), (-1, 1 + N_PERT)):
                    P = oracle.core.perturb(th, SEED, 0, i, s, e32, j0=first)
                    out[off + i] = oracle.core.quad_loss(P, Ds)

        def apply_step(Lp, Lm, L0):
            pc = oracle.core.precond(Lp.numpy(), Lm.numpy(), float(L0[0]), e32,
                                     float(np.float32(LR)), float(np.float32(LAM)),
                                     float(np.float32(0.1)))
            state["a"] = pc["a"].astype(np.float32)
            state["theta"] = oracle.core.update_mirror(th, state["a"], SEED, 0, j0=first)

        tot = zdist.element_parallel_step(N_PERT, partial_losses, apply_step, "cpu")
        np.savez(os.path.join(out_dir, f"e{rank}.npz"), theta=state["theta"], a=state["a"],
                 tot=tot.numpy(), first=first)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_element_parallel_step_matches_single_rank(tmp_path, world):
    """Every rank sums the same totals (bit for bit); they equal the whole vector's losses to
    fp64 rounding; each rank's updated slice equals the whole-vector update with the same
    coefficients, element by element."""
    import oracle
    import synth
    mp.start_processes(_element_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    theta, D = synth.quad_problem(M, seed=1)
    _, rec = oracle.step.spsa_step(theta, lambda P: oracle.core.quad_loss(P, D), N_PERT, EPS,
                                   LR, LAM, SEED, 0, update="mirror")
    outs = [np.load(tmp_path / f"e{r}.npz") for r in range(world)]
    ref = np.concatenate([[rec["L0"]], rec["Lp"], rec["Lm"]])
    for o in outs:
        assert np.array_equal(o["tot"], outs[0]["tot"]) and np.array_equal(o["a"], outs[0]["a"])
        assert np.allclose(o["tot"], ref, rtol=1e-13, atol=0)
    full = oracle.core.update_mirror(theta, outs[0]["a"], SEED, 0)
    got = np.concatenate([o["theta"] for o in outs])
    assert got.tobytes() == full.tobytes()


def test_batch_share_covers_every_sequence_once():
    for batch in (0, 1, 2, 7, 8, 16):
        for world in (1, 2, 3, 8):
            got = []
            for r in range(world):
                first, count = zdist.batch_share(batch, r, world)
                assert count >= 0
                got += list(range(first, first + count))
            assert got == list(range(batch))


def _clean_shared_worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_seq = np.arange(1, 8, dtype=np.float64) * 0.1  # per-sequence clean losses
        first, count = zdist.batch_share(per_seq.size, rank, world)

        def clean(out):
            out[0] = float(per_seq[first:first + count].sum())

        def loss_at(sign, probe, out):
            out[0] = 10.0 * probe + sign

        seen = {}

        def apply_step(Lp, Lm, L0):
            seen["L0"] = float(L0[0])

        L0, Lp, Lm = zdist.probe_parallel_step(5, loss_at, clean, apply_step, "cpu",
                                               clean_shared=True)
        np.savez(os.path.join(out_dir, f"c{rank}.npz"), L0=L0.numpy(), Lp=Lp.numpy(),
                 Lm=Lm.numpy(), seen=seen["L0"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_clean_loss_shared_by_batch(tmp_path, world):
    mp.start_processes(_clean_shared_worker, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    rs = [np.load(os.path.join(tmp_path, f"c{r}.npz")) for r in range(world)]
    per_seq = np.arange(1, 8, dtype=np.float64) * 0.1
    parts = [per_seq[slice(*(lambda f, c: (f, f + c))(*zdist.batch_share(7, r, world)))].sum()
             for r in range(world)]
    want = parts[0]
    for p in parts[1:]:
        want += p  # rank order
    for r in rs:
        assert r["L0"][0] == want and float(r["seen"]) == want
        assert np.array_equal(r["Lp"], 10.0 * np.arange(5) + 1)
        assert np.array_equal(r["Lm"], 10.0 * np.arange(5) - 1)
