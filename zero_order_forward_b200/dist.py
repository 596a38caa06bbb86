"""Probe-parallel zero-order steps across ranks (one process per GPU).

Splitting probe evaluation across devices needs no gradient communication
("Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section "How 1.5-SPSA
Works", implementation paragraph: there are no gradients to communicate).  Every rank holds
the same theta and seed, so the probes z_i are identical everywhere; rank r evaluates the
probes i = r, r + N, r + 2N, ... .  The only exchange is an all-gather of the 2*n_pert fp64
losses; afterwards every rank runs the same deterministic preconditioner and update, so the
replicas of theta stay bit-identical with no parameter traffic.

The per-rank loss evaluation and the update are passed in as callables, so this module
holds only the partition and the exchange (torch.distributed: NCCL on GPUs; gloo works for
host-side tests).
"""
import math

import torch
import torch.distributed as dist


def rank_probes(n_pert, rank, world):
    """Probes evaluated by `rank`, ascending: i = rank (mod world)."""
    if not (0 <= rank < world) or n_pert < 1:
        raise ValueError("bad partition arguments")
    return list(range(rank, n_pert, world))


def slots(n_pert, world):
    """Loss slots per rank in the exchange buffer (the largest share)."""
    return math.ceil(n_pert / world)


def global_order(n_pert, world, device=None):
    """Index of each gathered slot in the global probe order, -1 for padding.

    The gathered buffer is [world][2][slots]; entry (r, s, k) holds probe r + k*world."""
    k = slots(n_pert, world)
    idx = torch.full((world, k), -1, dtype=torch.long)
    for r in range(world):
        p = rank_probes(n_pert, r, world)
        idx[r, :len(p)] = torch.tensor(p, dtype=torch.long)
    return idx.to(device) if device is not None else idx


def gather_losses(local, n_pert, group=None):
    """All-gather every rank's [2][slots] losses (row 0: L+, row 1: L-) and return the
    full (L+[n_pert], L-[n_pert]) in global probe order, on every rank."""
    world = dist.get_world_size(group)
    k = slots(n_pert, world)
    if tuple(local.shape) != (2, k):
        raise ValueError(f"local losses must be [2][{k}]")
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    full = torch.stack(parts)  # [world][2][k]
    idx = global_order(n_pert, world, full.device)
    valid = idx >= 0
    Lp = torch.empty(n_pert, dtype=local.dtype, device=local.device)
    Lm = torch.empty(n_pert, dtype=local.dtype, device=local.device)
    Lp[idx[valid]] = full[:, 0, :][valid]
    Lm[idx[valid]] = full[:, 1, :][valid]
    return Lp, Lm


def probe_parallel_step(n_pert, loss_at, clean_loss, apply_step, device, dtype=torch.float64,
                        group=None, pair_at=None):
    """One step with this rank's share of the probes.

    loss_at(sign, probe, out) writes L(theta + sign*eps*z_probe) into the 1-element tensor
    `out`; pair_at(probe, out_plus, out_minus), if given, writes both signs at once instead;
    clean_loss(out) writes L0 (every rank computes it: same theta, same data, same value, no
    exchange); apply_step(Lp, Lm, L0) runs the preconditioner and the update.
    Returns (L0, Lp, Lm)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    k = slots(n_pert, world)
    local = torch.zeros((2, k), dtype=dtype, device=device)
    L0 = torch.zeros(1, dtype=dtype, device=device)
    clean_loss(L0)
    for j, i in enumerate(rank_probes(n_pert, rank, world)):
        if pair_at is not None:
            pair_at(i, local[0, j:j + 1], local[1, j:j + 1])
        else:
            loss_at(+1, i, local[0, j:j + 1])
            loss_at(-1, i, local[1, j:j + 1])
    Lp, Lm = gather_losses(local, n_pert, group)
    apply_step(Lp, Lm, L0)
    return L0, Lp, Lm
