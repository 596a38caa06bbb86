"""Probe-parallel and element-parallel zero-order steps across ranks (one process per GPU).

Splitting probe evaluation across devices needs no gradient communication
("Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section "How 1.5-SPSA
Works", implementation paragraph: there are no gradients to communicate).  Every rank holds
the same theta and seed, so the probes z_i are identical everywhere; rank r evaluates the
probes i = r, r + N, r + 2N, ... (or, with block = B, the blocks of B consecutive probes
u = r, r + N, ...: the probe octets of the quadratic's one-pass evaluation).  The only exchange is an all-gather of the 2*n_pert fp64
losses; afterwards every rank runs the same deterministic preconditioner and update, so the
replicas of theta stay bit-identical with no parameter traffic.

For a loss that is a sum of per-element terms (the diagonal quadratic), the parameters can
instead be cut into contiguous slices, one per rank (element_parallel_step): every rank
evaluates all 2 n + 1 losses over its own slice's terms (the context's element offset keeps
each element's signs those of its global index), the partial losses are all-gathered and
summed in rank order, so every rank holds the same totals bit for bit, and each rank runs the
preconditioner and updates its own slice.  This is the batch-parallel split with the loss's
terms as the batch; the parameters are sharded with them, so neither the evaluation nor the
update is repeated on every rank, and only 2 n + 1 numbers per rank cross the network.

The per-rank loss evaluation and the update are passed in as callables, so this module
holds only the partition and the exchange (torch.distributed: NCCL on GPUs; gloo works for
host-side tests).
"""
import math

import torch
import torch.distributed as dist


def rank_units(n_pert, rank, world, block=1):
    """(first, count) of the probe blocks evaluated by `rank`: blocks u = rank (mod world)
    of `block` consecutive probes (the last block may be short)."""
    if not (0 <= rank < world) or n_pert < 1 or block < 1:
        raise ValueError("bad partition arguments")
    units = math.ceil(n_pert / block)
    return [(u * block, min(block, n_pert - u * block)) for u in range(rank, units, world)]


def rank_probes(n_pert, rank, world, block=1):
    """Probes evaluated by `rank`, ascending."""
    return [f + t for f, c in rank_units(n_pert, rank, world, block) for t in range(c)]


def slots(n_pert, world, block=1):
    """Loss slots per rank in the exchange buffer (the largest share)."""
    return max(len(rank_probes(n_pert, r, world, block)) for r in range(world))


def global_order(n_pert, world, device=None, block=1):
    """Index of each gathered slot in the global probe order, -1 for padding.

    The gathered buffer is [world][2][slots]; entry (r, s, k) holds the k-th probe of
    rank_probes(n_pert, r, world, block)."""
    k = slots(n_pert, world, block)
    idx = torch.full((world, k), -1, dtype=torch.long)
    for r in range(world):
        p = rank_probes(n_pert, r, world, block)
        idx[r, :len(p)] = torch.tensor(p, dtype=torch.long)
    return idx.to(device) if device is not None else idx


def gather_losses(local, n_pert, group=None, block=1):
    """All-gather every rank's [2][slots] losses (row 0: L+, row 1: L-) and return the
    full (L+[n_pert], L-[n_pert]) in global probe order, on every rank."""
    world = dist.get_world_size(group)
    k = slots(n_pert, world, block)
    if tuple(local.shape) != (2, k):
        raise ValueError(f"local losses must be [2][{k}]")
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    full = torch.stack(parts)  # [world][2][k]
    idx = global_order(n_pert, world, full.device, block)
    valid = idx >= 0
    Lp = torch.empty(n_pert, dtype=local.dtype, device=local.device)
    Lm = torch.empty(n_pert, dtype=local.dtype, device=local.device)
    Lp[idx[valid]] = full[:, 0, :][valid]
    Lm[idx[valid]] = full[:, 1, :][valid]
    return Lp, Lm


def batch_share(batch, rank, world):
    """(first, count) of rank's contiguous share of `batch` sequences (count may be 0)."""
    if not (0 <= rank < world) or batch < 0:
        raise ValueError("bad batch partition arguments")
    per = -(-batch // world) if batch else 0
    first = min(batch, rank * per)
    return first, min(batch, first + per) - first


def probe_parallel_step(n_pert, loss_at, clean_loss, apply_step, device, dtype=torch.float64,
                        group=None, pair_at=None, block=1, block_at=None, clean_shared=False):
    """One step with this rank's share of the probes.

    loss_at(sign, probe, out) writes L(theta + sign*eps*z_probe) into the 1-element tensor
    `out`; pair_at(probe, out_plus, out_minus), if given, writes both signs at once instead;
    block_at(first, count, out_plus, out_minus), if given, writes both signs of the `count`
    probes from `first` (one block of the partition, `block` probes) at once;
    clean_loss(out) writes L0: with clean_shared False every rank computes the whole clean
    loss (same theta, same data, same value, no exchange); with clean_shared True it writes
    this rank's partial sum over its share of the batch (batch_share), and the partials are
    all-gathered and added in rank order, so every rank holds the same L0 bits;
    apply_step(Lp, Lm, L0) runs the preconditioner and the update.
    Returns (L0, Lp, Lm)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if block_at is None:
        block = 1
    k = slots(n_pert, world, block)
    local = torch.zeros((2, k), dtype=dtype, device=device)
    L0 = torch.zeros(1, dtype=dtype, device=device)
    clean_loss(L0)
    if clean_shared:
        L0 = sum_partials(L0, group)
    j = 0
    for first, count in rank_units(n_pert, rank, world, block):
        if block_at is not None:
            block_at(first, count, local[0, j:j + count], local[1, j:j + count])
        else:
            for i in range(first, first + count):
                jj = j + i - first
                if pair_at is not None:
                    pair_at(i, local[0, jj:jj + 1], local[1, jj:jj + 1])
                else:
                    loss_at(+1, i, local[0, jj:jj + 1])
                    loss_at(-1, i, local[1, jj:jj + 1])
        j += count
    Lp, Lm = gather_losses(local, n_pert, group, block)
    apply_step(Lp, Lm, L0)
    return L0, Lp, Lm


def shard_range(M, rank, world, align=16):
    """(first, count) of rank's contiguous slice of M elements: slices of ceil(M / world)
    elements rounded up to a multiple of `align` (whole sign groups), the last one shorter."""
    if not (0 <= rank < world) or M < 1 or align < 1:
        raise ValueError("bad shard arguments")
    per = -(-M // world)
    per = -(-per // align) * align
    first = min(M, rank * per)
    return first, min(M, first + per) - first


def sum_partials(local, group=None):
    """All-gather every rank's partial sums (a 1-D tensor) and add them in rank order, so
    that every rank obtains the same bits."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local.contiguous(), group=group)
    total = parts[0].clone()
    for p in parts[1:]:
        total += p
    return total


def element_parallel_step(n_pert, partial_losses, apply_step, device, dtype=torch.float64,
                          group=None):
    """One step with the parameters sharded by elements, for a loss that is a sum over
    elements.  partial_losses(out) writes this rank's [L0, L+_0..L+_{n-1}, L-_0..L-_{n-1}]
    over its slice's terms (2 n + 1 values); apply_step(Lp, Lm, L0) runs the preconditioner and
    the update of this rank's slice with the summed losses.  Returns the summed losses."""
    local = torch.zeros(2 * n_pert + 1, dtype=dtype, device=device)
    partial_losses(local)
    total = sum_partials(local, group)
    apply_step(total[1:1 + n_pert], total[1 + n_pert:], total[0:1])
    return total
