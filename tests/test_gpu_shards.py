"""Contexts on disjoint slices of one parameter vector, each with its element offset, behave
as one context on the whole vector: perturbed windows, packed probe bytes and updates agree
element by element (bit for bit), and the quadratic's losses are the sums of the slices'
losses (fp64 rounding).  One device holds all slices here; across devices the same contexts
run one per rank (zero_order_forward_b200.dist.element_parallel_step)."""
import pytest
import torch

import synth
from zero_order_forward_b200 import dist as zdist

pytestmark = pytest.mark.gpu

M = (1 << 20) + 40
WORLD = 3


def _contexts(zo, th, seed, step):
    """A context on th and contexts on the slices of a copy of th."""
    full = zo.zo_create(th, seed=seed)
    zo.zo_set_step(full, step)
    copy = th.clone()
    parts = []
    for r in range(WORLD):
        first, count = zdist.shard_range(M, r, WORLD)
        c = zo.zo_create(copy[first:first + count], seed=seed)
        zo.zo_set_element_offset(c, first)
        zo.zo_set_step(c, step)
        parts.append((first, count, c))
    return full, parts


def test_slices_perturb_and_pack_like_the_whole_vector(zo):
    th_np, _ = synth.quad_problem(M, seed=3)
    th = torch.from_numpy(th_np).cuda()
    full, parts = _contexts(zo, th, 9, 4)
    whole = torch.empty(M, device="cuda")
    zo.zo_perturb(full, -1, 1e-3, 13)
    zo.zo_perturb_range(full, 0, M, whole)
    zo.zo_restore(full)
    packed = torch.empty(M // 8 + 1, dtype=torch.uint8, device="cuda")
    zo.zo_pack_probe(full, 0, 13, 0, (M + 7) // 8, packed)
    for first, count, c in parts:
        out = torch.empty(count, device="cuda")
        zo.zo_perturb(c, -1, 1e-3, 13)
        zo.zo_perturb_range(c, 0, count, out)
        zo.zo_restore(c)
        assert torch.equal(out, whole[first:first + count])
        pb = torch.empty((count + 7) // 8, dtype=torch.uint8, device="cuda")
        zo.zo_pack_probe(c, 0, 13, 0, (count + 7) // 8, pb)
        assert torch.equal(pb, packed[first // 8:first // 8 + (count + 7) // 8])
        c.close()
    full.close()


def test_slices_losses_sum_and_updates_agree(zo):
    th_np, D_np = synth.quad_problem(M, seed=4)
    th = torch.from_numpy(th_np).cuda()
    D = torch.from_numpy(D_np).cuda()
    n, eps = 64, 1e-3
    full, parts = _contexts(zo, th, 2, 7)
    ref = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_quad_loss_octet(full, D, 0, 64, eps, ref[1:65], ref[65:129], ref[0:1])
    tot = torch.zeros_like(ref)
    for first, count, c in parts:
        loc = torch.zeros_like(ref)
        zo.zo_quad_loss_octet(c, D[first:first + count], 0, 64, eps, loc[1:65], loc[65:129], loc[0:1])
        tot += loc
    assert torch.allclose(tot, ref, rtol=1e-12, atol=0)
    # the same summed losses drive the whole-vector step and every slice's step
    th_full = full.params
    zo.zo_step(full, tot[1:65], tot[65:129], n, tot[0:1], 1e-7, eps, 1e-3)
    for first, count, c in parts:
        zo.zo_step(c, tot[1:65], tot[65:129], n, tot[0:1], 1e-7, eps, 1e-3)
    torch.cuda.synchronize()
    for first, count, c in parts:
        assert zo.zo_sync(c) == 0
        assert torch.equal(c.params, th_full[first:first + count])
        assert zo.zo_get_step(c) == zo.zo_get_step(full) == 8
        c.close()
    full.close()


def test_offset_rules(zo):
    th = torch.zeros(synth.mlp_param_count(), device="cuda")
    c = zo.zo_create(th, seed=1)
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_set_element_offset(c, 8)  # not a whole sign group
    assert ei.value.status == zo.ZO_ERR_INVALID
    zo.zo_set_element_offset(c, 32)
    X = torch.zeros((64, 64), device="cuda")
    y = torch.zeros(64, dtype=torch.int32, device="cuda")
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    with pytest.raises(zo.ZoError) as ei:  # the MLP loss is not a sum over slices
        zo.zo_mlp_loss(c, X, y, 64, 64, 256, 10, 1.0, out[0:1])
    assert ei.value.status == zo.ZO_ERR_UNSUPPORTED
    zo.zo_set_element_offset(c, 0)
    zo.zo_mlp_loss(c, X, y, 64, 64, 256, 10, 1.0, out[0:1])
    assert zo.zo_sync(c) == 0
    c.close()
