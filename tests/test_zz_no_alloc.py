"""The allocation-free MLP loss (zo_mlp_loss_noalloc) against the context-based one.

zo_mlp_loss_noalloc serves callers that must not call cudaMalloc (a host framework that
owns every device allocation): it takes inputs and outputs only and keeps its reduction
scratch in the library's static device memory.
This file is collected last so that a run stopping at the first failure has already run
every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _inputs(batch):
    P = synth.mlp_params(3)
    teacher = synth.mlp_params(3, tag="teacher")
    X, y = synth.mlp_batch(3, 0, teacher, batch=batch)
    return (torch.from_numpy(P).cuda(), torch.from_numpy(X).cuda(), torch.from_numpy(y).cuda())


def test_noalloc_matches_context_entry_point_on_two_calls(zo):
    batch = 64
    P, X, y = _inputs(batch)
    ctx = zo.zo_create(P, seed=0)
    ref = torch.zeros(1, dtype=torch.float64, device="cuda")
    zo.zo_mlp_loss(ctx, X, y, batch, 64, 256, 10, 1.0 / batch, ref)
    out = torch.full((2,), -1.0, dtype=torch.float64, device="cuda")
    # a first call loads whatever the driver loads lazily for this code; the memory check
    # covers the calls after it
    zo.zo_mlp_loss_noalloc(P, X, y, batch, 64, 256, 10, 1.0 / batch, out[0:1])
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()
    # two calls in a row share the static scratch (the counter is re-armed each call)
    zo.zo_mlp_loss_noalloc(P, X, y, batch, 64, 256, 10, 1.0 / batch, out[0:1])
    zo.zo_mlp_loss_noalloc(P, X, y, batch, 64, 256, 10, 1.0 / batch, out[1:2])
    torch.cuda.synchronize()
    # nothing was allocated, by torch or by the library (memory may only have been released,
    # by an unrelated tensor going out of scope)
    assert torch.cuda.memory_allocated() <= torch_before
    assert torch.cuda.mem_get_info()[0] >= free_before
    r = ref.item()
    got = out.cpu().numpy()
    # the same kernel in the same reduction order as the context's entry point: equal bits
    assert np.all(got == r), (got, r)
    # accumulate mode on the second call of another pair
    acc = torch.zeros(1, dtype=torch.float64, device="cuda")
    zo.zo_mlp_loss_noalloc(P, X[:32], y[:32], 32, 64, 256, 10, 1.0 / batch, acc)
    zo.zo_mlp_loss_noalloc(P, X[32:], y[32:], 32, 64, 256, 10, 1.0 / batch, acc, accumulate=True)
    torch.cuda.synchronize()
    assert abs(acc.item() - r) <= 1e-5 * abs(r)
    ctx.close()


def test_noalloc_rejects_batches_beyond_its_scratch(zo):
    P, X, y = _inputs(8)
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_mlp_loss_noalloc(P, X, y, zo.ZO_NOALLOC_MAX_BATCH + 1, 64, 256, 10, 1.0, out)
    assert ei.value.status == zo.ZO_ERR_INVALID
