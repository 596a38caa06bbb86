"""Parity of the CUDA path (through the C ABI) with the CPU oracle, element by element.

Tolerances (written per test):
  - probe bits, perturbed parameters, restore: bit-exact;
  - update with given coefficients: bit-exact against the oracle's fixed fp32 order;
  - quadratic loss (fp64 on both sides, different summation order): 1e-12 relative;
  - MLP loss (fp32 on the GPU, fp64 oracle): 1e-5 relative;
  - full step: losses as above, theta' within the propagated bound stated in the test.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import core

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def host_bits(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


_CUDART = None


def copy_raw(dst, src_ptr):
    """Device-to-device copy of dst.nbytes from a raw device address into dst."""
    global _CUDART
    import ctypes
    if _CUDART is None:
        for name in ("libcudart.so.12", "libcudart.so"):
            try:
                _CUDART = ctypes.CDLL(name)
                break
            except OSError:
                continue
    torch.cuda.synchronize()
    rc = _CUDART.cudaMemcpy(ctypes.c_void_p(dst.data_ptr()), ctypes.c_void_p(src_ptr),
                            ctypes.c_size_t(dst.numel() * dst.element_size()), 3)
    assert rc == 0
    torch.cuda.synchronize()


SIZES = [1, 7, 127, 128, 129, 1000, 4096 + 5, 19210, (1 << 17) + 77]


@pytest.mark.parametrize("M", SIZES)
def test_pack_probe_bit_exact(zo, M):
    th = torch.zeros(max(M, 4), device="cuda")
    seed = 0x0123456789ABCDEF
    ctx = zo.zo_create(th, seed=seed, M=M)
    # the step is an argument: the context's own counter (0 here) is not read
    for step in (0, 5, 0xFFFFFFFF):
        for probe in (0, 3, 1023):
            nbytes = (M + 7) // 8
            out = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
            zo.zo_pack_probe(ctx, step, probe, 0, nbytes, out)
            torch.cuda.synchronize()
            assert (out.cpu().numpy() == core.pack_probe(seed, step, probe, M)).all()
            if nbytes > 20:  # a window starting mid-group
                w = torch.zeros(nbytes - 19, dtype=torch.uint8, device="cuda")
                zo.zo_pack_probe(ctx, step, probe, 19, nbytes - 19, w)
                torch.cuda.synchronize()
                assert (w.cpu().numpy() == core.pack_probe(seed, step, probe, M)[19:]).all()
    ctx.close()


def _theta(M, dtype, seed=1):
    r = np.random.default_rng(seed)
    x = r.standard_normal(M).astype(np.float32)
    x[: min(M, 6)] = [0.0, -0.0, 1e-40, 1.0, -1.0, 3e38][: min(M, 6)]
    if dtype == "f32":
        return x
    return synth.to_bf16_bits(x * 0.02)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M", SIZES)
def test_perturb_bit_exact_and_restore_exact(zo, M, dtype):
    th_np = _theta(M, dtype)
    th = dev(th_np) if dtype == "f32" else bf16_dev(th_np)
    before = host_bits(th).copy()
    ctx = zo.zo_create(th, seed=42)
    zo.zo_set_step(ctx, 3)
    zo.zo_set_live_buffer(ctx, True)
    for sign in (+1, -1):
        for probe, eps in ((0, 1e-3), (7, 0.25)):
            zo.zo_perturb(ctx, sign, eps, probe)
            ref = core.perturb(th_np, 42, 3, probe, sign, eps)
            # the whole vector as materialised into the live buffer by zo_perturb
            live = torch.empty_like(th)
            copy_raw(live, zo.zo_live_params(ctx))
            assert (host_bits(live) == ref).all()
            out = torch.empty_like(th)
            zo.zo_perturb_range(ctx, 0, M, out)
            torch.cuda.synchronize()
            assert (host_bits(out) == ref).all()
            # ragged windows (unaligned start, odd length)
            for first, count in ((1, M - 1), (M // 3, M - M // 3 - 1), (0, 0)):
                if count <= 0 or first + count > M:
                    continue
                w = torch.empty(count, dtype=th.dtype, device="cuda")
                zo.zo_perturb_range(ctx, first, count, w)
                torch.cuda.synchronize()
                assert (host_bits(w) == ref[first:first + count]).all()
            zo.zo_restore(ctx)
    # clean state: the window copy is theta itself
    out = torch.empty_like(th)
    zo.zo_perturb_range(ctx, 0, M, out)
    torch.cuda.synchronize()
    assert (host_bits(out) == before).all()
    assert (host_bits(th) == before).all()  # exact restore: theta never written
    ctx.close()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("first,count", [(0, (1 << 23) + 40), (8, (1 << 23) + 5)])
def test_perturb_window_many_chunks_per_cta(zo, dtype, first, count):
    """A window far larger than one pass of the grid (each CTA streams several chunks through
    its ring of stages): bit-exact against the oracle, clean and perturbed."""
    M = first + count + 3
    th_np = _theta(M, dtype, seed=5)
    th = dev(th_np) if dtype == "f32" else bf16_dev(th_np)
    ctx = zo.zo_create(th, seed=13)
    zo.zo_set_step(ctx, 2)
    out = torch.empty(count, dtype=th.dtype, device="cuda")
    zo.zo_perturb_range(ctx, first, count, out)
    torch.cuda.synchronize()
    assert (host_bits(out) == host_bits(th)[first:first + count]).all()
    zo.zo_perturb(ctx, -1, 1e-3, 21)
    zo.zo_perturb_range(ctx, first, count, out)
    torch.cuda.synchronize()
    zo.zo_restore(ctx)
    ref = core.perturb(th_np, 13, 2, 21, -1, 1e-3)
    assert (host_bits(out) == ref[first:first + count]).all()
    ctx.close()


def test_live_buffer_switches_back_on_restore(zo):
    M = 19210
    th_np = _theta(M, "f32")
    th = dev(th_np)
    ctx = zo.zo_create(th, seed=9)
    zo.zo_set_live_buffer(ctx, True)
    zo.zo_perturb(ctx, -1, 1e-3, 11)
    assert zo.zo_live_params(ctx) != th.data_ptr()
    buf = torch.empty_like(th)
    copy_raw(buf, zo.zo_live_params(ctx))
    assert (buf.cpu().numpy() == core.perturb(th_np, 9, 0, 11, -1, 1e-3)).all()
    zo.zo_restore(ctx)
    assert zo.zo_live_params(ctx) == th.data_ptr()
    ctx.close()


@pytest.mark.parametrize("M", [1, 129, 4096 + 3, 1 << 20])
def test_quad_loss_matches_oracle(zo, M):
    th_np, D_np = synth.quad_problem(M, seed=2)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=5)
    zo.zo_set_step(ctx, 2)
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    zo.zo_quad_loss(ctx, D, out[0:1])
    zo.zo_perturb(ctx, +1, 1e-3, 4)
    zo.zo_quad_loss(ctx, D, out[1:2])
    zo.zo_restore(ctx)
    zo.zo_perturb(ctx, -1, 1e-3, 4)
    zo.zo_quad_loss(ctx, D, out[2:3])
    zo.zo_quad_loss(ctx, D, out[2:3], accumulate=True)  # accumulate doubles it
    zo.zo_restore(ctx)
    got = out.cpu().numpy()
    ref0 = core.quad_loss(th_np, D_np)
    refp = core.quad_loss(core.perturb(th_np, 5, 2, 4, +1, 1e-3), D_np)
    refm = core.quad_loss(core.perturb(th_np, 5, 2, 4, -1, 1e-3), D_np)
    for g, r in ((got[0], ref0), (got[1], refp), (got[2], 2 * refm)):
        assert abs(g - r) <= 1e-12 * abs(r)
    ctx.close()


def test_quad_loss_is_deterministic(zo):
    th_np, D_np = synth.quad_problem(1 << 20, seed=3)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=1)
    out = torch.zeros(8, dtype=torch.float64, device="cuda")
    for k in range(8):
        zo.zo_perturb(ctx, +1, 1e-3, 1)
        zo.zo_quad_loss(ctx, D, out[k:k + 1])
        zo.zo_restore(ctx)
    v = out.cpu().numpy()
    assert (v == v[0]).all()
    ctx.close()


def test_mlp_loss_matches_oracle(zo):
    M = synth.mlp_param_count()
    P_np = synth.mlp_params(0)
    teacher = synth.mlp_params(0, tag="teacher")
    X_np, y_np = synth.mlp_batch(0, 0, teacher)
    th = dev(P_np)
    ctx = zo.zo_create(th, seed=0)
    zo.zo_set_live_buffer(ctx, True)
    X, y = dev(X_np), dev(y_np)
    out = torch.zeros(3, dtype=torch.float64, device="cuda")
    zo.zo_mlp_loss(ctx, X, y, 64, 64, 256, 10, 1.0 / 64, out[0:1])
    zo.zo_perturb(ctx, +1, 1e-3, 2)
    zo.zo_mlp_loss(ctx, X, y, 64, 64, 256, 10, 1.0 / 64, out[1:2])
    zo.zo_restore(ctx)
    # micro-batch accumulation: two halves with scale 1/64 each add up to the mean
    zo.zo_mlp_loss(ctx, X[:32], y[:32], 32, 64, 256, 10, 1.0 / 64, out[2:3])
    zo.zo_mlp_loss(ctx, X[32:], y[32:], 32, 64, 256, 10, 1.0 / 64, out[2:3], accumulate=True)
    got = out.cpu().numpy()
    ref0 = oracle.mlp.loss(P_np, X_np, y_np)
    refp = oracle.mlp.loss(core.perturb(P_np, 0, 0, 2, +1, 1e-3), X_np, y_np)
    assert abs(got[0] - ref0) <= 1e-5 * abs(ref0)
    assert abs(got[1] - refp) <= 1e-5 * abs(refp)
    assert abs(got[2] - ref0) <= 1e-5 * abs(ref0)
    assert M == ctx.M
    ctx.close()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,M", [(n, M) for n in (1, 7, 8, 13, 64, 160)
                                  for M in (1, 127, 129, 19210, (1 << 20) + 77)] +
                         # many chunks per CTA: the streaming ring wraps around several times
                         [(16, (1 << 24) + 77), (17, (1 << 24) + 3)] +
                         # every shared-memory plan: 32 or 16 table replicas beside a 4- or
                         # 3-stage ring, two CTAs per SM or one
                         [(32, (1 << 22) + 5), (40, (1 << 20) + 77)])
def test_update_bit_exact_vs_mirror_order(zo, M, n, dtype):
    th_np = _theta(M, dtype, seed=M + n)
    th = dev(th_np) if dtype == "f32" else bf16_dev(th_np)
    a = synth.coefficients(n, seed=n)
    ctx = zo.zo_create(th, seed=77)
    zo.zo_set_step(ctx, 9)
    zo.zo_update(ctx, dev(a), n)
    torch.cuda.synchronize()
    ref = core.update_mirror(th_np, a, 77, 9)
    got = host_bits(th)
    if dtype == "f32":
        assert (got.view(np.uint32) == ref.view(np.uint32)).all()
    else:
        assert (got == ref).all()
    assert zo.zo_get_step(ctx) == 9  # the update alone does not advance the step
    ctx.close()


@pytest.mark.parametrize("preconditioned", [True, False])
def test_step_from_given_losses(zo, preconditioned):
    """zo_step with synthetic losses: coefficients vs the oracle's fp64 preconditioner,
    theta' bit-exact vs the oracle's fixed order fed with those fp32 coefficients, and
    within the fp64 result's rounding bound."""
    M, n, eps, lr, lam = 50000, 32, 1e-3, 1e-2, 1e-3
    th_np = _theta(M, "f32", seed=4)
    th = dev(th_np)
    lp, lm, L0 = synth.losses(n, seed=11, eps=eps)
    ctx = zo.zo_create(th, seed=3)
    zo.zo_set_step(ctx, 6)
    dlp, dlm = dev(lp), dev(lm)
    dl0 = dev(np.array([L0])) if preconditioned else None
    zo.zo_step(ctx, dlp, dlm, n, dl0, lr, eps, lam)
    torch.cuda.synchronize()
    assert zo.zo_get_step(ctx) == 7
    g, c, w, a = zo.zo_get_precond(ctx, n)
    e32, lr32, lam32 = (float(np.float32(v)) for v in (eps, lr, lam))
    pc = core.precond(lp, lm, L0 if preconditioned else None, e32, lr32, lam32,
                      float(np.float32(0.1)))
    assert np.allclose(g, pc["g"], rtol=1e-13, atol=0)
    assert np.allclose(c, pc["c"], rtol=1e-12, atol=1e-9)
    assert np.allclose(w, pc["w"], rtol=1e-14, atol=0)
    a_ref = pc["a"].astype(np.float32)
    assert (np.abs(a.astype(np.float64) - a_ref) <= np.spacing(np.abs(a_ref))).all()
    got = th.cpu().numpy()
    mirror = core.update_mirror(th_np, a, 3, 6)  # oracle order, the GPU's fp32 coefficients
    assert (got.view(np.uint32) == mirror.view(np.uint32)).all()
    exact = core.update_f64(th_np, pc["a"], 3, 6)
    bound = (7 + (n + 7) // 8 + 1) * 2.0 ** -24 * np.abs(pc["a"]).sum() + np.spacing(np.abs(exact))
    assert (np.abs(got.astype(np.float64) - exact) <= bound).all()
    ctx.close()


def test_nonfinite_loss_skips_the_step(zo):
    M, n = 4096, 8
    th_np = _theta(M, "f32")
    th = dev(th_np)
    lp, lm, L0 = synth.losses(n, seed=1)
    lp[3] = np.nan
    ctx = zo.zo_create(th, seed=3)
    zo.zo_step(ctx, dev(lp), dev(lm), n, dev(np.array([L0])), 0.1, 1e-3, 1e-3)
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_sync(ctx)
    assert ei.value.status == zo.ZO_ERR_NONFINITE
    assert zo.zo_get_step(ctx) == 0
    assert (th.cpu().numpy().view(np.uint32) == th_np.view(np.uint32)).all()
    assert zo.zo_sync(ctx) == 0  # flags were cleared
    # an infinite clean loss is caught as well
    lp, lm, _ = synth.losses(n, seed=1)
    zo.zo_step(ctx, dev(lp), dev(lm), n, dev(np.array([np.inf])), 0.1, 1e-3, 1e-3)
    assert zo.zo_sync(ctx, raise_nonfinite=False) == zo.ZO_FLAG_NONFINITE
    ctx.close()


def test_state_machine_errors(zo):
    th = torch.zeros(1024, device="cuda")
    ctx = zo.zo_create(th)
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_restore(ctx)
    assert ei.value.status == zo.ZO_ERR_STATE
    zo.zo_perturb(ctx, 1, 1e-3, 0)
    for call in (lambda: zo.zo_perturb(ctx, 1, 1e-3, 1),
                 lambda: zo.zo_update(ctx, torch.zeros(4, device="cuda"), 4),
                 lambda: zo.zo_set_live_buffer(ctx, True)):
        with pytest.raises(zo.ZoError) as ei:
            call()
        assert ei.value.status == zo.ZO_ERR_STATE
    zo.zo_restore(ctx)
    for bad in ((0, 1e-3, 0), (1, 0.0, 0), (1, float("nan"), 0), (1, 1e-3, -1)):
        with pytest.raises(zo.ZoError) as ei:
            zo.zo_perturb(ctx, *bad)
        assert ei.value.status == zo.ZO_ERR_INVALID
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_update(ctx, torch.zeros(4, device="cuda"), zo.ZO_MAX_PROBES + 1)
    assert ei.value.status == zo.ZO_ERR_INVALID
    ctx.close()


@pytest.mark.parametrize("preconditioned", [True, False])
def test_quad_full_step_matches_oracle(zo, preconditioned):
    M, n, eps, lr, lam = 1 << 16, 16, 1e-3, 4e-7 * 64, 1e-3
    th_np, D_np = synth.quad_problem(M, seed=5)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=0)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_quad_step(ctx, D, n, eps, lr, lam, preconditioned, losses)
    torch.cuda.synchronize()
    nxt, rec = oracle.step.spsa_step(th_np, lambda P: core.quad_loss(P, D_np), n, eps, lr, lam,
                                     0, 0, preconditioned=preconditioned, update="mirror")
    L = losses.cpu().numpy()
    if preconditioned:
        assert abs(L[0] - rec["L0"]) <= 1e-12 * rec["L0"]
    assert np.allclose(L[1:n + 1], rec["Lp"], rtol=1e-12, atol=0)
    assert np.allclose(L[n + 1:], rec["Lm"], rtol=1e-12, atol=0)
    # losses agree to ~1e-13 relative, so g agrees to ~L*1e-13/eps; propagate to theta'
    dg = 4e-13 * np.abs(rec["Lp"]).max() / (2 * eps)
    da = float(np.float32(lr)) * 1.0 * dg  # w <= 1 here, 1/n cancels the sum over n
    got = th.cpu().numpy().astype(np.float64)
    bound = da + (9 + n) * 2.0 ** -24 * np.abs(rec["a"]).sum() + 2 * np.spacing(np.abs(nxt))
    assert (np.abs(got - nxt) <= bound).all()
    assert zo.zo_get_step(ctx) == 1
    ctx.close()


def test_mlp_full_step_matches_oracle(zo):
    n, eps, lr, lam = 16, 1e-3, 1e-2, 1e-3
    P_np = synth.mlp_params(0)
    teacher = synth.mlp_params(0, tag="teacher")
    X_np, y_np = synth.mlp_batch(0, 0, teacher)
    th = dev(P_np)
    ctx = zo.zo_create(th, seed=0)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_mlp_step(ctx, dev(X_np), dev(y_np), 64, 64, 256, 10, n, eps, lr, lam, True, losses)
    torch.cuda.synchronize()
    loss = lambda P: oracle.mlp.loss(P, X_np, y_np)  # noqa: E731
    nxt, rec = oracle.step.spsa_step(P_np, loss, n, eps, lr, lam, 0, 0)
    L = losses.cpu().numpy()
    ref = np.concatenate([[rec["L0"]], rec["Lp"], rec["Lm"]])
    assert np.allclose(L, ref, rtol=1e-5, atol=0)
    # Propagated bound: |dL| <= 1e-5 L per loss gives |dg_i| <= 1e-5 (L+ + L-)/(2 eps);
    # |dc_i| <= 1e-5 (L+ + L- + 2 L0)/eps^2 moves w_i by at most alpha*w_i*|dc_i|/(|c_i|+lam).
    dL = 1e-5 * ref.max()
    dg = 2 * dL / (2 * eps)
    dc = 4 * dL / eps ** 2
    dw = 0.1 * rec["w"] * dc / (np.abs(rec["c"]) + lam)
    da = float(np.float32(lr)) / n * (rec["w"] * dg + dw * np.abs(rec["g"]))
    got = th.cpu().numpy().astype(np.float64)
    bound = da.sum() + 4 * np.spacing(np.abs(nxt).astype(np.float32))
    assert (np.abs(got - nxt) <= bound).all()
    ctx.close()


def test_quad_full_size_sampled(zo):
    """The full diagonal-quadratic workload (M = 2^24, n = 64) in the launch configuration
    the benchmark times: a few losses in full against the oracle, theta' on sampled
    windows against the oracle's update fed with the oracle's coefficients."""
    M, n, eps, lr, lam = 1 << 24, 64, 1e-3, 4e-7, 1e-3
    th_np, D_np = synth.quad_problem(M, seed=0)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=0)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_quad_step(ctx, D, n, eps, lr, lam, True, losses)
    torch.cuda.synchronize()
    L = losses.cpu().numpy()
    ref0 = core.quad_loss(th_np, D_np)
    assert abs(L[0] - ref0) <= 1e-12 * ref0
    for i in (0, 63):
        for s, off in ((+1, 1), (-1, 1 + n)):
            r = core.quad_loss(core.perturb(th_np, 0, 0, i, s, eps), D_np)
            assert abs(L[off + i] - r) <= 1e-12 * r
    # the curvature of every probe is tr(D) (closed form) to the fp32 rounding of P
    g, c, w, a = zo.zo_get_precond(ctx, n)
    trD = float(D_np.astype(np.float64).sum())
    assert np.all(np.abs(c - trD) <= 1e-4 * trD)
    # theta' on windows, from the GPU's own losses via the oracle's precond + update
    e32 = float(np.float32(eps))
    pc = core.precond(L[1:n + 1], L[n + 1:], L[0], e32, float(np.float32(lr)),
                      float(np.float32(lam)), float(np.float32(0.1)))
    got = th.cpu().numpy()
    rng = np.random.default_rng(0)
    for start in list(rng.integers(0, M - 4096, 6)) + [0, M - 4096]:
        win = slice(int(start), int(start) + 4096)
        # the oracle's update of the window; probe bits follow the global index j0 + k
        ref = core.update_mirror(th_np[win], pc["a"].astype(np.float32), 0, 0, j0=int(start))
        assert (np.abs(got[win].astype(np.float64) - ref) <=
                2 * np.spacing(np.abs(ref)) + 4 * 2.0 ** -24 * np.abs(pc["a"]).sum()).all()
    ctx.close()


@pytest.mark.parametrize("M", [1, 5, 4096 + 3, 1 << 20, (1 << 22) + 17])
def test_quad_loss_pair_is_bit_identical_to_two_passes(zo, M):
    """zo_quad_loss_pair computes L(theta +- eps z) in one pass; each result must equal the
    corresponding single-sign pass bit for bit (same terms, same order), and the oracle."""
    th_np, D_np = synth.quad_problem(M, seed=12)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=4)
    zo.zo_set_step(ctx, 3)
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    zo.zo_quad_loss_pair(ctx, D, 9, 1e-3, out[0:1], out[1:2])
    zo.zo_perturb(ctx, +1, 1e-3, 9)
    zo.zo_quad_loss(ctx, D, out[2:3])
    zo.zo_restore(ctx)
    zo.zo_perturb(ctx, -1, 1e-3, 9)
    zo.zo_quad_loss(ctx, D, out[3:4])
    zo.zo_restore(ctx)
    v = out.cpu().numpy()
    assert v[0] == v[2] and v[1] == v[3]
    refp = core.quad_loss(core.perturb(th_np, 4, 3, 9, +1, 1e-3), D_np)
    refm = core.quad_loss(core.perturb(th_np, 4, 3, 9, -1, 1e-3), D_np)
    assert abs(v[0] - refp) <= 1e-12 * refp and abs(v[1] - refm) <= 1e-12 * refm
    with pytest.raises(zo.ZoError):  # needs the clean state
        zo.zo_perturb(ctx, +1, 1e-3, 0)
        try:
            zo.zo_quad_loss_pair(ctx, D, 0, 1e-3, out[0:1], out[1:2])
        finally:
            zo.zo_restore(ctx)
    ctx.close()


@pytest.mark.parametrize("M", [1, 7, 4096 * 3 + 5, 1 << 20, (1 << 22) + 17])
@pytest.mark.parametrize("first,count", [(0, 8), (16, 8), (8, 3), (0, 16), (24, 11), (0, 32),
                                         (8, 24), (16, 19), (0, 64), (8, 40), (0, 33)])
def test_quad_loss_octet_matches_pairs_and_oracle(zo, M, first, count):
    """zo_quad_loss_octet computes the 2*count losses of up to eight probe octets in one pass
    (each element's two perturbed values, each loss taking one per element; L- from the
    common sum of both terms): equal to the per-probe pair passes and to the oracle within
    fp64 rounding of sums of M terms (1e-12 relative), the clean loss from the same pass too.
    Outputs past count are left untouched."""
    th_np, D_np = synth.quad_problem(M, seed=13)
    th, D = dev(th_np), dev(D_np)
    ctx = zo.zo_create(th, seed=6)
    zo.zo_set_step(ctx, 2)
    oct_p = torch.full((65,), -7.0, dtype=torch.float64, device="cuda")
    oct_m = torch.full((65,), -7.0, dtype=torch.float64, device="cuda")
    clean = torch.zeros(2, dtype=torch.float64, device="cuda")
    zo.zo_quad_loss_octet(ctx, D, first, count, 1e-3, oct_p, oct_m, clean[0:1])
    zo.zo_quad_loss(ctx, D, clean[1:2])
    pair = torch.zeros((count, 2), dtype=torch.float64, device="cuda")
    for t in range(count):
        zo.zo_quad_loss_pair(ctx, D, first + t, 1e-3, pair[t, 0:1], pair[t, 1:2])
    assert zo.zo_sync(ctx) == 0
    P, Mn, pr = oct_p.cpu().numpy(), oct_m.cpu().numpy(), pair.cpu().numpy()
    assert np.allclose(P[:count], pr[:, 0], rtol=1e-13, atol=0)
    assert np.allclose(Mn[:count], pr[:, 1], rtol=1e-13, atol=0)
    assert (P[count:] == -7.0).all() and (Mn[count:] == -7.0).all()
    c = clean.cpu().numpy()
    assert abs(c[0] - c[1]) <= 1e-13 * c[1] and abs(c[0] - core.quad_loss(th_np, D_np)) <= 1e-12 * c[1]
    e32 = float(np.float32(1e-3))
    for t in range(count):
        refp = core.quad_loss(core.perturb(th_np, 6, 2, first + t, +1, e32), D_np)
        refm = core.quad_loss(core.perturb(th_np, 6, 2, first + t, -1, e32), D_np)
        assert abs(P[t] - refp) <= 1e-12 * refp and abs(Mn[t] - refm) <= 1e-12 * refm
    with pytest.raises(zo.ZoError):
        zo.zo_quad_loss_octet(ctx, D, 3, 8, 1e-3, oct_p, oct_m)  # not an octet boundary
    with pytest.raises(zo.ZoError):
        zo.zo_quad_loss_octet(ctx, D, 0, 65, 1e-3, oct_p, oct_m)  # more than eight octets
    ctx.close()


def test_pipelined_host_steps_equal_synchronous_steps(zo):
    """zo_quad_step_host_async (D copied on the context's copy stream into alternating
    staging slots, no synchronisation) gives the same theta, step counter and losses as
    the synchronous host-buffer step, bit for bit."""
    M, n = (1 << 16) + 5, 16
    th_np, D_np = synth.quad_problem(M, seed=21)
    D_pin = torch.from_numpy(D_np).pin_memory()
    a, b = dev(th_np), dev(th_np)
    ca, cb = zo.zo_create(a, seed=3), zo.zo_create(b, seed=3)
    La = torch.zeros((4, 2 * n + 1), dtype=torch.float64).pin_memory()
    Lb = torch.zeros((4, 2 * n + 1), dtype=torch.float64).pin_memory()
    for k in range(4):
        zo.zo_quad_step_host(ca, D_pin, n, 1e-3, 1e-5, 1e-3, True, La[k])
        zo.zo_quad_step_host_async(cb, D_pin, n, 1e-3, 1e-5, 1e-3, True, Lb[k])
    assert zo.zo_sync(cb) == 0 and zo.zo_sync(ca) == 0
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    assert torch.equal(La, Lb)
    assert zo.zo_get_step(ca) == zo.zo_get_step(cb) == 4
    ca.close()
    cb.close()
