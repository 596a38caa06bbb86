"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test names what it is pinned to: an independent implementation (NVIDIA cuRAND's
host Philox generator, numpy's IEEE fp32 arithmetic, torch's bf16 rounding and
autograd), a closed form of the method ("Stanford's 1.5-SPSA Trains OPT-30B Without
Backpropagation", sections "How 1.5-SPSA Works" and "Probe-Space Preconditioning"),
or brute-force enumeration on tiny inputs.
"""
import ctypes
import ctypes.util
import glob
import math
import os

import numpy as np
import pytest

import oracle
import synth
from oracle import core


# ------------------------------------------------------------------ Philox vs cuRAND

def _curand():
    cands = [ctypes.util.find_library("curand"), "/usr/local/cuda/lib64/libcurand.so"]
    try:
        import nvidia.curand  # noqa: F401  (torch's bundled copy)
        cands += glob.glob(os.path.join(os.path.dirname(nvidia.curand.__file__), "lib", "libcurand.so*"))
    except Exception:
        pass
    for c in cands:
        if c and os.path.exists(c) or (c and not c.startswith("/")):
            try:
                return ctypes.CDLL(c)
            except OSError:
                continue
    return None


CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161


def _curand_host_words(seed, nwords):
    cr = _curand()
    if cr is None:
        pytest.skip("libcurand not found")
    g = ctypes.c_void_p()
    assert cr.curandCreateGeneratorHost(ctypes.byref(g), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert cr.curandSetPseudoRandomGeneratorSeed(g, ctypes.c_ulonglong(seed)) == 0
        out = np.zeros(nwords, np.uint32)
        assert cr.curandGenerate(g, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(nwords)) == 0
    finally:
        cr.curandDestroyGenerator(g)
    return out.reshape(-1, 4)


@pytest.mark.parametrize("seed", [0, 0x123456789ABCDEF, 0xDEADBEEFCAFEF00D])
def test_philox_matches_curand_host_generator(seed):
    """cuRAND's host Philox4x32-10 emits block k = Philox(counter = (k // 65536, 0,
    k % 65536, 0), key = (seed lo, seed hi)): an independent implementation of the
    published generator, covering the round function, constants, key schedule and
    counter words 0 and 2."""
    blocks = _curand_host_words(seed, 4 * 70000)
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for k in list(range(0, 64)) + [4095, 4096, 65535, 65536, 65537, 69999]:
        ref = blocks[k]
        got = core.philox4x32_10([k // 65536, 0, k % 65536, 0], key)
        assert (got == ref).all(), (k, got, ref)


def test_philox_counter_words_1_and_3_matter():
    """Every counter word and both key words change the output (no ignored input)."""
    base = core.philox4x32_10([5, 6, 7, 8], [9, 10])
    for w in range(4):
        c = [5, 6, 7, 8]
        c[w] ^= 1
        assert not (core.philox4x32_10(c, [9, 10]) == base).all()
    for w in range(2):
        k = [9, 10]
        k[w] ^= 1
        assert not (core.philox4x32_10([5, 6, 7, 8], k) == base).all()


# ------------------------------------------------------------------ probe layout and statistics

def test_sign_layout_from_raw_philox_blocks():
    """Element j, probe i: bit (i & 7) of byte (j & 15) of the little-endian 16-byte Philox
    block with counter (j >> 4, 0, i >> 3, step); rebuilt here from raw blocks by numpy's
    byte view, and the packed form of one probe holds element 8q + t in bit t of byte q."""
    seed, step, M = 0xABCDEF0123, 7, 16 * 9 + 13
    key = [seed & 0xFFFFFFFF, seed >> 32]
    groups = (M + 15) // 16
    for probe in (0, 5, 8, 13, 70):
        raw = np.concatenate([core.philox4x32_10([g, 0, probe >> 3, step], key)
                              for g in range(groups)])
        byte = raw.astype("<u4").view(np.uint8)[:M]
        bits = (byte >> (probe & 7)) & 1
        packed = core.pack_probe(seed, step, probe, M)
        assert (np.unpackbits(packed, bitorder="little")[:M] == bits).all()
        assert not np.unpackbits(packed, bitorder="little")[M:].any()  # padding bits are 0
        for j in [0, 1, 3, 4, 15, 16, 17, M - 1]:
            assert core.probe_sign(seed, step, probe, j) == (-1 if bits[j] else 1)
    # the 8 probes of an octet share one block: byte j of that block is element j's signs
    raw = core.philox4x32_10([2, 0, 1, step], key).astype("<u4").view(np.uint8)
    for t in range(8):
        z = [core.probe_sign(seed, step, 8 + t, 32 + b) for b in range(16)]
        assert z == [-1 if (raw[b] >> t) & 1 else 1 for b in range(16)]


def test_probe_statistics():
    """Rademacher balance and independence (the pages' probes are i.i.d. +/-1)."""
    M, n = 1 << 16, 16
    Z = np.stack([core.probe_signs(3, 11, i, M) for i in range(n)]).astype(np.int64)
    sigma = math.sqrt(M)
    for i in range(n):
        assert abs(Z[i].sum()) < 5 * sigma  # sum of M +/-1 has std sqrt(M)
        for k in range(i + 1, n):
            assert abs((Z[i] * Z[k]).sum()) < 5 * sigma  # agreement rate 1/2
    # per byte position within the 16-element group, for every bit position of the octet
    pos = Z[:, : M - M % 16].reshape(n, -1, 16).sum(axis=1)  # [probe][byte position]
    assert np.abs(pos).max() < 5 * math.sqrt(M / 16) * 1.2
    # different steps give independent probes
    Z2 = core.probe_signs(3, 12, 0, M).astype(np.int64)
    assert abs((Z[0] * Z2).sum()) < 5 * sigma
    # no repeated probe across (step, probe) pairs on a 128-bit window
    seen = set()
    for s in range(40):
        for i in range(40):
            seen.add(core.pack_probe(3, s, i, 128).tobytes())
    assert len(seen) == 1600


# ------------------------------------------------------------------ perturbation

def _theta_f32(M, seed=1):
    r = np.random.default_rng(seed)
    t = r.standard_normal(M).astype(np.float32)
    t[:8] = [0.0, -0.0, 1e-40, -1e-40, 1.0, -1.0, 3.0e38, 2.0 ** -20]
    return t


def test_perturb_f32_matches_numpy_ieee_add():
    """P = theta + s*eps*z as one IEEE fp32 add (numpy float32 arithmetic)."""
    M = 5000
    th = _theta_f32(M)
    for sign in (+1, -1):
        for eps in (1e-3, 0.37, 2.0 ** -24):
            P = core.perturb(th, 9, 2, 4, sign, eps)
            z = core.probe_signs(9, 2, 4, M).astype(np.float32)
            ref = th + np.float32(sign) * np.float32(eps) * z
            assert P.view(np.uint32).tolist() == ref.view(np.uint32).tolist()


def test_perturb_bf16_matches_torch_rounding():
    """bf16: widen, add in fp32, round-to-nearest-even back to bf16 (torch's rounding)."""
    import torch
    M = 4096
    r = np.random.default_rng(2)
    base = (r.standard_normal(M) * 0.02).astype(np.float32)
    base[:6] = [0.0, 1.0, -1.0, 1e-3, 3.0e-6, 0.0078125]
    th = torch.from_numpy(base).to(torch.bfloat16)
    bits = th.view(torch.int16).numpy().view(np.uint16)
    for sign in (+1, -1):
        P = core.perturb(bits, 1, 0, 3, sign, 1e-3)
        z = core.probe_signs(1, 0, 3, M).astype(np.float32)
        s32 = th.float().numpy() + np.float32(sign) * np.float32(1e-3) * z
        ref = torch.from_numpy(s32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert (P == ref).all()
    # the oracle's own fp32->bf16 rounding agrees with torch on ties and specials
    vals = np.array([1.00390625, 1.01171875, -1.00390625, 65504.0, 1e-40, 3.4e38], np.float32)
    assert (core.f32_to_bf16(vals) ==
            torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)).all()


def test_perturbation_leaves_theta_untouched():
    """Restore is exact: the oracle never writes theta when perturbing."""
    th = _theta_f32(3000)
    before = th.tobytes()
    core.perturb(th, 0, 0, 0, +1, 1e-3)
    core.perturb(th, 0, 0, 0, -1, 1e-3)
    assert th.tobytes() == before


# ------------------------------------------------------------------ quadratic closed forms

def test_quadratic_loss_vs_correctly_rounded_sum():
    _, D = synth.quad_problem(20000, seed=4)
    P = np.random.default_rng(5).standard_normal(20000).astype(np.float32)
    terms = [0.5 * float(d) * float(p) * float(p) for d, p in zip(D, P)]
    exact = math.fsum(terms)
    got = core.quad_loss(P, D)
    assert abs(got - exact) <= 20000 * 2.0 ** -53 * math.fsum(abs(t) for t in terms)


def _dyadic_quadratic(M, seed):
    """theta on a 2^-10 grid and eps = 2^-10, so theta +/- eps is exact in fp32."""
    r = np.random.default_rng(seed)
    th = (np.round(r.standard_normal(M) * 1024) / 1024).astype(np.float32)
    D = (10.0 ** r.uniform(-3, 3, M)).astype(np.float32)
    return th, D, 2.0 ** -10


def test_quadratic_curvature_is_trace_for_every_probe():
    """z^T D z = tr(D) for every Rademacher z, so c_i = tr(D) and g_i = z_i^T D theta
    (the closed forms of the diagonal quadratic)."""
    M, n = 4096, 12
    th, D, eps = _dyadic_quadratic(M, 6)
    # theta = 0: L(+-eps z) = eps^2/2 * tr(D) exactly (up to the fp64 sum)
    zero = np.zeros(M, np.float32)
    trD = math.fsum(float(d) for d in D)
    for i in range(4):
        L = core.quad_loss(core.perturb(zero, 8, 0, i, +1, eps), D)
        assert abs(L - 0.5 * eps * eps * trD) <= 1e-12 * L
    loss = lambda P: core.quad_loss(P, D)  # noqa: E731
    _, rec = oracle.step.spsa_step(th, loss, n, eps, 1.0, 1e-3, 8, 3)
    for i in range(n):
        z = core.probe_signs(8, 3, i, M).astype(np.float64)
        gz = float(np.dot(z, D.astype(np.float64) * th.astype(np.float64)))
        assert abs(rec["g"][i] - gz) <= 1e-9 * (abs(gz) + trD)
        assert abs(rec["c"][i] - trD) <= 1e-7 * trD


def test_quadratic_step_closed_form():
    """On the diagonal quadratic, w_i = (tr D + lambda)^(-alpha) for all i, and the step
    is theta' = theta - lr*w*(1/n) * sum_i (z_i^T D theta) z_i."""
    M, n, lr, lam = 2048, 8, 1e-5, 1e-3
    th, D, eps = _dyadic_quadratic(M, 7)
    loss = lambda P: core.quad_loss(P, D)  # noqa: E731
    nxt, rec = oracle.step.spsa_step(th, loss, n, eps, lr, lam, 1, 0)
    trD = float(D.astype(np.float64).sum())
    w = (trD + float(np.float32(lam))) ** -float(np.float32(0.1))
    assert np.allclose(rec["w"], w, rtol=1e-9)
    Z = np.stack([core.probe_signs(1, 0, i, M) for i in range(n)]).astype(np.float64)
    gz = Z @ (D.astype(np.float64) * th)
    step = float(np.float32(lr)) * w / n * (Z.T @ gz)
    ref = (th.astype(np.float64) - step).astype(np.float32)
    ulp = np.spacing(np.abs(ref)).astype(np.float64)
    assert (np.abs(nxt.astype(np.float64) - ref) <= ulp).all()


# ------------------------------------------------------------------ preconditioner

def test_precond_recovers_difference_quotients_and_downweights_curvature():
    eps = 1e-3
    lp, lm, L0 = synth.losses(64, seed=3, eps=eps)
    pc = core.precond(lp, lm, L0, eps, 0.5, 1e-3)
    # L+- = L0 +- eps g + eps^2 c/2  =>  the quotients return g and c (fp64 cancellation)
    r = synth.rng(3, "loss", 64)
    g = r.standard_normal(64)
    assert np.allclose(pc["g"], g, atol=1e-9)
    order = np.argsort(np.abs(pc["c"]))
    assert (np.diff(pc["w"][order]) <= 0).all()  # higher curvature -> smaller weight
    assert np.allclose(pc["a"], 0.5 * pc["w"] * pc["g"] / 64)
    # 1SPSA: no clean loss, unit weights, a = lr * g / n
    p1 = core.precond(lp, lm, None, eps, 0.5, 1e-3)
    assert (p1["w"] == 1.0).all() and np.allclose(p1["a"], 0.5 * p1["g"] / 64)
    # alpha = 0 turns the preconditioner off; huge damping flattens it
    p0 = core.precond(lp, lm, L0, eps, 0.5, 1e-3, alpha=0.0)
    assert (p0["w"] == 1.0).all()
    pd = core.precond(lp, lm, L0, eps, 0.5, 1e12)
    assert np.allclose(pd["w"], 1e12 ** -0.1, rtol=1e-9)
    # non-finite losses are rejected
    bad = lp.copy()
    bad[5] = np.nan
    assert core.precond(bad, lm, L0, eps, 0.5, 1e-3) is None
    assert core.precond(lp, lm, float("inf"), eps, 0.5, 1e-3) is None


# ------------------------------------------------------------------ update

@pytest.mark.parametrize("n", [1, 7, 8, 13, 64])
def test_update_matches_dense_matvec(n):
    """theta' = rd(theta - Z^T a): numpy's fp64 matrix-vector product on unpacked probes."""
    M, seed, step = 3000, 21, 4
    th = _theta_f32(M)[8:]
    M = th.size
    a = synth.coefficients(n, seed=n).astype(np.float64)
    Z = np.stack([core.probe_signs(seed, step, i, M) for i in range(n)]).astype(np.float64)
    ref = (th.astype(np.float64) - Z.T @ a).astype(np.float32)
    got = core.update_f64(th, a, seed, step)
    ulp = np.spacing(np.abs(ref)).astype(np.float64)
    assert (np.abs(got.astype(np.float64) - ref) <= ulp).all()
    # the fixed fp32 order stays within its rounding bound of the fp64 result
    mir = core.update_mirror(th, a.astype(np.float32), seed, step)
    bound = (7 + (n + 7) // 8) * 2.0 ** -24 * np.abs(a).sum() + 2 * ulp
    assert (np.abs(mir.astype(np.float64) - ref) <= bound + 1e-12).all()


def test_update_bf16_within_one_ulp_of_dense():
    import torch
    M, n = 2048, 16
    r = np.random.default_rng(8)
    th = torch.from_numpy((r.standard_normal(M) * 0.02).astype(np.float32)).to(torch.bfloat16)
    bits = th.view(torch.int16).numpy().view(np.uint16)
    a = (r.standard_normal(n) * 1e-3).astype(np.float64)
    Z = np.stack([core.probe_signs(2, 1, i, M) for i in range(n)]).astype(np.float64)
    exact = th.double().numpy() - Z.T @ a
    ref = torch.from_numpy(exact).to(torch.bfloat16).float().numpy()
    got = core.bf16_to_f32(core.update_f64(bits, a, 2, 1))
    ulp = np.spacing(np.abs(ref).astype(np.float32)) * 65536
    assert (np.abs(got - ref) <= ulp).all()


# ------------------------------------------------------------------ estimator (exact and Monte Carlo)

def test_rademacher_identity_by_enumeration():
    """Average over all 2^M sign vectors of (z^T v) z equals v (M = 10): the identity that
    makes the projected difference times z an unbiased gradient estimate."""
    M = 10
    v = np.random.default_rng(0).standard_normal(M)
    acc = np.zeros(M)
    for code in range(1 << M):
        z = 1.0 - 2.0 * ((code >> np.arange(M)) & 1)
        acc += np.dot(z, v) * z
    assert np.allclose(acc / (1 << M), v, atol=1e-12)


def test_mlp_loss_matches_torch_and_estimator_matches_autograd():
    """MLP loss against torch's own layers in fp64; then, enumerating every z for a tiny
    MLP (2 -> 2 -> 2, M = 12), mean_z g(z) z reproduces torch autograd's gradient to O(eps^2)."""
    import torch
    import torch.nn.functional as F
    n_in, n_h, n_out, B = 2, 2, 2, 5
    M = synth.mlp_param_count(n_in, n_h, n_out)
    assert M == 12
    r = np.random.default_rng(3)
    P = r.standard_normal(M) * 0.7
    X = r.standard_normal((B, n_in))
    y = np.array([0, 1, 1, 0, 1])
    got = oracle.mlp.loss(P, X, y, n_in, n_h, n_out)
    Pt = torch.tensor(P, dtype=torch.float64, requires_grad=True)
    W1 = Pt[:4].view(2, 2); b1 = Pt[4:6]; W2 = Pt[6:10].view(2, 2); b2 = Pt[10:12]
    out = F.linear(F.relu(F.linear(torch.tensor(X), W1, b1)), W2, b2)
    ref = F.cross_entropy(out, torch.tensor(y))
    assert abs(got - ref.item()) < 1e-13
    ref.backward()
    grad = Pt.grad.numpy()
    eps = 1e-4
    acc = np.zeros(M)
    for code in range(1 << M):
        z = 1.0 - 2.0 * ((code >> np.arange(M)) & 1)
        g = (oracle.mlp.loss(P + eps * z, X, y, n_in, n_h, n_out)
             - oracle.mlp.loss(P - eps * z, X, y, n_in, n_h, n_out)) / (2 * eps)
        acc += g * z
    assert np.allclose(acc / (1 << M), grad, atol=1e-7)


def test_estimator_mean_and_variance_law():
    """With exact directional derivatives (a linear loss L = v^T theta, so g_i = z_i^T v),
    the estimator mean is v and E||ghat - v||^2 = (M - 1)/n ||v||^2 (the pages' M/n_pert
    variance law, exact for Rademacher probes)."""
    M, n, trials = 24, 4, 3000
    v = np.random.default_rng(1).standard_normal(M)
    errs = np.zeros(trials)
    mean = np.zeros(M)
    for t in range(trials):
        Z = np.stack([core.probe_signs(77, t, i, M) for i in range(n)]).astype(np.float64)
        ghat = (Z @ v) @ Z / n
        mean += ghat
        errs[t] = np.sum((ghat - v) ** 2)
    mean /= trials
    expect = (M - 1) / n * np.dot(v, v)
    assert abs(errs.mean() - expect) < 5 * errs.std() / math.sqrt(trials)
    assert np.all(np.abs(mean - v) < 5 * math.sqrt(expect / M / trials) * 2)
