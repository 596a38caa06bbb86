"""Parity of the decoder forward (tcgen05 GEMM, attention, LayerNorm, embedding, head) with
the CPU oracle and with plain numpy references of each component.

Tolerances:
  - GEMM, bf16 output: |gpu - ref| <= 2^-8 |ref| + 2^-8 * rms(ref) (one bf16 rounding of
    an fp32-accumulated dot product); fp32 residual output: 1e-5 of sum |a_k b_k|;
  - attention (bf16 probabilities and output): 2e-2 absolute on unit-scale inputs;
  - LayerNorm (bf16 output): 2^-8 relative + 1e-3 absolute;
  - decoder hidden states: relative Frobenius error <= 1e-2 per layer;
  - decoder loss (bf16 forward): 2e-2 relative.
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import core

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).cuda()


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.fixture(scope="module")
def ctx(zo):
    th = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    c = zo.zo_create(th, seed=0)
    yield c
    c.close()


GEMM_SHAPES = [(128, 128, 64), (256, 384, 256), (300, 200, 72), (129, 136, 8),
               (2048, 2560, 512), (4096, 768, 768),
               # at least 148 tiles of 256 x 256: the CTA-pair kernel (cta_group::2), also
               # with M, N and K off the tile grid
               (4096, 2560, 512), (4000, 2600, 520), (2304, 4352, 1024)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("epi", [0, 1, 2])
def test_gemm_matches_numpy(zo, ctx, M, N, K, epi):
    r = np.random.default_rng(M * 7 + N * 3 + K + epi)
    A = bf16(r.standard_normal((M, K)))
    B = bf16(r.standard_normal((N, K)) * 0.05)
    bias = bf16(r.standard_normal(N))
    ref = f64(A) @ f64(B).T + f64(bias)
    if epi == 2:
        h0 = torch.from_numpy(r.standard_normal((M, N)).astype(np.float32)).cuda()
        out = h0.clone()
    else:
        out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    zo.zo_gemm_bf16(ctx, A, B, bias, out, M, N, K, N, epi)
    torch.cuda.synchronize()
    assert zo.zo_sync(ctx) == 0
    if epi == 2:
        scale = np.abs(f64(A)) @ np.abs(f64(B)).T + np.abs(f64(bias))
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - (h0.cpu().numpy() + ref)) <= 1e-5 * (scale + 1) + 1e-6)
    else:
        if epi == 1:
            ref = np.maximum(ref, 0.0)
        got = f64(out)
        rms = np.sqrt(np.mean(ref ** 2)) + 1e-30
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * (np.abs(ref) + rms))


def _np_attention(qkv, B, S, H, d):
    hd = d // H
    x = qkv.reshape(B, S, 3, H, hd)
    q, k, v = (x[:, :, i].transpose(0, 2, 1, 3) for i in range(3))
    s = q @ k.transpose(0, 1, 3, 2) / np.sqrt(hd)
    s = np.where(np.triu(np.ones((S, S), bool), 1), -np.inf, s)
    w = np.exp(s - s.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    return (w @ v).transpose(0, 2, 1, 3).reshape(B * S, d)


@pytest.mark.parametrize("B,S,H,d", [(2, 64, 2, 128), (2, 200, 2, 256), (1, 256, 4, 256),
                                     (3, 130, 3, 192), (1, 512, 1, 128)])
def test_attention_matches_numpy(zo, ctx, B, S, H, d):
    r = np.random.default_rng(S + d)
    qkv = bf16(r.standard_normal((B * S, 3 * d)))
    out = torch.zeros((B * S, d), dtype=torch.bfloat16, device="cuda")
    zo.zo_attention(ctx, qkv, out, B, S, H, d)
    torch.cuda.synchronize()
    assert zo.zo_sync(ctx) == 0  # no bounded wait expired
    ref = _np_attention(f64(qkv), B, S, H, d)
    assert np.max(np.abs(f64(out) - ref)) <= 2e-2


@pytest.mark.parametrize("B,S,H,d", [(2, 300, 2, 256), (1, 256, 2, 128)])
def test_attention_rescaling_matches_numpy(zo, ctx, B, S, H, d):
    """Scores that grow along the keys (k_j = mean(q) * j / 2 plus noise: about 2^16 from one
    64-key tile to the next), so that the running maximum grows by more than 2^8 at every tile
    and the softmax rescales O and the row sum each time (after waiting for the previous
    tile's P V)."""
    r = np.random.default_rng(S + d + 7)
    hd = d // H
    q = np.ones((B, S, H, hd)) * 2.0 / np.sqrt(hd) + 0.1 * r.standard_normal((B, S, H, hd))
    k = q.mean(axis=1, keepdims=True) * (np.arange(S)[None, :, None, None] / 2.0) \
        + 0.1 * r.standard_normal((B, S, H, hd))
    v = r.standard_normal((B, S, H, hd))
    qkv = bf16(np.stack([q, k, v], axis=2).reshape(B * S, 3 * d))
    out = torch.zeros((B * S, d), dtype=torch.bfloat16, device="cuda")
    zo.zo_attention(ctx, qkv, out, B, S, H, d)
    torch.cuda.synchronize()
    assert zo.zo_sync(ctx) == 0
    ref = _np_attention(f64(qkv), B, S, H, d)
    assert np.max(np.abs(f64(out) - ref)) <= 2e-2


# rows of whole and ragged last warps (8 columns per thread), up to the 8192-column limit
@pytest.mark.parametrize("d", [7168, 8192, 2064, 2056, 768])
def test_layernorm_matches_numpy(zo, ctx, d):
    r = np.random.default_rng(d)
    rows = 37
    x = torch.from_numpy((r.standard_normal((rows, d)) * 3 + 1).astype(np.float32)).cuda()
    g = bf16(1 + 0.1 * r.standard_normal(d))
    b = bf16(0.1 * r.standard_normal(d))
    out = torch.zeros((rows, d), dtype=torch.bfloat16, device="cuda")
    zo.zo_layernorm(ctx, x, g, b, out, rows, d)
    torch.cuda.synchronize()
    xx = x.cpu().numpy().astype(np.float64)
    ref = (xx - xx.mean(1, keepdims=True)) / np.sqrt(xx.var(1, keepdims=True) + 1e-5) * f64(g) + f64(b)
    assert np.all(np.abs(f64(out) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3)


# the perturbation fused into the GEMM's operand path: narrow (128-column) and wide
# (256-column) tiles, ragged M and N, K off the 64-column stage grid, all three epilogues
@pytest.mark.parametrize("M,N,K,epi,j0", [(300, 320, 144, 0, 0), (1024, 1536, 512, 1, 0),
                                          (4096, 1024, 272, 2, 0), (4100, 2048, 2048, 0, 0),
                                          # a context over a slice: signs of global indices
                                          (512, 384, 320, 1, (1 << 20) + 48)])
@pytest.mark.parametrize("sign", [+1, -1])
def test_fused_perturbation_gemm_equals_the_window_product(zo, M, N, K, epi, j0, sign):
    """zo_gemm_bf16_perturbed (signs regenerated per weight tile in shared memory) against the
    same single-CTA kernel run clean on the zo_perturb_range window: bit for bit; the window
    itself against the oracle's perturbation, bit for bit."""
    r = np.random.default_rng(M + N + K + epi)
    w_off, eps, probe, seed, step = 48, 1e-3, 13, 21, 5
    total = w_off + N * K + 40
    theta = bf16(r.standard_normal(total) * 0.02)
    A = bf16(r.standard_normal((M, K)))
    bias = bf16(r.standard_normal(N) * 0.1)
    if epi == 2:
        h0 = torch.from_numpy(r.standard_normal((M, N)).astype(np.float32)).cuda()
        out1, out2 = h0.clone(), h0.clone()
    else:
        out1 = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
        out2 = torch.zeros_like(out1)
    c = zo.zo_create(theta, seed=seed)
    if j0:
        zo.zo_set_element_offset(c, j0)
    zo.zo_set_step(c, step)
    zo.zo_perturb(c, sign, eps, probe)
    zo.zo_gemm_bf16_perturbed(c, A, w_off, bias, out1, M, N, K, N, epi)
    win = torch.empty(N * K, dtype=torch.bfloat16, device="cuda")
    zo.zo_perturb_range(c, w_off, N * K, win)
    zo.zo_restore(c)
    cw = zo.zo_create(win, seed=seed)  # clean: the same kernel form on the window
    zo.zo_gemm_bf16_perturbed(cw, A, 0, bias, out2, M, N, K, N, epi)
    torch.cuda.synchronize()
    assert zo.zo_sync(c) == 0 and zo.zo_sync(cw) == 0
    bits = theta.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_win = core.perturb(bits, seed, step, probe, sign, float(np.float32(eps)), j0)[w_off:w_off + N * K]
    assert np.array_equal(win.view(torch.int16).cpu().numpy().view(np.uint16), ref_win)
    if epi == 2:
        assert torch.equal(out1, out2)
    else:
        assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    # and the product itself, against fp64 on the window
    ref = f64(A) @ f64(win.reshape(N, K)).T + f64(bias)
    if epi == 2:
        scale = np.abs(f64(A)) @ np.abs(f64(win.reshape(N, K))).T + np.abs(f64(bias))
        got = out1.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - (h0.cpu().numpy() + ref)) <= 1e-5 * (scale + 1) + 1e-6)
    else:
        if epi == 1:
            ref = np.maximum(ref, 0.0)
        rms = np.sqrt(np.mean(ref ** 2)) + 1e-30  # one bf16 rounding of the output
        assert np.all(np.abs(f64(out1) - ref) <= 2.0 ** -8 * (np.abs(ref) + rms))
    cw.close()
    c.close()


def test_fused_perturbation_gemm_rejects_bad_arguments(zo):
    theta = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((64, 32), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    c = zo.zo_create(theta, seed=1)
    for w_off, N, K, epi in [(8, 64, 32, 0),      # offset not 16-element aligned
                             (0, 64, 24, 0),      # K % 16 != 0
                             (2048, 64, 64, 0),   # past the end of the context
                             (0, 32, 32, 3)]:     # SwiGLU
        with pytest.raises(zo.ZoError):
            zo.zo_gemm_bf16_perturbed(c, A, w_off, None, out, 64, N, K, 64, epi)
    c.close()
    f = zo.zo_create(torch.zeros(4096, dtype=torch.float32, device="cuda"), seed=1)
    with pytest.raises(zo.ZoError):  # fp32 context
        zo.zo_gemm_bf16_perturbed(f, A, 0, None, out, 64, 64, 32, 64, 0)
    f.close()


TINY = [
    dict(n_layers=2, d_model=128, n_heads=2, d_ffn=512, vocab=1000, max_pos=128, class_ids=(3, 7)),
    dict(n_layers=2, d_model=256, n_heads=2, d_ffn=320, vocab=777, max_pos=160, class_ids=(0, 776)),
]


def _setup(zo, cfg, B, S, seed=0, max_tokens=None):
    bits = synth.opt_params(cfg, seed=seed, varied=True)
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=seed)
    model = zo.zo_model_create(ctx, cfg, max_tokens or B * S)
    tokens, labels = synth.opt_batch(cfg, B, S, seed=seed)
    return bits, theta, ctx, model, tokens, labels


def _rel_fro(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("cfg", TINY)
@pytest.mark.parametrize("B,S", [(3, 100), (2, 128)])
def test_decoder_hidden_states_and_loss(zo, cfg, B, S):
    bits, theta, ctx, model, tokens, labels = _setup(zo, cfg, B, S)
    dtok = torch.from_numpy(tokens).cuda()
    dlab = torch.from_numpy(labels).cuda()
    d = cfg["d_model"]
    for sign, probe in ((0, 0), (+1, 3), (-1, 3)):
        if sign:
            zo.zo_perturb(ctx, sign, 1e-3, probe)
            P = core.bf16_to_f32(core.perturb(bits, 0, 0, probe, sign, 1e-3)).astype(np.float64)
        else:
            P = core.bf16_to_f32(bits).astype(np.float64)
        for n_run in range(cfg["n_layers"] + 1):
            h = torch.zeros((B * S, d), dtype=torch.float32, device="cuda")
            zo.zo_model_hidden(model, dtok, B, S, n_run, h)
            torch.cuda.synchronize()
            ref = oracle.opt.hidden_states(P, cfg, tokens, n_layers=n_run).reshape(B * S, d)
            assert _rel_fro(h.cpu().numpy().astype(np.float64), ref) <= 1e-2, (sign, n_run)
        out = torch.zeros(1, dtype=torch.float64, device="cuda")
        zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out)
        torch.cuda.synchronize()
        ref = oracle.opt.loss(P, cfg, tokens, labels)
        assert abs(out.item() - ref) <= 2e-2 * abs(ref), (sign, out.item(), ref)
        if sign:
            zo.zo_restore(ctx)
    assert zo.zo_sync(ctx) == 0
    model.close()
    ctx.close()


def test_decoder_rejects_bad_tokens_without_reading_out_of_range(zo):
    cfg = TINY[0]
    bits, theta, ctx, model, tokens, labels = _setup(zo, cfg, 2, 64)
    tokens[1, 5] = cfg["vocab"] + 10
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    zo.zo_model_loss(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                     2, 64, 0.5, out)
    torch.cuda.synchronize()
    assert np.isnan(out.item())
    with pytest.raises(zo.ZoError):  # longer than the position table
        zo.zo_model_loss(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                         1, cfg["max_pos"] + 1, 1.0, out)
    model.close()
    ctx.close()


def _teacher_forced(bits, L, n, eps, lr, lam, seed, step=0):
    """The oracle's preconditioner and fixed-order update fed with the given losses
    [L0, L+..., L-...] (the GPU's): (theta', precond record)."""
    e32 = float(np.float32(eps))
    pc = core.precond(L[1:1 + n], L[1 + n:], L[0], e32, float(np.float32(lr)),
                      float(np.float32(lam)), float(np.float32(0.1)))
    return core.update_mirror(bits, pc["a"].astype(np.float32), seed, step), pc


def _run_step(zo, cfg, bits, tokens, labels, B, S, k, n, eps, lr, lam, seed):
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=seed)
    model = zo.zo_model_create(ctx, cfg, B * S)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_model_step(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                     B, S, k, n, eps, lr, lam, True, losses)
    assert zo.zo_sync(ctx) == 0
    assert zo.zo_get_step(ctx) == 1
    g, c, w, a = zo.zo_get_precond(ctx, n)
    out = (theta.view(torch.int16).cpu().numpy().view(np.uint16), losses.cpu().numpy(), (g, c, w, a))
    model.close()
    ctx.close()
    return out


def test_decoder_step_matches_oracle(zo):
    """One 1.5-SPSA step with 2 micro-batches.  The losses match the oracle's within the bf16
    forward's tolerance (2e-2), and, fed the GPU's own losses (teacher forcing), the oracle's
    preconditioner gives the GPU's g, c, w, a and its fixed-order update gives the GPU's
    theta' bit for bit: the step's arithmetic after the losses is exact, so any error in
    the perturbation, the probe signs or the update shows up as a mismatch."""
    cfg = TINY[0]
    B, S, n_micro, n, eps, lr, lam = 2, 64, 2, 4, 1e-3, 2e-2, 1e-3
    bits = synth.opt_params(cfg, seed=1, varied=True)
    toks, labs = zip(*(synth.opt_batch(cfg, B, S, seed=1, step=k) for k in range(n_micro)))
    tokens, labels = np.stack(toks), np.stack(labs)
    got, L, (g, c, w, a) = _run_step(zo, cfg, bits, tokens, labels, B, S, n_micro, n, eps, lr,
                                     lam, 1)
    flat_t, flat_l = tokens.reshape(-1, S), labels.reshape(-1)
    loss = lambda Pb: oracle.opt.loss(core.bf16_to_f32(Pb), cfg, flat_t, flat_l)  # noqa: E731
    _, rec = oracle.step.spsa_step(bits, loss, n, eps, lr, lam, 1, 0)
    ref = np.concatenate([[rec["L0"]], rec["Lp"], rec["Lm"]])
    assert np.allclose(L, ref, rtol=2e-2, atol=0)
    nxt, pc = _teacher_forced(bits, L, n, eps, lr, lam, 1)
    assert np.array_equal(got, nxt)
    assert np.allclose(g, pc["g"], rtol=1e-13, atol=0)
    assert np.allclose(c, pc["c"], rtol=1e-12, atol=1e-6)
    assert np.allclose(w, pc["w"], rtol=1e-13, atol=0)
    assert np.array_equal(a, pc["a"].astype(np.float32))
    assert not np.array_equal(got, bits)  # the step moved theta


def test_probe_quantities_match_oracle(zo):
    """The per-probe quantities the method consumes, as the library's preconditioner computes
    them from its own losses (zo_get_precond), against the oracle's from its fp64 losses:
    at the method's eps = 1e-3 every g_i = (L+ - L-)/(2 eps) with the oracle's sign and within
    G_TOL; at eps = 1e-2, where the curvature is above the forward's rounding, every
    c_i = (L+ + L- - 2 L0)/eps^2 within C_REL_TOL of the largest and every weight
    w_i = (|c_i| + damping)^-0.1 within W_REL_TOL (tests/probe_tolerances.py)."""
    from probe_tolerances import C_REL_TOL, G_TOL, W_REL_TOL
    cfg = TINY[0]
    B, S, n, lam = 4, 64, 8, 1e-3
    bits = synth.opt_params(cfg, seed=1, varied=True)
    tokens, labels = synth.opt_batch(cfg, B, S, seed=1)
    lf = lambda Pb: oracle.opt.loss(core.bf16_to_f32(Pb).astype(np.float64), cfg, tokens, labels)  # noqa: E731
    L0 = lf(bits)
    for eps in (1e-3, 1e-2):
        got, L, (g, c, w, a) = _run_step(zo, cfg, bits, tokens[None], labels[None], B, S, 1, n,
                                         eps, 0.0, lam, 1)
        assert np.array_equal(got, bits)  # lr = 0: theta unchanged
        e32 = float(np.float32(eps))
        Lp = np.array([lf(core.perturb(bits, 1, 0, i, +1, e32)) for i in range(n)])
        Lm = np.array([lf(core.perturb(bits, 1, 0, i, -1, e32)) for i in range(n)])
        pc = core.precond(Lp, Lm, L0, e32, 0.0, float(np.float32(lam)), float(np.float32(0.1)))
        if eps == 1e-3:
            assert np.all(np.sign(g) == np.sign(pc["g"])), (g, pc["g"])
            assert np.max(np.abs(g - pc["g"])) <= G_TOL, (g, pc["g"])
        else:
            assert np.max(np.abs(c - pc["c"])) <= C_REL_TOL * np.max(np.abs(pc["c"])), (c, pc["c"])
            assert np.max(np.abs(w / pc["w"] - 1)) <= W_REL_TOL, (w, pc["w"])


def test_c4_shaped_step_matches_oracle(zo):
    """The OPT-1.3B workload's step structure at its real loop counts (8 micro-batches per
    effective batch, n_pert = 160: 321 x 8 micro-forwards) on a narrow 2-layer model: every
    loss against the oracle's (2e-2), and theta' bit for bit against the oracle's
    preconditioner and fixed-order update fed with the GPU's losses."""
    cfg = TINY[0]
    B, S, k, n, eps, lr, lam = 2, 32, 8, 160, 1e-3, 1e-2, 1e-3
    bits = synth.opt_params(cfg, seed=6, varied=True)
    toks, labs = zip(*(synth.opt_batch(cfg, B, S, seed=6, step=j) for j in range(k)))
    tokens, labels = np.stack(toks), np.stack(labs)
    got, L, _ = _run_step(zo, cfg, bits, tokens, labels, B, S, k, n, eps, lr, lam, 6)
    flat_t, flat_l = tokens.reshape(-1, S), labels.reshape(-1)
    loss = lambda Pb: oracle.opt.loss(core.bf16_to_f32(Pb), cfg, flat_t, flat_l)  # noqa: E731
    e32 = float(np.float32(eps))
    ref = np.array([loss(bits)] + [loss(core.perturb(bits, 6, 0, i, s, e32))
                                   for s in (+1, -1) for i in range(n)])
    assert np.allclose(L, ref, rtol=2e-2, atol=0)
    nxt, _ = _teacher_forced(bits, L, n, eps, lr, lam, 6)
    assert np.array_equal(got, nxt)


def test_opt125m_full_size_sampled(zo):
    """The OPT-125M-shaped workload at full size (16 x 256 tokens): the clean loss and one
    perturbed loss against the oracle (fp32 numpy forward), and the hidden state after the
    first layer."""
    cfg = synth.OPT_CONFIGS["opt-125m"]
    B, S = 16, 256
    bits = synth.opt_params(cfg, seed=0)
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=0)
    model = zo.zo_model_create(ctx, cfg, B * S)
    tokens, labels = synth.opt_batch(cfg, B, S, seed=0)
    dtok, dlab = torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda()
    out = torch.zeros(2, dtype=torch.float64, device="cuda")
    zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out[0:1])
    h = torch.zeros((B * S, cfg["d_model"]), dtype=torch.float32, device="cuda")
    zo.zo_model_hidden(model, dtok, B, S, 1, h)
    zo.zo_perturb(ctx, +1, 1e-3, 0)
    zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out[1:2])
    zo.zo_restore(ctx)
    assert zo.zo_sync(ctx) == 0
    P0 = core.bf16_to_f32(bits)
    ref0 = oracle.opt.loss(P0, cfg, tokens, labels, dtype=np.float32)
    href = oracle.opt.hidden_states(P0, cfg, tokens, n_layers=1, dtype=np.float32)
    assert _rel_fro(h.cpu().numpy().astype(np.float64), href.reshape(B * S, -1).astype(np.float64)) <= 1e-2
    P1 = core.bf16_to_f32(core.perturb(bits, 0, 0, 0, +1, 1e-3))
    ref1 = oracle.opt.loss(P1, cfg, tokens, labels, dtype=np.float32)
    got = out.cpu().numpy()
    assert abs(got[0] - ref0) <= 2e-2 * abs(ref0)
    assert abs(got[1] - ref1) <= 2e-2 * abs(ref1)
    model.close()
    ctx.close()


def test_bounded_wait_expiry_is_reported_and_context_survives(zo):
    """A pipeline barrier that is never satisfied (test hook: 16 bytes more expected than
    the loads deliver) makes every waiter give up after ~2 s: ZO_ERR_TIMEOUT is reported by
    zo_sync, and the same context then runs a correct GEMM."""
    th = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    ctx = zo.zo_create(th, seed=0)
    r = np.random.default_rng(5)
    A = bf16(r.standard_normal((128, 64)))
    B = bf16(r.standard_normal((128, 64)))
    out = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    zo.zo_debug_gemm_timeout(ctx, A, B, out, 128, 128, 64)
    with pytest.raises(zo.ZoError) as ei:
        zo.zo_sync(ctx)
    assert ei.value.status == zo.ZO_ERR_TIMEOUT
    zo.zo_gemm_bf16(ctx, A, B, None, out, 128, 128, 64, 128, 0)
    assert zo.zo_sync(ctx) == 0
    ref = f64(A) @ f64(B).T
    assert np.all(np.abs(f64(out) - ref) <= 2.0 ** -8 * (np.abs(ref) + np.sqrt(np.mean(ref ** 2))))
    ctx.close()


@pytest.mark.parametrize("B,S", [(3, 100), (2, 1), (1, 127)])
def test_pruned_last_layer_matches_full_layer(zo, B, S):
    """The loss forward prunes the last layer to the last position of each sequence (keys
    and values still for every position).  Same loss as the full layer, clean and perturbed:
    the only difference is the last query's softmax probabilities, kept in fp32 by the
    pruned kernel and rounded to bf16 by the full one (5e-3 relative); and both against the
    oracle (2e-2)."""
    cfg = TINY[0]
    bits, theta, ctx, model, tokens, labels = _setup(zo, cfg, B, S)
    dtok, dlab = torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda()
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    for i, (sign, probe) in enumerate(((0, 0), (+1, 2))):
        if sign:
            zo.zo_perturb(ctx, sign, 1e-3, probe)
        zo.zo_model_set_pruning(model, True)
        zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out[2 * i:2 * i + 1])
        zo.zo_model_set_pruning(model, False)
        zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out[2 * i + 1:2 * i + 2])
        if sign:
            zo.zo_restore(ctx)
    assert zo.zo_sync(ctx) == 0
    got = out.cpu().numpy()
    for i, (sign, probe) in enumerate(((0, 0), (+1, 2))):
        P = core.bf16_to_f32(core.perturb(bits, 0, 0, probe, sign, 1e-3) if sign else bits)
        ref = oracle.opt.loss(P.astype(np.float64), cfg, tokens, labels)
        assert abs(got[2 * i] - got[2 * i + 1]) <= 5e-3 * abs(got[2 * i + 1])
        assert abs(got[2 * i] - ref) <= 2e-2 * abs(ref)
    model.close()
    ctx.close()
