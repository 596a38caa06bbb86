"""Qwen3-shaped decoder forward on the GPU against the oracle's fp64 forward: hidden states
after every layer prefix, clean and perturbed, the loss, and one full 1.5-SPSA step, on tiny
configurations that exercise grouped-query attention (2 and 4 query heads per key/value
head, and plain multi-head), head dims 64 and 128, head width H*e different from d_model,
ragged sequence tails and bias-free projections.  Tolerances are those of the OPT-shaped
forward: bf16 activations between the kernels bound the hidden-state error to about 1e-2
relative (Frobenius) and the loss to 2e-2 relative."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import core

pytestmark = pytest.mark.gpu

TINY = [
    dict(family="qwen3", n_layers=2, d_model=128, n_heads=4, n_kv_heads=2, head_dim=64, d_ffn=320,
         vocab=1000, max_pos=160, rope_theta=1.0e4, norm_eps=1e-6, class_ids=(3, 7)),
    dict(family="qwen3", n_layers=2, d_model=256, n_heads=4, n_kv_heads=1, head_dim=128,
         d_ffn=512, vocab=777, max_pos=200, rope_theta=1.0e6, norm_eps=1e-6, class_ids=(0, 776)),
    dict(family="qwen3", n_layers=1, d_model=192, n_heads=3, n_kv_heads=3, head_dim=64, d_ffn=256,
         vocab=500, max_pos=300, rope_theta=1.0e6, norm_eps=1e-5, class_ids=(10, 11)),
]


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


def _np_gqa(qkv, B, S, H, Hk, e):
    """Causal grouped-query attention in fp64: query head h uses key/value head h // (H/Hk)."""
    x = qkv.reshape(B, S, H + 2 * Hk, e)
    q = x[:, :, :H].transpose(0, 2, 1, 3)
    k = np.repeat(x[:, :, H:H + Hk].transpose(0, 2, 1, 3), H // Hk, axis=1)
    v = np.repeat(x[:, :, H + Hk:].transpose(0, 2, 1, 3), H // Hk, axis=1)
    s = q @ k.transpose(0, 1, 3, 2) / np.sqrt(e)
    s = np.where(np.triu(np.ones((S, S), bool), 1), -np.inf, s)
    w = np.exp(s - s.max(-1, keepdims=True))
    w /= w.sum(-1, keepdims=True)
    return (w @ v).transpose(0, 2, 1, 3).reshape(B * S, H * e)


@pytest.mark.parametrize("B,S,H,Hk,e", [(2, 64, 4, 2, 64), (1, 300, 8, 2, 128),
                                        (3, 130, 6, 1, 64), (2, 257, 16, 8, 128)])
def test_gqa_attention_matches_numpy(zo, ctx, B, S, H, Hk, e):
    r = np.random.default_rng(B * 1000 + S + H)
    qkv = bf16(r.standard_normal((B * S, (H + 2 * Hk) * e)))
    out = torch.zeros((B * S, H * e), dtype=torch.bfloat16, device="cuda")
    zo.zo_attention_gqa(ctx, qkv, out, B, S, H, Hk, e)
    torch.cuda.synchronize()
    assert zo.zo_sync(ctx) == 0  # no bounded wait expired
    assert np.max(np.abs(f64(out) - _np_gqa(f64(qkv), B, S, H, Hk, e))) <= 2e-2
    bad = next(k for k in range(2, H + 1) if H % k)  # H not a multiple of Hk: rejected
    with pytest.raises(zo.ZoError):
        zo.zo_attention_gqa(ctx, qkv, out, B, S, H, bad, e)


@pytest.mark.parametrize("M,N,K", [(128, 64, 64), (300, 320, 136), (1024, 1536, 512),
                                   (4096, 1024, 256),
                                   # CTA-pair tiles (>= 148 tiles of 256 x 256), ragged edges
                                   (4096, 1280, 256), (4000, 1304, 136)])
def test_swiglu_gemm_matches_numpy(zo, ctx, M, N, K):
    """Epilogue 3: out = silu(A Wg^T) * (A Wu^T) from one GEMM over [Wg; Wu], against fp64;
    one bf16 rounding of fp32-accumulated products (tolerance as the other bf16 outputs)."""
    r = np.random.default_rng(M + N + K)
    A = bf16(r.standard_normal((M, K)))
    W = bf16(r.standard_normal((2 * N, K)) * 0.1)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    zo.zo_gemm_bf16(ctx, A, W, None, out, M, N, K, N, 3)
    assert zo.zo_sync(ctx) == 0
    gu = f64(A) @ f64(W).T
    g, u = gu[:, :N], gu[:, N:]
    ref = g / (1 + np.exp(-g)) * u
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(f64(out) - ref) <= 2.0 ** -8 * (np.abs(ref) + rms))
    with pytest.raises(zo.ZoError):  # no bias with this epilogue
        zo.zo_gemm_bf16(ctx, A, W, torch.zeros(2 * N, dtype=torch.bfloat16, device="cuda"), out,
                        M, N, K, N, 3)


def test_rmsnorm_matches_numpy(zo, ctx):
    r = np.random.default_rng(1)
    rows, d, eps = 37, 4096, 1e-6
    x = torch.from_numpy((r.standard_normal((rows, d)) * 3 + 1).astype(np.float32)).cuda()
    w = bf16(1 + 0.1 * r.standard_normal(d))
    out = torch.zeros((rows, d), dtype=torch.bfloat16, device="cuda")
    zo.zo_rmsnorm(ctx, x, w, out, rows, d, eps)
    torch.cuda.synchronize()
    xx = x.cpu().numpy().astype(np.float64)
    ref = xx / np.sqrt((xx * xx).mean(1, keepdims=True) + eps) * f64(w)
    assert np.all(np.abs(f64(out) - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-3)


def _rel_fro(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _setup(zo, cfg, B, S, seed=0):
    bits = synth.qwen_params(cfg, seed=seed, varied=True)
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=seed)
    model = zo.zo_model_create(ctx, cfg, B * S)
    tokens, labels = synth.opt_batch(cfg, B, S, seed=seed)
    return bits, theta, ctx, model, tokens, labels


@pytest.mark.parametrize("cfg", TINY)
@pytest.mark.parametrize("B,S", [(3, 100), (2, 160)])
def test_qwen_hidden_states_and_loss(zo, cfg, B, S):
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
            ref = oracle.qwen.hidden_states(P, cfg, tokens, n_layers=n_run).reshape(B * S, d)
            assert _rel_fro(h.cpu().numpy().astype(np.float64), ref) <= 1e-2, (sign, n_run)
        out = torch.zeros(1, dtype=torch.float64, device="cuda")
        zo.zo_model_loss(model, dtok, dlab, B, S, 1.0 / B, out)
        torch.cuda.synchronize()
        ref = oracle.qwen.loss(P, cfg, tokens, labels)
        assert abs(out.item() - ref) <= 2e-2 * abs(ref), (sign, out.item(), ref)
        if sign:
            zo.zo_restore(ctx)
    assert zo.zo_sync(ctx) == 0
    model.close()
    ctx.close()


def test_qwen_step_matches_oracle(zo):
    """One 1.5-SPSA step of the Qwen3-shaped model with 2 micro-batches: the 2n+1 losses
    against the oracle's (2e-2), and theta' bit for bit against the oracle's preconditioner
    and fixed-order update fed with the GPU's own losses (teacher forcing)."""
    cfg = TINY[0]
    B, S, n_micro, n, eps, lr, lam = 2, 64, 2, 4, 1e-3, 2e-2, 1e-3
    bits = synth.qwen_params(cfg, seed=1, varied=True)
    theta = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ctx = zo.zo_create(theta, seed=1)
    model = zo.zo_model_create(ctx, cfg, B * S)
    toks, labs = zip(*(synth.opt_batch(cfg, B, S, seed=1, step=k) for k in range(n_micro)))
    tokens, labels = np.stack(toks), np.stack(labs)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device="cuda")
    zo.zo_model_step(model, torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda(),
                     B, S, n_micro, n, eps, lr, lam, True, losses)
    assert zo.zo_sync(ctx) == 0
    assert zo.zo_get_step(ctx) == 1
    flat_t, flat_l = tokens.reshape(-1, S), labels.reshape(-1)
    loss = lambda Pb: oracle.qwen.loss(core.bf16_to_f32(Pb), cfg, flat_t, flat_l)  # noqa: E731
    _, rec = oracle.step.spsa_step(bits, loss, n, eps, lr, lam, 1, 0)
    L = losses.cpu().numpy()
    ref = np.concatenate([[rec["L0"]], rec["Lp"], rec["Lm"]])
    assert np.allclose(L, ref, rtol=2e-2, atol=0)
    e32 = float(np.float32(eps))
    pc = core.precond(L[1:1 + n], L[1 + n:], L[0], e32, float(np.float32(lr)),
                      float(np.float32(lam)), float(np.float32(0.1)))
    nxt = core.update_mirror(bits, pc["a"].astype(np.float32), 1, 0)
    got = theta.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, nxt)
    assert not np.array_equal(got, bits)
    model.close()
    ctx.close()
def test_qwen_rejects_sequences_beyond_the_rotary_table(zo):
    cfg = TINY[0]
    bits, theta, ctx, model, tokens, labels = _setup(zo, cfg, 1, cfg["max_pos"])
    out = torch.zeros(1, dtype=torch.float64, device="cuda")
    long_t = torch.zeros((1, cfg["max_pos"] + 1), dtype=torch.int32, device="cuda")
    with pytest.raises(zo.ZoError):
        zo.zo_model_loss(model, long_t, torch.zeros(1, dtype=torch.int32, device="cuda"), 1,
                         cfg["max_pos"] + 1, 1.0, out)
    model.close()
    ctx.close()


@pytest.mark.parametrize("cfg", [TINY[0], TINY[1]])
def test_qwen_pruned_last_layer_matches_full_layer(zo, cfg):
    """As for the OPT shape: the pruned last layer (keys and values for every position,
    queries rotated at position S-1) gives the full layer's loss within 5e-3, clean and
    perturbed, and the oracle's within 2e-2."""
    B, S = 3, 100
    bits, theta, ctx, model, tokens, labels = _setup(zo, cfg, B, S)
    dtok, dlab = torch.from_numpy(tokens).cuda(), torch.from_numpy(labels).cuda()
    out = torch.zeros(4, dtype=torch.float64, device="cuda")
    for i, (sign, probe) in enumerate(((0, 0), (-1, 5))):
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
    for i, (sign, probe) in enumerate(((0, 0), (-1, 5))):
        P = core.bf16_to_f32(core.perturb(bits, 0, 0, probe, sign, 1e-3) if sign else bits)
        ref = oracle.qwen.loss(P.astype(np.float64), cfg, tokens, labels)
        assert abs(got[2 * i] - got[2 * i + 1]) <= 5e-3 * abs(got[2 * i + 1])
        assert abs(got[2 * i] - ref) <= 2e-2 * abs(ref)
    model.close()
    ctx.close()
