"""A model of the decoder forward's bf16 activation rounding, for deriving test tolerances.

Test-side reference, not the oracle: it follows the oracle's Qwen3-shaped forward step by step
in fp64 and additionally rounds to bf16 (round to nearest even) at every point where the
decoder's reading of the precision ("GEMM inputs bf16, fp32 accumulation, norms, softmax and
the loss in fp32, residual stream fp32") stores a bf16 activation: the norm outputs, the QKV
projection, the normalised and rotated queries and keys, the attention probabilities and
output, and the SwiGLU product.  Its deviation from the exact fp64 forward measures how far
that precision alone moves the hidden states, which is the basis of the full-depth
tolerances of the GPU tests.  It does not import the CUDA path.
"""
import numpy as np


def round_bf16(x):
    """x rounded to the nearest bf16 value (ties to even), through fp32, returned as fp64."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


def _rmsnorm(x, w, eps):
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * w


def _rope(x, positions, base):
    e = x.shape[-1]
    inv = 1.0 / base ** (np.arange(0, e, 2, dtype=np.float64) / e)
    ang = positions[:, None].astype(np.float64) * inv[None, :]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], axis=-1)
    sin = np.concatenate([np.sin(ang), np.sin(ang)], axis=-1)
    rot = np.concatenate([-x[..., e // 2:], x[..., : e // 2]], axis=-1)
    return x * cos + rot * sin


def qwen_hidden_states(E_rows, blocks, cfg, n_layers, rounding=True):
    """Residual stream [S, d] of one sequence after n_layers Qwen3-shaped layers, with bf16
    activations (rounding=False: none, which must reproduce the exact forward).  E_rows [S, d]:
    the sequence's embedding rows; blocks(l): dict of layer l's parameters (names and shapes
    of the oracle's Qwen3 layout), real values."""
    d, H, Hk, e = cfg["d_model"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    f, eps = cfg["d_ffn"], cfg["norm_eps"]
    S = E_rows.shape[0]
    h = np.asarray(E_rows, np.float64)
    pos = np.arange(S)
    causal = np.triu(np.ones((S, S), bool), k=1)
    r = round_bf16 if rounding else (lambda x: x)
    for li in range(n_layers):
        p = blocks(li)
        x = r(_rmsnorm(h, p["in_norm"], eps))
        qkv = r(x @ p["wqkv"].T)
        q = qkv[:, :H * e].reshape(S, H, e)
        k = qkv[:, H * e:(H + Hk) * e].reshape(S, Hk, e)
        v = qkv[:, (H + Hk) * e:].reshape(S, Hk, e).transpose(1, 0, 2)
        q = r(_rope(_rmsnorm(q, p["q_norm"], eps).transpose(1, 0, 2), pos, cfg["rope_theta"]))
        k = r(_rope(_rmsnorm(k, p["k_norm"], eps).transpose(1, 0, 2), pos, cfg["rope_theta"]))
        k = np.repeat(k, H // Hk, axis=0)
        v = np.repeat(v, H // Hk, axis=0)
        s = q @ k.transpose(0, 2, 1) / np.sqrt(e)
        s = np.where(causal, -np.inf, s)
        pexp = np.exp(s - s.max(axis=-1, keepdims=True))
        att = r((r(pexp) @ v) / pexp.sum(axis=-1, keepdims=True))  # bf16 P, fp32 row sum
        h = h + att.transpose(1, 0, 2).reshape(S, H * e) @ p["wo"].T
        x = r(_rmsnorm(h, p["post_norm"], eps))
        gu = x @ p["wgu"].T
        g, u = gu[:, :f], gu[:, f:]
        h = h + r(g / (1.0 + np.exp(-g)) * u) @ p["wd"].T
    return h
