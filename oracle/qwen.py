"""Loss-only forward of the Qwen3-shaped decoder, in fp64 (or fp32) numpy.

TEST INFRASTRUCTURE (see oracle/__init__.py).  Qwen3 is the pages' second model family
("Probe-Space Preconditioning for Fast and Stable Zero-Order Training", abstract: post-
training benchmarks on Qwen3 and OPT).  Its architecture (from the public Qwen3 release):
pre-RMSNorm decoder layers (eps 1e-6), grouped-query attention with per-head RMSNorm on the
queries and keys followed by rotary position embeddings (rotate-half convention, base
rope_theta), no projection biases, SwiGLU feed-forward silu(x Wg^T) * (x Wu^T) Wd^T, final
RMSNorm, head tied to the token embedding.  The loss is the same 2-class last-position
cross-entropy as the OPT-shaped workload.

Flat parameter order (d = d_model, H / Hk = query / key-value heads, e = head_dim, f = d_ffn):
  E[V][d],
  per layer: in_norm[d], Wqkv[(H + 2 Hk) e][d] (rows: q heads, k heads, v heads),
             q_norm[e], k_norm[e], Wo[d][H e], post_norm[d], Wgu[2f][d] (rows: gate, up),
             Wd[d][f],
  then final_norm[d].
"""
import numpy as np

LAYER_FIELDS = ("in_norm", "wqkv", "q_norm", "k_norm", "wo", "post_norm", "wgu", "wd")


def layer_shapes(cfg):
    d, H, Hk, e, f = (cfg["d_model"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                      cfg["d_ffn"])
    return {"in_norm": (d,), "wqkv": ((H + 2 * Hk) * e, d), "q_norm": (e,), "k_norm": (e,),
            "wo": (d, H * e), "post_norm": (d,), "wgu": (2 * f, d), "wd": (d, f)}


def layout(cfg):
    d, V = cfg["d_model"], cfg["vocab"]
    out = {"E": (0, (V, d))}
    o = V * d
    shapes = layer_shapes(cfg)
    for layer in range(cfg["n_layers"]):
        for name in LAYER_FIELDS:
            out[f"L{layer}.{name}"] = (o, shapes[name])
            o += int(np.prod(shapes[name]))
    out["final_norm"] = (o, (d,))
    o += d
    out["total"] = o
    return out


def param_count(cfg):
    return layout(cfg)["total"]


def _view(theta, lay, name):
    off, shape = lay[name]
    return theta[off:off + int(np.prod(shape))].reshape(shape)


def _rmsnorm(x, w, eps):
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps) * w


def _rope(x, positions, theta_base):
    """Rotary embedding, rotate-half convention: x [B, heads, S, e]."""
    e = x.shape[-1]
    inv = 1.0 / theta_base ** (np.arange(0, e, 2, dtype=np.float64) / e)  # [e/2]
    ang = positions[:, None].astype(np.float64) * inv[None, :]             # [S, e/2]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], axis=-1)
    sin = np.concatenate([np.sin(ang), np.sin(ang)], axis=-1)
    x1, x2 = x[..., : e // 2], x[..., e // 2:]
    rot = np.concatenate([-x2, x1], axis=-1)
    return x * cos + rot * sin


def hidden_states(theta, cfg, tokens, n_layers=None, dtype=np.float64):
    lay = layout(cfg)
    th = np.asarray(theta, dtype)
    d, H, Hk, e = cfg["d_model"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    f, eps = cfg["d_ffn"], cfg["norm_eps"]
    tokens = np.asarray(tokens)
    B, S = tokens.shape
    h = _view(th, lay, "E")[tokens]
    pos = np.arange(S)
    causal = np.triu(np.ones((S, S), bool), k=1)
    group = H // Hk
    for layer in range(cfg["n_layers"] if n_layers is None else n_layers):
        p = {name: _view(th, lay, f"L{layer}.{name}") for name in LAYER_FIELDS}
        x = _rmsnorm(h, p["in_norm"], eps)
        qkv = x @ p["wqkv"].T
        q = qkv[..., :H * e].reshape(B, S, H, e)
        k = qkv[..., H * e:(H + Hk) * e].reshape(B, S, Hk, e)
        v = qkv[..., (H + Hk) * e:].reshape(B, S, Hk, e)
        q = _rmsnorm(q, p["q_norm"], eps).transpose(0, 2, 1, 3)
        k = _rmsnorm(k, p["k_norm"], eps).transpose(0, 2, 1, 3)
        v = v.transpose(0, 2, 1, 3)
        q = _rope(q, pos, cfg["rope_theta"])
        k = _rope(k, pos, cfg["rope_theta"])
        k = np.repeat(k, group, axis=1)  # query head h uses key/value head h // group
        v = np.repeat(v, group, axis=1)
        scores = q @ k.transpose(0, 1, 3, 2) / np.sqrt(e)
        scores = np.where(causal, -np.inf, scores)
        scores = scores - scores.max(axis=-1, keepdims=True)
        w = np.exp(scores)
        w = w / w.sum(axis=-1, keepdims=True)
        att = (w @ v).transpose(0, 2, 1, 3).reshape(B, S, H * e)
        h = h + att @ p["wo"].T
        x = _rmsnorm(h, p["post_norm"], eps)
        gu = x @ p["wgu"].T
        g, u = gu[..., :f], gu[..., f:]
        h = h + ((g / (1.0 + np.exp(-g))) * u) @ p["wd"].T
    return h


def per_sample_loss(theta, cfg, tokens, labels, dtype=np.float64):
    lay = layout(cfg)
    th = np.asarray(theta, dtype)
    h = hidden_states(th, cfg, tokens, dtype=dtype)
    xl = _rmsnorm(h[:, -1, :], _view(th, lay, "final_norm"), cfg["norm_eps"])
    logits = xl @ _view(th, lay, "E")[list(cfg["class_ids"])].T
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    return lse - logits[np.arange(len(labels)), np.asarray(labels)]


def loss(theta, cfg, tokens, labels, dtype=np.float64):
    return float(per_sample_loss(theta, cfg, tokens, labels, dtype).mean())
