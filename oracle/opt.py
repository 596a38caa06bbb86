"""Loss-only forward of the OPT-shaped decoder, in fp64 (or fp32) numpy.

TEST INFRASTRUCTURE (see oracle/__init__.py).  The architecture is OPT's as the pages
use it for fine-tuning ("Probe-Space Preconditioning for Fast and Stable Zero-Order
Training", abstract: OPT-13B/30B trained in inference mode): pre-LayerNorm decoder layers,
learned positions with an offset of 2, ReLU feed-forward, biases on every projection,
final LayerNorm, head tied to the token embedding.  The loss is the 2-class cross-entropy
of the last position's logits restricted to two class tokens, per sequence.

Flat parameter order (d = d_model, f = d_ffn, V = vocab, P = max_pos + 2):
  E[V][d], Pos[P][d],
  per layer: ln1.g[d], ln1.b[d], Wqkv[3d][d] (rows q, k, v), bqkv[3d], Wo[d][d], bo[d],
             ln2.g[d], ln2.b[d], W1[f][d], b1[f], W2[d][f], b2[d],
  then lnf.g[d], lnf.b[d].
Every step below is written out plainly: library matrix products are the only primitive.
"""
import numpy as np

LAYER_FIELDS = ("ln1g", "ln1b", "wqkv", "bqkv", "wo", "bo", "ln2g", "ln2b", "w1", "b1", "w2", "b2")


def layer_shapes(d, f):
    return {"ln1g": (d,), "ln1b": (d,), "wqkv": (3 * d, d), "bqkv": (3 * d,), "wo": (d, d),
            "bo": (d,), "ln2g": (d,), "ln2b": (d,), "w1": (f, d), "b1": (f,), "w2": (d, f),
            "b2": (d,)}


def layout(cfg):
    """{name: (offset, shape)} for the flat vector, plus 'total'."""
    d, f, V, P = cfg["d_model"], cfg["d_ffn"], cfg["vocab"], cfg["max_pos"] + 2
    out = {"E": (0, (V, d)), "Pos": (V * d, (P, d))}
    o = V * d + P * d
    shapes = layer_shapes(d, f)
    for layer in range(cfg["n_layers"]):
        for name in LAYER_FIELDS:
            n = int(np.prod(shapes[name]))
            out[f"L{layer}.{name}"] = (o, shapes[name])
            o += n
    out["lnf.g"] = (o, (d,))
    o += d
    out["lnf.b"] = (o, (d,))
    o += d
    out["total"] = o
    return out


def param_count(cfg):
    return layout(cfg)["total"]


def _view(theta, lay, name):
    off, shape = lay[name]
    n = int(np.prod(shape))
    return theta[off:off + n].reshape(shape)


def _layernorm(x, g, b, eps=1e-5):
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * g + b


def embed(E, Pos, tokens):
    """Residual stream at the input of the first layer: [B, S, d] = E[token] + Pos[s + 2]."""
    tokens = np.asarray(tokens)
    S = tokens.shape[1]
    return E[tokens] + Pos[np.arange(S) + 2][None, :, :]


def layer(h, p, n_heads):
    """One pre-LN decoder layer on the residual stream h [B, S, d]; p maps the LAYER_FIELDS
    names to the layer's parameters (shapes of layer_shapes)."""
    B, S, d = h.shape
    H = n_heads
    hd = d // H
    causal = np.triu(np.ones((S, S), bool), k=1)  # True where key > query
    x = _layernorm(h, p["ln1g"], p["ln1b"])
    qkv = x @ p["wqkv"].T + p["bqkv"]
    q = qkv[..., 0:d].reshape(B, S, H, hd).transpose(0, 2, 1, 3)
    k = qkv[..., d:2 * d].reshape(B, S, H, hd).transpose(0, 2, 1, 3)
    v = qkv[..., 2 * d:3 * d].reshape(B, S, H, hd).transpose(0, 2, 1, 3)
    scores = q @ k.transpose(0, 1, 3, 2) / np.sqrt(hd)
    scores = np.where(causal, -np.inf, scores)
    scores = scores - scores.max(axis=-1, keepdims=True)
    w = np.exp(scores)
    w = w / w.sum(axis=-1, keepdims=True)
    att = (w @ v).transpose(0, 2, 1, 3).reshape(B, S, d)
    h = h + (att @ p["wo"].T + p["bo"])
    x = _layernorm(h, p["ln2g"], p["ln2b"])
    return h + (np.maximum(x @ p["w1"].T + p["b1"], 0.0) @ p["w2"].T + p["b2"])


def layer_params(block, d, f):
    """The LAYER_FIELDS views of one layer's flat parameter block (in flat order)."""
    shapes = layer_shapes(d, f)
    out, o = {}, 0
    for name in LAYER_FIELDS:
        n = int(np.prod(shapes[name]))
        out[name] = block[o:o + n].reshape(shapes[name])
        o += n
    return out


def head_losses(h_last, lnf_g, lnf_b, E_class, labels):
    """Per-sequence 2-class cross-entropy from the last position's residual rows [B, d]: the
    final LayerNorm, logits against the two tied class rows E_class [2, d]."""
    xl = _layernorm(h_last, lnf_g, lnf_b)
    logits = xl @ E_class.T  # [B, 2]
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    return lse - logits[np.arange(len(labels)), np.asarray(labels)]


def hidden_states(theta, cfg, tokens, n_layers=None, dtype=np.float64):
    """Residual stream after the embedding and the first n_layers layers: [B, S, d].
    theta: flat parameters as real numbers (bf16 values widened), any float dtype."""
    lay = layout(cfg)
    th = np.asarray(theta, dtype)
    h = embed(_view(th, lay, "E"), _view(th, lay, "Pos"), tokens)
    for li in range(cfg["n_layers"] if n_layers is None else n_layers):
        p = {name: _view(th, lay, f"L{li}.{name}") for name in LAYER_FIELDS}
        h = layer(h, p, cfg["n_heads"])
    return h


def per_sample_loss(theta, cfg, tokens, labels, dtype=np.float64):
    """2-class cross-entropy of each sequence's last position."""
    lay = layout(cfg)
    th = np.asarray(theta, dtype)
    h = hidden_states(th, cfg, tokens, dtype=dtype)
    E = _view(th, lay, "E")
    return head_losses(h[:, -1, :], _view(th, lay, "lnf.g"), _view(th, lay, "lnf.b"),
                       E[list(cfg["class_ids"])], labels)


def loss(theta, cfg, tokens, labels, dtype=np.float64):
    """Mean over the batch."""
    return float(per_sample_loss(theta, cfg, tokens, labels, dtype).mean())
