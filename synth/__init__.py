"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module only draws inputs (weights, curvature vectors, data batches, loss values
used as test inputs); it holds none of the zero-order method's arithmetic (no probes,
perturbations, losses of the trained model, preconditioner or update).  Every array is
a pure function of its arguments: numpy's PCG64 seeded with (seed, stream tag, ...).

Workload shapes follow the pages' setups as restated in the design notes:
  - diagonal quadratic: theta_0 ~ N(0, 1), D_j = 10^U(-3, 3) (log-uniform on [1e-3, 1e3]);
  - MLP classifier 64 -> 256 (ReLU) -> 10, parameters N(0, 0.05), inputs N(0, 1),
    labels = argmax of a fixed random teacher MLP of the same shape;
  - OPT-shaped decoders: matrices and embeddings N(0, 0.02) in bf16, biases 0,
    LayerNorm gains 1 and shifts 0, tokens uniform over the vocabulary, binary labels;
  - Qwen3-shaped decoders: the same, with RMSNorm gains 1 and no biases;
  - the conditioning-study quadratic: theta_0 ~ N(0, 1), D log-uniform on [1e-3, 1e-1],
    eigenvalues of the rank-one terms tr(D) * (30, 10, 3, 1), a seed for their directions.
"""
import numpy as np

_TAGS = {"quad": 1, "mlp": 2, "teacher": 3, "batch": 4, "loss": 5, "coef": 6, "opt": 7,
         "tokens": 8, "labels": 9, "theta": 10, "lowrank": 11}


def rng(seed, tag, *more):
    return np.random.default_rng([int(seed) & 0xFFFFFFFF, _TAGS[tag]] + [int(m) for m in more])


def to_bf16_bits(x):
    """float32 -> bf16 bit pattern (uint16), round to nearest even (inputs only)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# ---------------------------------------------------------------- diagonal quadratic

def quad_problem(M, seed=0):
    """(theta_0 float32 [M], D float32 [M])."""
    r = rng(seed, "quad", M)
    theta = r.standard_normal(M, dtype=np.float32)
    D = (10.0 ** r.uniform(-3.0, 3.0, M)).astype(np.float32)
    return theta, D


LOWRANK_SCALES = (30.0, 10.0, 3.0, 1.0)  # eigenvalues of the directions, in units of tr(D)


def lowrank_problem(M, seed=0, rank=4):
    """Conditioning-study quadratic: (theta_0 float32 [M], D float32 [M] log-uniform in
    [1e-3, 1e-1], lam [rank] = tr(D) * LOWRANK_SCALES[:rank], vseed)."""
    r = rng(seed, "lowrank", M)
    theta = r.standard_normal(M, dtype=np.float32)
    D = (10.0 ** r.uniform(-3.0, -1.0, M)).astype(np.float32)
    tr = float(D.astype(np.float64).sum())
    lam = [float(np.float32(tr * c)) for c in LOWRANK_SCALES[:rank]]
    vseed = int(r.integers(1, 2 ** 63))
    return theta, D, lam, vseed


# ---------------------------------------------------------------- MLP classifier

MLP_IN, MLP_HIDDEN, MLP_OUT, MLP_BATCH = 64, 256, 10, 64


def mlp_param_count(n_in=MLP_IN, n_hidden=MLP_HIDDEN, n_out=MLP_OUT):
    return n_hidden * n_in + n_hidden + n_out * n_hidden + n_out


def mlp_params(seed=0, tag="mlp", n_in=MLP_IN, n_hidden=MLP_HIDDEN, n_out=MLP_OUT, std=0.05):
    """Flat float32 parameters in the order W1[h][in], b1[h], W2[out][h], b2[out]."""
    M = mlp_param_count(n_in, n_hidden, n_out)
    return (rng(seed, tag, M).standard_normal(M) * std).astype(np.float32)


def mlp_batch(seed, step, teacher, n_in=MLP_IN, n_hidden=MLP_HIDDEN, n_out=MLP_OUT,
              batch=MLP_BATCH):
    """(X float32 [batch][n_in], labels int32 [batch]) for one step.

    Labels are the argmax (lowest index on ties) of the teacher network's outputs,
    evaluated in fp64 here purely to label the synthetic data.
    """
    X = rng(seed, "batch", step).standard_normal((batch, n_in), dtype=np.float32)
    t = teacher.astype(np.float64)
    o = 0
    W1 = t[o:o + n_hidden * n_in].reshape(n_hidden, n_in); o += n_hidden * n_in
    b1 = t[o:o + n_hidden]; o += n_hidden
    W2 = t[o:o + n_out * n_hidden].reshape(n_out, n_hidden); o += n_out * n_hidden
    b2 = t[o:o + n_out]
    h = np.maximum(X.astype(np.float64) @ W1.T + b1, 0.0)
    y = np.argmax(h @ W2.T + b2, axis=1).astype(np.int32)
    return X, y


# ---------------------------------------------------------------- loss values as inputs

def losses(n, seed=0, L0=2.3, eps=1e-3, g_scale=1.0, c_scale=50.0):
    """Synthetic (loss_plus[n], loss_minus[n], loss0) in fp64, shaped like a real step:
    L+- = L0 +- eps*g + eps^2*c/2 with random g, c (used as inputs to the update path)."""
    r = rng(seed, "loss", n)
    g = r.standard_normal(n) * g_scale
    c = np.abs(r.standard_normal(n)) * c_scale * np.where(r.uniform(size=n) < 0.1, -1, 1)
    lp = L0 + eps * g + 0.5 * eps * eps * c
    lm = L0 - eps * g + 0.5 * eps * eps * c
    return lp, lm, float(L0)


def coefficients(n, seed=0, scale=1e-3):
    """Synthetic fp32 update coefficients a[n] (mixed signs and magnitudes)."""
    r = rng(seed, "coef", n)
    return (r.standard_normal(n) * scale * 10.0 ** r.uniform(-2, 0, n)).astype(np.float32)


# ---------------------------------------------------------------- OPT-shaped decoders

OPT_CONFIGS = {
    # the pages' model family at three sizes; vocabulary and position table of OPT
    "opt-125m": dict(n_layers=12, d_model=768, n_heads=12, d_ffn=3072, vocab=50272,
                     max_pos=2048, class_ids=(1000, 2000)),
    "opt-1.3b": dict(n_layers=24, d_model=2048, n_heads=32, d_ffn=8192, vocab=50272,
                     max_pos=2048, class_ids=(1000, 2000)),
    "opt-30b": dict(n_layers=48, d_model=7168, n_heads=56, d_ffn=28672, vocab=50272,
                    max_pos=2048, class_ids=(1000, 2000)),
}


def opt_segments(cfg):
    """(kind, count) runs of the flat parameter vector in order; kind is one of
    'matrix' (embeddings and projection weights), 'bias', 'gain', 'shift'."""
    d, f, V, P = cfg["d_model"], cfg["d_ffn"], cfg["vocab"], cfg["max_pos"] + 2
    segs = [("matrix", V * d), ("matrix", P * d)]
    for _ in range(cfg["n_layers"]):
        segs += [("gain", d), ("shift", d), ("matrix", 3 * d * d), ("bias", 3 * d),
                 ("matrix", d * d), ("bias", d), ("gain", d), ("shift", d),
                 ("matrix", f * d), ("bias", f), ("matrix", d * f), ("bias", d)]
    segs += [("gain", d), ("shift", d)]
    return segs


def opt_params(cfg, seed=0, varied=False):
    """bf16 bits (uint16) of the flat parameters.  OPT-style init (varied=False): matrices
    N(0, 0.02), biases 0, LayerNorm gains 1 and shifts 0.  varied=True (parity tests)
    also draws biases N(0, 0.02), gains 1 + N(0, 0.1) and shifts N(0, 0.02) so that every
    parameter kind influences the loss."""
    segs = opt_segments(cfg)
    total = sum(n for _, n in segs)
    r = rng(seed, "opt", total)
    out = np.empty(total, np.uint16)
    o = 0
    for kind, n in segs:
        if kind == "matrix":
            x = r.standard_normal(n, dtype=np.float32) * np.float32(0.02)
        elif kind == "bias" or kind == "shift":
            x = (r.standard_normal(n, dtype=np.float32) * np.float32(0.02) if varied
                 else np.zeros(n, np.float32))
        else:  # gain
            x = (1.0 + r.standard_normal(n, dtype=np.float32) * np.float32(0.1) if varied
                 else np.ones(n, np.float32))
        out[o:o + n] = to_bf16_bits(x)
        o += n
    return out


def opt_batch(cfg, batch, seq, seed=0, step=0):
    """(tokens int32 [batch][seq] uniform over the vocabulary, labels int32 [batch] in {0,1})."""
    tokens = rng(seed, "tokens", step, batch, seq).integers(0, cfg["vocab"], (batch, seq),
                                                            dtype=np.int32)
    labels = rng(seed, "labels", step, batch).integers(0, 2, batch, dtype=np.int32)
    return tokens, labels


# ---------------------------------------------------------------- Qwen3-shaped decoders

QWEN_CONFIGS = {
    # the pages' second model family (synthetic weights; the head is tied to the embedding)
    "qwen3-1.7b": dict(family="qwen3", n_layers=28, d_model=2048, n_heads=16, n_kv_heads=8,
                       head_dim=128, d_ffn=6144, vocab=151936, max_pos=4096, rope_theta=1.0e6,
                       norm_eps=1e-6, class_ids=(1000, 2000)),
    "qwen3-8b": dict(family="qwen3", n_layers=36, d_model=4096, n_heads=32, n_kv_heads=8,
                     head_dim=128, d_ffn=12288, vocab=151936, max_pos=4096, rope_theta=1.0e6,
                     norm_eps=1e-6, class_ids=(1000, 2000)),
}


def qwen_segments(cfg):
    """(kind, count) runs of the flat Qwen3-shaped parameter vector: 'matrix' or 'gain'."""
    d, H, Hk, e, f = (cfg["d_model"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"],
                      cfg["d_ffn"])
    segs = [("matrix", cfg["vocab"] * d)]
    for _ in range(cfg["n_layers"]):
        segs += [("gain", d), ("matrix", (H + 2 * Hk) * e * d), ("gain", e), ("gain", e),
                 ("matrix", d * H * e), ("gain", d), ("matrix", 2 * f * d), ("matrix", d * f)]
    segs += [("gain", d)]
    return segs


def qwen_params(cfg, seed=0, varied=False):
    """bf16 bits of the flat parameters: matrices N(0, 0.02), RMSNorm gains 1 (varied=True:
    1 + N(0, 0.1), for parity tests)."""
    segs = qwen_segments(cfg)
    total = sum(n for _, n in segs)
    r = rng(seed, "opt", total, 3)
    out = np.empty(total, np.uint16)
    o = 0
    for kind, n in segs:
        if kind == "matrix":
            x = r.standard_normal(n, dtype=np.float32) * np.float32(0.02)
        else:
            x = (1.0 + r.standard_normal(n, dtype=np.float32) * np.float32(0.1) if varied
                 else np.ones(n, np.float32))
        out[o:o + n] = to_bf16_bits(x)
        o += n
    return out
