"""The seeded synthetic inputs follow the recipe the design notes state for each workload:
distributions, ranges, shapes, parameter counts, and determinism in (seed, stream tag)."""
import numpy as np
import pytest

import synth


def _z(mean, expect, sd, n):
    """Standard score of a sample mean against its expectation."""
    return abs(mean - expect) / (sd / np.sqrt(n))


def test_quadratic_recipe():
    M = 1 << 16
    th, D = synth.quad_problem(M, seed=0)
    assert th.dtype == np.float32 and D.dtype == np.float32 and th.shape == D.shape == (M,)
    assert _z(th.mean(), 0.0, 1.0, M) < 5 and abs(th.std() - 1.0) < 0.02
    assert D.min() >= 1e-3 * (1 - 1e-6) and D.max() <= 1e3 * (1 + 1e-6)
    lg = np.log10(D.astype(np.float64))  # U(-3, 3): mean 0, variance 3
    assert _z(lg.mean(), 0.0, np.sqrt(3.0), M) < 5 and abs(lg.var() - 3.0) < 0.1
    th2, D2 = synth.quad_problem(M, seed=0)
    assert np.array_equal(th, th2) and np.array_equal(D, D2)
    th3, _ = synth.quad_problem(M, seed=1)
    assert not np.array_equal(th, th3)


def test_lowrank_recipe():
    M = 1 << 14
    th, D, lam, vseed = synth.lowrank_problem(M, seed=2)
    assert D.min() >= 1e-3 * (1 - 1e-6) and D.max() <= 1e-1 * (1 + 1e-6)
    tr = float(D.astype(np.float64).sum())
    assert lam == [float(np.float32(tr * c)) for c in synth.LOWRANK_SCALES]
    assert 1 <= vseed < 2 ** 63
    assert len(synth.lowrank_problem(M, seed=2, rank=2)[2]) == 2


def test_mlp_recipe():
    assert synth.mlp_param_count() == 19210
    P = synth.mlp_params(0)
    T = synth.mlp_params(0, tag="teacher")
    assert P.shape == (19210,) and not np.array_equal(P, T)
    assert abs(P.std() - 0.05) < 0.002 and abs(T.std() - 0.05) < 0.002
    X, y = synth.mlp_batch(0, 3, T)
    assert X.shape == (64, 64) and y.shape == (64,) and y.dtype == np.int32
    assert 0 <= y.min() and y.max() < 10
    # labels are the teacher's argmax
    t = T.astype(np.float64)
    W1 = t[:256 * 64].reshape(256, 64)
    b1 = t[256 * 64:256 * 65]
    W2 = t[256 * 65:256 * 65 + 2560].reshape(10, 256)
    b2 = t[256 * 65 + 2560:]
    logits = np.maximum(X.astype(np.float64) @ W1.T + b1, 0) @ W2.T + b2
    assert np.array_equal(y, np.argmax(logits, axis=1))
    X2, _ = synth.mlp_batch(0, 4, T)
    assert not np.array_equal(X, X2)  # a fresh batch every step


@pytest.mark.parametrize("name,count", [("opt-125m", 125_239_296), ("opt-1.3b", 1_315_758_080),
                                        ("opt-30b", 29_974_540_288)])
def test_opt_parameter_counts(name, count):
    assert sum(n for _, n in synth.opt_segments(synth.OPT_CONFIGS[name])) == count


def test_opt_and_qwen_parameter_recipe_on_small_shapes():
    cfg = dict(synth.OPT_CONFIGS["opt-125m"], n_layers=2, d_model=64, n_heads=4, d_ffn=256,
               vocab=1000 + 1024, max_pos=64)
    bits = synth.opt_params(cfg)
    x = (bits.astype(np.uint32) << 16).view(np.float32)
    o = 0
    for kind, n in synth.opt_segments(cfg):
        seg = x[o:o + n]
        if kind == "matrix":
            assert abs(seg.std() - 0.02) < 0.02 * 0.1 or n < 4096
        elif kind in ("bias", "shift"):
            assert np.all(seg == 0)
        else:
            assert np.all(seg == 1)
        o += n
    assert o == len(x)
    qcfg = dict(synth.QWEN_CONFIGS["qwen3-1.7b"], n_layers=1, d_model=64, n_heads=4, n_kv_heads=2,
                head_dim=16, d_ffn=128, vocab=2048)
    qx = (synth.qwen_params(qcfg).astype(np.uint32) << 16).view(np.float32)
    assert len(qx) == sum(n for _, n in synth.qwen_segments(qcfg))
    tokens, labels = synth.opt_batch(cfg, 16, 32, seed=0, step=1)
    assert tokens.shape == (16, 32) and tokens.min() >= 0 and tokens.max() < cfg["vocab"]
    assert set(np.unique(labels)) <= {0, 1}
