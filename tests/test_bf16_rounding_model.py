"""The test-side bf16 rounding model of the Qwen3-shaped forward (tests/bf16_rounding_model.py)
pinned without a GPU: with its roundings switched off it reproduces the oracle's exact forward,
its rounding function agrees with torch's bf16 conversion, and with the roundings on it moves
the hidden states by about bf16 precision per layer."""
import numpy as np
import pytest

import oracle
import synth
from bf16_rounding_model import qwen_hidden_states, round_bf16

torch = pytest.importorskip("torch")

CFG = dict(family="qwen3", n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64,
           d_ffn=384, vocab=500, max_pos=64, rope_theta=1.0e6, norm_eps=1e-6, class_ids=(1, 2))


def _setup():
    bits = synth.qwen_params(CFG, seed=4, varied=True)
    theta = oracle.core.bf16_to_f32(bits).astype(np.float64)
    lay = oracle.qwen.layout(CFG)
    tokens, _ = synth.opt_batch(CFG, 1, 48, seed=4)

    def view(name):
        off, shape = lay[name]
        return theta[off:off + int(np.prod(shape))].reshape(shape)

    E_rows = view("E")[tokens[0]]
    blocks = lambda li: {n: view(f"L{li}.{n}") for n in oracle.qwen.LAYER_FIELDS}  # noqa: E731
    return theta, tokens, E_rows, blocks


def test_round_bf16_matches_torch():
    x = np.random.default_rng(0).standard_normal(10000) * np.logspace(-30, 30, 10000)
    x[:4] = [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8]  # ties round to even
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(round_bf16(x), ref)


def test_without_rounding_it_is_the_exact_forward():
    theta, tokens, E_rows, blocks = _setup()
    for n in (1, 3):
        ref = oracle.qwen.hidden_states(theta, CFG, tokens, n_layers=n)[0]
        got = qwen_hidden_states(E_rows, blocks, CFG, n, rounding=False)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_rounding_moves_the_hidden_states_by_about_bf16_precision():
    theta, tokens, E_rows, blocks = _setup()
    ref = oracle.qwen.hidden_states(theta, CFG, tokens, n_layers=3)[0]
    got = qwen_hidden_states(E_rows, blocks, CFG, 3)
    err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 2.0 ** -12 < err < 2.0 ** -4, err
