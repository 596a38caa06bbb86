"""Pins of the Qwen3-shaped decoder oracle (oracle/qwen.py) against transformers'
Qwen3ForCausalLM in fp64 on CPU (an independent implementation of the architecture), plus
causality and grouped-query structure."""
import numpy as np
import pytest

import oracle
import synth

TINY = dict(family="qwen3", n_layers=2, d_model=64, n_heads=4, n_kv_heads=2, head_dim=32,
            d_ffn=96, vocab=101, max_pos=32, rope_theta=1.0e4, norm_eps=1e-6, class_ids=(7, 9))


def _theta(cfg, seed=0):
    return oracle.core.bf16_to_f32(synth.qwen_params(cfg, seed=seed, varied=True)).astype(np.float64)


def _hf(cfg, theta):
    torch = pytest.importorskip("torch")
    transformers = pytest.importorskip("transformers")
    conf = transformers.Qwen3Config(
        vocab_size=cfg["vocab"], hidden_size=cfg["d_model"], intermediate_size=cfg["d_ffn"],
        num_hidden_layers=cfg["n_layers"], num_attention_heads=cfg["n_heads"],
        num_key_value_heads=cfg["n_kv_heads"], head_dim=cfg["head_dim"],
        max_position_embeddings=cfg["max_pos"], rms_norm_eps=cfg["norm_eps"],
        rope_theta=cfg["rope_theta"], tie_word_embeddings=True, attention_bias=False,
        attention_dropout=0.0, use_sliding_window=False)
    model = transformers.Qwen3ForCausalLM(conf).double().eval()
    model.config._attn_implementation = "eager"
    lay = oracle.qwen.layout(cfg)
    H, Hk, e, f = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["d_ffn"]

    def get(name):
        off, shape = lay[name]
        return torch.tensor(theta[off:off + int(np.prod(shape))].reshape(shape), dtype=torch.float64)

    sd = {"model.embed_tokens.weight": get("E"), "model.norm.weight": get("final_norm")}
    for l in range(cfg["n_layers"]):
        p = f"model.layers.{l}."
        w = get(f"L{l}.wqkv")
        sd[p + "self_attn.q_proj.weight"] = w[:H * e]
        sd[p + "self_attn.k_proj.weight"] = w[H * e:(H + Hk) * e]
        sd[p + "self_attn.v_proj.weight"] = w[(H + Hk) * e:]
        sd[p + "self_attn.q_norm.weight"] = get(f"L{l}.q_norm")
        sd[p + "self_attn.k_norm.weight"] = get(f"L{l}.k_norm")
        sd[p + "self_attn.o_proj.weight"] = get(f"L{l}.wo")
        sd[p + "input_layernorm.weight"] = get(f"L{l}.in_norm")
        sd[p + "post_attention_layernorm.weight"] = get(f"L{l}.post_norm")
        gu = get(f"L{l}.wgu")
        sd[p + "mlp.gate_proj.weight"] = gu[:f]
        sd[p + "mlp.up_proj.weight"] = gu[f:]
        sd[p + "mlp.down_proj.weight"] = get(f"L{l}.wd")
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected, unexpected
    assert all(m.startswith("lm_head") for m in missing), missing
    model.tie_weights()
    return model


@pytest.mark.parametrize("cfg", [TINY, dict(TINY, n_heads=2, n_kv_heads=1, head_dim=64, n_layers=3)])
def test_qwen_decoder_matches_transformers(cfg):
    torch = pytest.importorskip("torch")
    theta = _theta(cfg)
    tokens, labels = synth.opt_batch(cfg, 3, 11, seed=2)
    ours = oracle.qwen.per_sample_loss(theta, cfg, tokens, labels)
    model = _hf(cfg, theta)
    with torch.no_grad():
        logits = model(input_ids=torch.tensor(tokens, dtype=torch.long)).logits[:, -1, :]
    ref = torch.nn.functional.cross_entropy(logits[:, list(cfg["class_ids"])],
                                            torch.tensor(labels, dtype=torch.long),
                                            reduction="none").numpy()
    # transformers builds its rotary cos/sin tables in fp32 even for an fp64 model (the
    # oracle uses fp64 angles): agreement is ~1e-8; a wrong rotation, norm or head mapping
    # moves the loss by 1e-3 or more.
    assert np.allclose(ours, ref, rtol=1e-6, atol=1e-9)


def test_qwen_decoder_is_causal():
    theta = _theta(TINY, seed=3)
    tokens, _ = synth.opt_batch(TINY, 2, 9, seed=4)
    h = oracle.qwen.hidden_states(theta, TINY, tokens)
    t2 = tokens.copy()
    t2[:, 5] = (t2[:, 5] + 1) % TINY["vocab"]
    h2 = oracle.qwen.hidden_states(theta, TINY, t2)
    assert np.array_equal(h[:, :5], h2[:, :5]) and not np.allclose(h[:, 5:], h2[:, 5:])
