"""Pins of the decoder oracle (oracle/opt.py) against an independent implementation of
the OPT architecture (HuggingFace transformers' OPTForCausalLM, fp64 on CPU) and
against structural invariants (causality, batch permutation, softmax normalisation)."""
import numpy as np
import pytest

import oracle
import synth

TINY = dict(n_layers=2, d_model=64, n_heads=2, d_ffn=128, vocab=97, max_pos=16, class_ids=(5, 11))


def _theta(cfg, seed=0):
    return oracle.core.bf16_to_f32(synth.opt_params(cfg, seed=seed, varied=True)).astype(np.float64)


def _hf_model(cfg, theta):
    torch = pytest.importorskip("torch")
    transformers = pytest.importorskip("transformers")
    d, f = cfg["d_model"], cfg["d_ffn"]
    conf = transformers.OPTConfig(
        vocab_size=cfg["vocab"], hidden_size=d, num_hidden_layers=cfg["n_layers"], ffn_dim=f,
        num_attention_heads=cfg["n_heads"], max_position_embeddings=cfg["max_pos"],
        do_layer_norm_before=True, word_embed_proj_dim=d, activation_function="relu",
        enable_bias=True, layer_norm_elementwise_affine=True, dropout=0.0,
        attention_dropout=0.0, activation_dropout=0.0, layerdrop=0.0,
        pad_token_id=1, bos_token_id=2, eos_token_id=2, tie_word_embeddings=True)
    model = transformers.OPTForCausalLM(conf).double().eval()
    lay = oracle.opt.layout(cfg)

    def get(name):
        off, shape = lay[name]
        return torch.tensor(theta[off:off + int(np.prod(shape))].reshape(shape), dtype=torch.float64)

    sd = {"model.decoder.embed_tokens.weight": get("E"),
          "model.decoder.embed_positions.weight": get("Pos"),
          "model.decoder.final_layer_norm.weight": get("lnf.g"),
          "model.decoder.final_layer_norm.bias": get("lnf.b")}
    for l in range(cfg["n_layers"]):
        p = f"model.decoder.layers.{l}."
        wqkv, bqkv = get(f"L{l}.wqkv"), get(f"L{l}.bqkv")
        for i, nm in enumerate(("q_proj", "k_proj", "v_proj")):
            sd[p + f"self_attn.{nm}.weight"] = wqkv[i * d:(i + 1) * d]
            sd[p + f"self_attn.{nm}.bias"] = bqkv[i * d:(i + 1) * d]
        sd[p + "self_attn.out_proj.weight"] = get(f"L{l}.wo")
        sd[p + "self_attn.out_proj.bias"] = get(f"L{l}.bo")
        sd[p + "self_attn_layer_norm.weight"] = get(f"L{l}.ln1g")
        sd[p + "self_attn_layer_norm.bias"] = get(f"L{l}.ln1b")
        sd[p + "fc1.weight"] = get(f"L{l}.w1")
        sd[p + "fc1.bias"] = get(f"L{l}.b1")
        sd[p + "fc2.weight"] = get(f"L{l}.w2")
        sd[p + "fc2.bias"] = get(f"L{l}.b2")
        sd[p + "final_layer_norm.weight"] = get(f"L{l}.ln2g")
        sd[p + "final_layer_norm.bias"] = get(f"L{l}.ln2b")
    missing, unexpected = model.load_state_dict(sd, strict=False)
    assert not unexpected, unexpected
    assert all(m.startswith("lm_head") for m in missing), missing
    model.tie_weights()
    return model


@pytest.mark.parametrize("cfg", [TINY, dict(TINY, n_layers=3, d_model=128, n_heads=1, d_ffn=64)])
def test_decoder_matches_transformers_opt(cfg):
    torch = pytest.importorskip("torch")
    theta = _theta(cfg)
    tokens, labels = synth.opt_batch(cfg, 3, 12, seed=1)
    ours = oracle.opt.per_sample_loss(theta, cfg, tokens, labels)
    model = _hf_model(cfg, theta)
    with torch.no_grad():
        logits = model(input_ids=torch.tensor(tokens, dtype=torch.long)).logits[:, -1, :]
    two = logits[:, list(cfg["class_ids"])]
    ref = torch.nn.functional.cross_entropy(two, torch.tensor(labels, dtype=torch.long),
                                            reduction="none").numpy()
    assert np.allclose(ours, ref, rtol=1e-10, atol=1e-12)
    # the full logits row agrees too (tied head over the whole vocabulary)
    lay = oracle.opt.layout(cfg)
    h = oracle.opt.hidden_states(theta, cfg, tokens)
    off, shape = lay["lnf.g"]
    g = theta[off:off + cfg["d_model"]]
    off, _ = lay["lnf.b"]
    b = theta[off:off + cfg["d_model"]]
    xl = h[:, -1]
    xl = (xl - xl.mean(-1, keepdims=True)) / np.sqrt(xl.var(-1, keepdims=True) + 1e-5) * g + b
    E = theta[:cfg["vocab"] * cfg["d_model"]].reshape(cfg["vocab"], cfg["d_model"])
    assert np.allclose(xl @ E.T, logits.numpy(), rtol=1e-10, atol=1e-12)


def test_decoder_is_causal_and_batch_equivariant():
    cfg = TINY
    theta = _theta(cfg, seed=2)
    tokens, labels = synth.opt_batch(cfg, 4, 10, seed=3)
    h = oracle.opt.hidden_states(theta, cfg, tokens)
    t2 = tokens.copy()
    t2[:, 6] = (t2[:, 6] + 1) % cfg["vocab"]
    h2 = oracle.opt.hidden_states(theta, cfg, t2)
    assert np.array_equal(h[:, :6], h2[:, :6])         # positions before 6 are unaffected
    assert not np.allclose(h[:, 6:], h2[:, 6:])
    perm = np.array([2, 0, 3, 1])
    a = oracle.opt.per_sample_loss(theta, cfg, tokens, labels)
    b = oracle.opt.per_sample_loss(theta, cfg, tokens[perm], labels[perm])
    assert np.allclose(a[perm], b, rtol=1e-13, atol=0)


def test_two_class_loss_is_log2_for_equal_logits():
    """With identical class-token embeddings the two logits are equal: every loss is ln 2."""
    cfg = dict(TINY, class_ids=(5, 6))
    theta = _theta(cfg, seed=4)
    d = cfg["d_model"]
    theta[6 * d:7 * d] = theta[5 * d:6 * d]
    tokens, labels = synth.opt_batch(cfg, 3, 8, seed=5)
    assert np.allclose(oracle.opt.per_sample_loss(theta, cfg, tokens, labels), np.log(2.0),
                       rtol=1e-12)
