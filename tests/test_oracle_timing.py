"""The oracle timing helpers behind the benchmark's CPU baseline: they run the unmodified
oracle functions on small samples, and their command-line worker works."""
import json
import os
import subprocess
import sys

import numpy as np

import oracle
import oracle.timing
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_timed_steps_are_plain_oracle_steps():
    r = oracle.timing.quad_steps(4096, 5, 8, 1e-3, 4e-7, 1e-3, warmup=1, steps=2)
    assert len(r["times"]) == 2 and all(t > 0 for t in r["times"])
    assert r["t_end"] >= r["t_start"]


def test_element_rates_positive():
    r = oracle.timing.element_rates(1 << 12, 1 << 10, (16, 160))
    assert r["perturb"] > 0 and set(r["update"]) == {"16", "160"}
    assert all(v > 0 for v in r["update"].values())


def test_worker_command_line():
    out = subprocess.run([sys.executable, "-m", "oracle.timing", "steps", "2048", "1", "8",
                          "1e-3", "4e-7", "1e-3", "0", "1"], cwd=ROOT, capture_output=True,
                         text=True, check=True).stdout
    r = json.loads(out.strip().splitlines()[-1])
    assert len(r["times"]) == 1
    cfg = dict(synth.OPT_CONFIGS["opt-125m"], n_layers=1, d_model=64, n_heads=4, d_ffn=128,
               vocab=4096)
    out = subprocess.run([sys.executable, "-m", "oracle.timing", "forward", "opt",
                          json.dumps(cfg), "16"], cwd=ROOT, capture_output=True, text=True,
                         check=True).stdout
    assert json.loads(out.strip().splitlines()[-1])["tokens_per_s"] > 0


def test_forward_timing_runs_the_oracle_loss():
    cfg = dict(synth.QWEN_CONFIGS["qwen3-1.7b"], n_layers=1, d_model=64, n_heads=4,
               n_kv_heads=2, head_dim=16, d_ffn=128, vocab=4096)
    assert oracle.timing.forward_tokens_per_s("qwen3", cfg, 8) > 0
    # the same inputs give a finite oracle loss
    bits = synth.qwen_params(cfg)
    theta = (bits.astype(np.uint32) << 16).view(np.float32)
    tok, lab = synth.opt_batch(cfg, 1, 8)
    assert np.isfinite(oracle.qwen.loss(theta, cfg, tok, lab))


def test_mlp_step_timing():
    r = oracle.timing.mlp_steps(1)
    assert len(r["times"]) == 1 and r["times"][0] > 0
