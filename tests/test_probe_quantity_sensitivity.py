"""The GPU test of the per-probe quantities (test_gpu_decoder.py::test_probe_quantities_match_oracle)
can fail on an error confined to the head: planted here in the oracle, on the CPU.

If the final LayerNorm and the two tied class rows were read unperturbed (an error in the
head's on-load perturbation), the directional derivatives g_i = (L+ - L-)/(2 eps) of the tiny
decoder would move by far more than the tolerance the GPU test allows, and at least one would
change sign."""
import numpy as np

import oracle
import synth
from oracle import core
from probe_tolerances import G_TOL

CFG = dict(n_layers=2, d_model=128, n_heads=2, d_ffn=512, vocab=1000, max_pos=128, class_ids=(3, 7))


def test_head_perturbation_error_exceeds_the_gpu_tolerance():
    B, S, n, eps = 4, 64, 8, 1e-3
    bits = synth.opt_params(CFG, seed=1, varied=True)
    tokens, labels = synth.opt_batch(CFG, B, S, seed=1)
    lay = oracle.opt.layout(CFG)
    d = CFG["d_model"]
    fin = lay["lnf.g"][0]
    head = np.concatenate([np.arange(fin, fin + 2 * d)] +
                          [np.arange(c * d, c * d + d) for c in CFG["class_ids"]])
    loss = lambda Pb: oracle.opt.loss(core.bf16_to_f32(Pb).astype(np.float64), CFG, tokens, labels)  # noqa: E731
    e32 = float(np.float32(eps))
    g, g_bad = np.zeros(n), np.zeros(n)
    for i in range(n):
        Pp, Pm = core.perturb(bits, 1, 0, i, +1, e32), core.perturb(bits, 1, 0, i, -1, e32)
        g[i] = (loss(Pp) - loss(Pm)) / (2 * e32)
        Pp[head], Pm[head] = bits[head], bits[head]  # the planted error
        g_bad[i] = (loss(Pp) - loss(Pm)) / (2 * e32)
    assert np.max(np.abs(g - g_bad)) > 5 * G_TOL
    assert np.any(np.sign(g) != np.sign(g_bad))
