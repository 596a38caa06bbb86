"""Tolerances of the GPU test of the per-probe quantities (the tiny OPT-shaped decoder of
test_gpu_decoder.py::test_probe_quantities_match_oracle, 4 x 64 tokens, 8 probes).

Measured on B200 with this configuration (max over the probes, GPU losses from the bf16
forward against the oracle's fp64 losses): at eps = 1e-3, |g_gpu - g_oracle| <= 0.27 with
|g| between 2.4 and 34 (a second configuration of the same size: <= 0.58), the signs
always equal; c_i = (L+ + L- - 2 L0)/eps^2 is dominated by the forward's rounding at that eps
(errors up to a few thousand), and at eps = 1e-2, |c_gpu - c_oracle| <= 12 with |c| up to
2600 (the largest relative error, 4.4%, on a probe with |c| = 60, moves its weight w by
0.44%).  The bounds keep a margin of at least 4 over those measurements; an error confined to the
head's on-load perturbation moves g by up to 13 on this model
(test_probe_quantity_sensitivity.py)."""
G_TOL = 1.0      # |g_gpu - g_oracle| at eps = 1e-3
C_REL_TOL = 2e-2  # |c_gpu - c_oracle| / max |c_oracle| at eps = 1e-2
W_REL_TOL = 2e-2  # |w_gpu / w_oracle - 1| at eps = 1e-2
