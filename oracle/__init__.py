"""CPU oracle for the 1SPSA / 1.5-SPSA zero-order training step.

TEST INFRASTRUCTURE.  Plain, slow, obviously-correct reference code: a C library
(zo_oracle.c: Philox probes, perturbation, quadratic loss, preconditioner, update) and
numpy code (MLP, decoder and low-rank losses, the step driver); `timing` times these
functions unchanged for the benchmark's CPU baselines.  Only the tests, the smoke
check and the benchmark's CPU-baseline and reference legs may import it.  It shares no code
with the CUDA library and neither imports the other; both take their inputs from `synth`.
"""
from . import core, lowrank, mlp, opt, qwen, step  # noqa: F401
