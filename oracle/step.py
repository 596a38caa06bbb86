"""One 1SPSA / 1.5-SPSA step, composed from the oracle's parts in the pages' order.

TEST INFRASTRUCTURE (see oracle/__init__.py).  The loop follows the training-loop
flowchart of "Pretraining Transformers Without Backprop: What Two Zero-Order Papers
Actually Measure" (section "Backprop's memory tax"): draw the step's probes, evaluate
the loss only (no backward pass) at the perturbed weights, form the probe-space
preconditioned estimate, update the weights, repeat.  1.5-SPSA adds the clean loss
("Stanford's 1.5-SPSA Trains OPT-30B Without Backpropagation", section
"Probe-Space Preconditioning").
"""
import numpy as np

from . import core


def spsa_step(theta, loss_fn, n_pert, eps, lr, damping, seed, step, preconditioned=True,
              alpha=0.1, update="f64"):
    """Returns (theta_next, record).  theta is float32 or bf16 bits (uint16).

    loss_fn(P) -> float evaluates the loss at a parameter vector of theta's dtype.
    update = "f64" sums the probes in fp64; "mirror" uses the fixed fp32 order.
    On a non-finite loss theta is returned unchanged and record["ok"] is False.
    """
    eps32 = float(np.float32(eps))
    L0 = loss_fn(theta) if preconditioned else None
    Lp = np.zeros(n_pert)
    Lm = np.zeros(n_pert)
    for i in range(n_pert):
        Lp[i] = loss_fn(core.perturb(theta, seed, step, i, +1, eps32))
        Lm[i] = loss_fn(core.perturb(theta, seed, step, i, -1, eps32))
    pc = core.precond(Lp, Lm, L0, eps32, float(np.float32(lr)), float(np.float32(damping)),
                      float(np.float32(alpha)))
    rec = {"L0": L0, "Lp": Lp, "Lm": Lm, "ok": pc is not None}
    if pc is None:
        return np.array(theta, copy=True), rec
    rec.update(pc)
    if update == "f64":
        nxt = core.update_f64(theta, pc["a"], seed, step)
    elif update == "mirror":
        nxt = core.update_mirror(theta, pc["a"].astype(np.float32), seed, step)
    else:
        raise ValueError(update)
    return nxt, rec
