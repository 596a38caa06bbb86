"""Timing of the oracle as it stands, for the benchmark's CPU baseline.

TEST INFRASTRUCTURE, like the rest of this package: only the benchmark's CPU-baseline and
reference legs run it.  Nothing here changes what the oracle computes; it times the
unmodified functions on samples of the benchmark's workloads, either in the calling process
or as a command-line worker that the benchmark starts once per host core (independent
processes on disjoint samples, each single-threaded).

  python -m oracle.timing steps M_SAMPLE SEED N_PERT EPS LR DAMPING WARMUP STEPS
  python -m oracle.timing forward FAMILY CFG_JSON SEQ
  python -m oracle.timing mlp STEPS
  python -m oracle.timing forward_samples FAMILY CFG_JSON SEQ WARMUP STEPS

print one JSON object on stdout.
"""
import json
import sys
import time

import numpy as np


def quad_steps(M_sample, seed, n_pert, eps, lr, damping, warmup, steps):
    """warmup + steps full 1.5-SPSA steps of the oracle on a diagonal quadratic of M_sample
    elements (the benchmark workload's distribution, sample `seed`).  Returns the seconds of
    each timed step and the wall-clock bounds of the timed phase."""
    import synth

    from . import core, step
    th, D = synth.quad_problem(M_sample, seed=seed)

    def loss(P):
        return core.quad_loss(P, D)

    times, t_start = [], None
    for s in range(warmup + steps):
        if s == warmup:
            t_start = time.time()
        t0 = time.perf_counter()
        th, _ = step.spsa_step(th, loss, n_pert, eps, lr, damping, seed, s, update="mirror")
        if s >= warmup:
            times.append(time.perf_counter() - t0)
    return {"times": times, "t_start": t_start, "t_end": time.time()}


def mlp_steps(steps, n_pert=16, eps=1e-3, lr=1e-2, damping=1e-3):
    """Seconds of each of `steps` full oracle steps of the MLP workload (64-256-10, batch 64,
    teacher labels), after one untimed step."""
    import synth

    from . import mlp, step
    P = synth.mlp_params(0)
    teacher = synth.mlp_params(0, tag="teacher")
    times, t_start = [], None
    for k in range(steps + 1):
        X, y = synth.mlp_batch(0, k, teacher)
        if k == 1:
            t_start = time.time()
        t0 = time.perf_counter()
        P, _ = step.spsa_step(P, lambda Q: mlp.loss(Q, X, y), n_pert, eps, lr, damping, 0, k)
        if k:
            times.append(time.perf_counter() - t0)
    return {"times": times, "t_start": t_start, "t_end": time.time()}


def element_rates(M_perturb, M_update, ns):
    """Elements per second of the oracle's perturbation (one probe, one sign) and of its
    fp32-order update with n regenerated probes, for each n in ns (one thread)."""
    import synth

    from . import core
    th, _ = synth.quad_problem(max(M_perturb, M_update), seed=1)
    t0 = time.perf_counter()
    core.perturb(th[:M_perturb], 0, 0, 3, +1, 1e-3)
    out = {"perturb": M_perturb / (time.perf_counter() - t0), "update": {}}
    for n in ns:
        a = synth.coefficients(n)
        t0 = time.perf_counter()
        core.update_mirror(th[:M_update], a, 0, 0)
        out["update"][str(n)] = M_update / (time.perf_counter() - t0)
    return out


def forward_tokens_per_s(family, cfg, seq, batch=1):
    """Tokens per second of the oracle's decoder loss (fp64) at the given configuration."""
    import synth

    from . import opt, qwen
    if family == "qwen3":
        mod, bits = qwen, synth.qwen_params(cfg)
    else:
        mod, bits = opt, synth.opt_params(cfg)
    theta = (bits.astype(np.uint32) << 16).view(np.float32)
    tokens, labels = synth.opt_batch(cfg, batch, seq)
    t0 = time.perf_counter()
    mod.loss(theta, cfg, tokens, labels)
    return batch * seq / (time.perf_counter() - t0)


def forward_samples(family, cfg, seq, warmup, steps):
    """warmup + steps timed evaluations of the oracle's decoder loss (fp64) at the given
    configuration on one sequence of `seq` tokens, the weights generated once beforehand;
    returns the seconds of each timed evaluation and the wall-clock bounds of the timed phase."""
    import synth

    from . import opt, qwen
    if family == "qwen3":
        mod, bits = qwen, synth.qwen_params(cfg)
    else:
        mod, bits = opt, synth.opt_params(cfg)
    theta = (bits.astype(np.uint32) << 16).view(np.float32)
    del bits
    tokens, labels = synth.opt_batch(cfg, 1, seq)
    times, t_start = [], None
    for s in range(warmup + steps):
        if s == warmup:
            t_start = time.time()
        t0 = time.perf_counter()
        mod.loss(theta, cfg, tokens, labels)
        if s >= warmup:
            times.append(time.perf_counter() - t0)
    return {"times": times, "t_start": t_start, "t_end": time.time()}


def _main(argv):
    if argv[0] == "steps":
        M, seed, n, eps, lr, lam, w, k = argv[1:9]
        res = quad_steps(int(M), int(seed), int(n), float(eps), float(lr), float(lam), int(w), int(k))
    elif argv[0] == "mlp":
        res = mlp_steps(int(argv[1]))
    elif argv[0] == "forward":
        cfg = json.loads(argv[2])
        if "class_ids" in cfg:
            cfg["class_ids"] = tuple(cfg["class_ids"])
        res = {"tokens_per_s": forward_tokens_per_s(argv[1], cfg, int(argv[3]))}
    elif argv[0] == "forward_samples":
        cfg = json.loads(argv[2])
        if "class_ids" in cfg:
            cfg["class_ids"] = tuple(cfg["class_ids"])
        res = forward_samples(argv[1], cfg, int(argv[3]), int(argv[4]), int(argv[5]))
    else:
        raise SystemExit("usage: python -m oracle.timing steps|forward|forward_samples|mlp ...")
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    _main(sys.argv[1:])
