#!/usr/bin/env python
"""Benchmark of one 1.5-SPSA step of the diagonal-quadratic workload on B200.

Workload (the default, one GPU): L = 1/2 sum_j D_j theta_j^2 with M = 2^24 fp32
parameters, D_j log-uniform in [1e-3, 1e3], theta_0 ~ N(0, 1); n_pert = 64,
eps = 1e-3, lr = 4e-7, damping = 1e-3, 1.5-SPSA.  One step = clean loss + 2*n_pert
perturbed losses (the 128 losses of each eight probe octets from one pass over theta and D) +
preconditioner + update, all through the C ABI of libzo.so.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload quadratic|mlp|opt-125m|opt-1.3b|opt-30b|qwen3-1.7b|qwen3-8b]

The decoder workloads (OPT- or Qwen3-shaped, bf16 weights N(0, 0.02), uniform tokens,
2-class last-token loss) time whole 1.5-SPSA steps through zo_model_step and add a
per-GEMM-shape breakdown of the tcgen05 projections against the measured bf16 peak.

Prints ONE JSON line (rank 0).  With N > 1 (torchrun, one rank per GPU) the ranks share
one model ("scaling": "strong"): every rank holds a contiguous slice of theta and D (its
element offset keeps the global probe signs), evaluates all 2*n_pert + 1 losses over its
slice's terms, the partial losses are all-gathered over NCCL and summed in rank order (the
same bits everywhere), and every rank runs the preconditioner and updates its slice; the
step time is the max over ranks.  `--impl reference` times the CPU oracle on bounded
samples of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "1.5-SPSA steps/s & probe fwd tokens/s; perturb/update HBM GB/s as % of peak"
M_FULL = 1 << 24
N_PERT, EPS, LR, DAMPING = 64, 1e-3, 4e-7, 1e-3
WORKLOAD = ("diagonal quadratic L=1/2*sum D_j theta_j^2, M=2^24 fp32, D log-uniform [1e-3,1e3], "
            "theta0~N(0,1); 1.5-SPSA n_pert=64 eps=1e-3 lr=4e-7 damping=1e-3")
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (read + write) per launch of the octet loss kernel from the ncu capture
# summarised in profiles/quad_octet_kernel.quadratic_M2p24.md, valid for the kernel sources
# whose SHA-256 (of zo_loss.cu and zo_internal.cuh, concatenated) is recorded with it;
# reported as null when a source has changed since the capture.
LOSS_TRAFFIC = {"sources_sha256": "d1b68b988680111f9d369faf40a77a5e8e770b8100af06f1e229ee733b2a03b3",
                "bytes": 139.3e6}
LOSS_SOURCES = ("zo_loss.cu", "zo_internal.cuh")
# Warp instructions one launch of the loss kernel executes (ncu smsp__inst_executed.sum, same
# capture and validity rule as LOSS_TRAFFIC): the pass is bound by instruction issue, so its
# roofline is the issue limit, 148 SMs x 4 warp-instructions per clock at the sampled clock.
LOSS_WARP_INSTRUCTIONS = 90.41e6
SM_COUNT, ISSUE_PER_SM_CLOCK = 148, 4


def loss_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for name in LOSS_SOURCES:
        with open(os.path.join(ROOT, "zero_order_forward_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def loss_traffic():
    try:
        h = loss_sources_sha256()
    except OSError:
        return None
    return LOSS_TRAFFIC["bytes"] if h == LOSS_TRAFFIC["sources_sha256"] else None


FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED = 1590.0, 1400.0

DECODER_WORKLOADS = {
    # model shape, micro-batch, micro-batches per effective batch, probes per step
    "opt-125m": dict(batch=16, seq=256, n_micro=1, n_pert=32),
    "opt-1.3b": dict(batch=16, seq=512, n_micro=8, n_pert=160),
    "opt-30b": dict(batch=8, seq=2048, n_micro=1, n_pert=16),
    "qwen3-1.7b": dict(batch=16, seq=512, n_micro=1, n_pert=32),
    "qwen3-8b": dict(batch=8, seq=1024, n_micro=1, n_pert=16),
}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def bf16_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


# ------------------------------------------------------------------ CPU oracle timing

def time_oracle(M_sample, n_steps, seed=0):
    """Times the oracle's full step on the first M_sample elements of the workload.
    Returns seconds per sample step (single-threaded C + numpy)."""
    import oracle
    import synth
    th, D = synth.quad_problem(M_sample, seed=seed)
    loss = lambda P: oracle.core.quad_loss(P, D)  # noqa: E731
    times = []
    for s in range(n_steps):
        t0 = time.perf_counter()
        th, _ = oracle.step.spsa_step(th, loss, N_PERT, EPS, LR, DAMPING, seed, s, update="mirror")
        times.append(time.perf_counter() - t0)
    return times


def host_cpu():
    """The host's CPU model and logical core count (for the CPU baselines' context)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "logical_cores": os.cpu_count()}


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_workers(jobs, threads=1, timeout=900):
    """Runs `python -m oracle.timing <job...>` once per job, all concurrently, each limited to
    `threads` BLAS/OpenMP threads; returns their JSON results in job order."""
    env = dict(os.environ, OMP_NUM_THREADS=str(threads), OPENBLAS_NUM_THREADS=str(threads),
               MKL_NUM_THREADS=str(threads))
    procs = [subprocess.Popen([sys.executable, "-m", "oracle.timing"] + [str(a) for a in job],
                              cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                              text=True) for job in jobs]
    out = []
    for p in procs:
        o, e = p.communicate(timeout=timeout)
        if p.returncode:
            raise RuntimeError("oracle worker failed: " + e[-400:])
        out.append(json.loads(o.strip().splitlines()[-1]))
    return out


def oracle_all_cores(M_sample, warmup, steps, max_procs=32):
    """Oracle steps on every host core: one single-threaded process per core (at most
    max_procs), each on its own M_sample-element sample of the workload.  Returns
    (steps/s of the full workload, processes): total work / the union of the timed phases."""
    P = max(1, min(host_cores(), max_procs))
    res = oracle_workers([("steps", M_sample, 100 + i, N_PERT, EPS, LR, DAMPING, warmup, steps)
                          for i in range(P)])
    wall = max(r["t_end"] for r in res) - min(r["t_start"] for r in res)
    return P * steps * (M_sample / M_FULL) / wall, P


def reference_arm(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    # the sample per step shrinks with the step count so that the run stays near 30 s: a
    # power of two <= 2^18 elements, from a calibration step on 2^12
    t_cal = min(time_oracle(1 << 12, 2))
    per_elem = t_cal / (1 << 12)
    M_sample = 1 << 18
    while M_sample > (1 << 10) and per_elem * M_sample * (args.warmup + args.steps) > 30.0:
        M_sample >>= 1
    # every host core runs the oracle as it stands (single-threaded) on its own sample
    value, P = oracle_all_cores(M_sample, args.warmup, args.steps)
    lg = M_sample.bit_length() - 1
    sample = (f"{P} concurrent single-threaded oracle processes, each {args.steps} timed steps "
              f"after {args.warmup} warm-up on its own 2^{lg}-element sample of the workload "
              f"(1/{M_FULL // M_sample} of 2^24 parameters); full-workload steps/s = total "
              f"sample steps / wall time, scaled by 1/{M_FULL // M_sample}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 / value, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M_FULL, "n_pert": N_PERT},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": P, "kind": "oracle",
                             "sample": sample, "host": host_cpu()},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        """Starts sampling every 20 ms and returns once the first sample is in, so that the
        samples cover the region that follows."""
        import threading
        self.proc, self.lines = None, []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        self._wait_for(1, 10.0)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def _wait_for(self, n, timeout):
        t0 = time.perf_counter()
        while len(self.lines) < n and time.perf_counter() - t0 < timeout:
            time.sleep(0.005)

    def stop(self):
        """Takes one more sample after the region (so that a short region is bracketed),
        then stops."""
        if self.proc is None:
            return None
        self._wait_for(len(self.lines) + 1, 2.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.reader.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm

def gpu_arm(args):
    import torch
    import torch.distributed as dist

    import synth
    import zero_order_forward_b200 as zo

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    hbm_peak, peak_kind = peaks()

    th_np, D_np = synth.quad_problem(M_FULL, seed=0)  # one shared model across ranks
    # N > 1: every rank holds a contiguous slice of theta and D (its element offset keeps the
    # global probe signs); the quadratic's loss is the sum of the slices' losses
    first, count = 0, M_FULL
    if world > 1:
        from zero_order_forward_b200 import dist as zdist
        first, count = zdist.shard_range(M_FULL, rank, world)
    theta = torch.from_numpy(th_np[first:first + count]).to(dev)
    D = torch.from_numpy(D_np[first:first + count]).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n = N_PERT
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream(dev)
    ctx = zo.zo_create(theta, seed=0, stream=stream.cuda_stream)
    if first:
        zo.zo_set_element_offset(ctx, first)
    n_oct = (n + 63) // 64  # loss passes per step (64 probes each)

    def apply_step(Lp, Lm, L0):
        zo.zo_step(ctx, Lp, Lm, n, L0, LR, EPS, DAMPING)

    def partial_losses(out):  # all 2n + 1 losses over this rank's slice, L0 in the first pass
        for o in range(n_oct):
            c = min(64, n - 64 * o)
            zo.zo_quad_loss_octet(ctx, D, 64 * o, c, EPS, out[1 + 64 * o:1 + 64 * o + c],
                                  out[1 + n + 64 * o:1 + n + 64 * o + c],
                                  out[0:1] if o == 0 else None)

    def one_step():
        if world > 1:  # element-parallel: partial losses, all-gather + rank-order sum, slice update
            zdist.element_parallel_step(n, partial_losses, apply_step, dev)
        else:  # the native step driver: every launch of the step enqueued from C++
            zo.zo_quad_step(ctx, D, n, EPS, LR, DAMPING, True, losses)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    for k in range(args.steps):
        flush.zero_()  # evict theta and D from the 126 MB L2 between steps (not timed)
        evs[k][0].record(stream)
        one_step()
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    zo.zo_sync(ctx)

    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    n_ph = 0
    if world == 1:
        # The per-phase (and so per-kernel) durations come from further identical steps with
        # the library's phase events: those events sit between the step's launches and cost
        # the programmatic-launch overlap (about 9 us per step), so the timed steps above run
        # without them.
        n_ph = min(args.steps, 50)
        zo.zo_enable_phase_timing(ctx, n_ph)
        for _ in range(n_ph):
            flush.zero_()
            one_step()
        torch.cuda.synchronize()
        ph = zo.zo_phase_times(ctx, n_ph)
        zo.zo_enable_phase_timing(ctx, 0)
        clean_ms, probe_ms, upd_ms = (list(map(float, ph[:, i])) for i in range(3))
    else:
        clean_ms = probe_ms = upd_ms = [float("nan")]
    total_s = sum(step_ms) / 1e3
    if world > 1:
        t = torch.tensor([total_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_s = float(t.item())
    value = args.steps / total_s  # steps of the one shared model

    # dominant kernel: the loss pass (perturbation on load).  At one GPU the probe phase
    # holds n/64 launches of the octet kernel (the 128 losses L(theta +- eps z_i) of eight
    # probe octets from one pass over theta and D); with N ranks the phase is not bracketed
    # separately: time the kernel alone.
    if world > 1:
        le = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        flush.zero_()
        le[0].record(stream)
        for o in range(n_oct):
            zo.zo_quad_loss_octet(ctx, D, 64 * o, min(64, n - 64 * o), EPS, losses[1:65],
                                  losses[65:129], losses[0:1] if o == 0 else None)
        le[1].record(stream)
        torch.cuda.synchronize()
        probe_ms = [le[0].elapsed_time(le[1])]
    loss_us = 1e3 * statistics.mean(probe_ms) / n_oct
    loss_bytes = 8 * count  # this rank's theta and D read once per pass, fp32
    achieved = loss_bytes / (loss_us * 1e-6) / 1e9
    upd_bytes = 8 * count  # theta read + written, fp32

    # the one-probe form (both signs of one probe per pass), timed alone for comparison
    pe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    flush.zero_()
    pe[0].record(stream)
    for i in range(n):
        zo.zo_quad_loss_pair(ctx, D, i, EPS, losses[1:2], losses[2:3])
    pe[1].record(stream)
    torch.cuda.synchronize()
    pair_us = 1e3 * pe[0].elapsed_time(pe[1]) / n

    # single-kernel timing of the update (same stream), for its own roofline
    coef = torch.from_numpy(synth.coefficients(n, seed=1) * 0).to(dev)  # zero: theta unchanged
    ue = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    flush.zero_()
    ue[0].record(stream)
    reps = 10
    for _ in range(reps):
        zo.zo_update(ctx, coef, n)
    ue[1].record(stream)
    torch.cuda.synchronize()
    upd_us = 1e3 * ue[0].elapsed_time(ue[1]) / reps

    # the streaming kernels across probe counts and dtypes (theta 128 MiB, larger than L2):
    # the update's and the unpack/apply kernel's bandwidth against the measured HBM peak
    streaming = {}
    if world == 1:
        for dt, elems, esz in (("f32", 1 << 25, 4), ("bf16", 1 << 26, 2)):
            g = torch.Generator(device=dev)
            g.manual_seed(5)
            th_s = (torch.randn(elems, device=dev, generator=g)
                    .to(torch.float32 if dt == "f32" else torch.bfloat16))
            out_s = torch.empty_like(th_s)
            cs = zo.zo_create(th_s, seed=7, stream=stream.cuda_stream)
            ent = {"elements": elems, "update": {}}
            for nn in (1, 2, 4, 8, 16, 32, 64, 160):
                cz = torch.zeros(nn, dtype=torch.float32, device=dev)  # theta unchanged
                zo.zo_update(cs, cz, nn)
                ue2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                ue2[0].record(stream)
                for _ in range(5):
                    zo.zo_update(cs, cz, nn)
                ue2[1].record(stream)
                torch.cuda.synchronize()
                us = 1e3 * ue2[0].elapsed_time(ue2[1]) / 5
                gbs = 2 * esz * elems / (us * 1e-6) / 1e9
                ent["update"][str(nn)] = {"us": us, "GBps": gbs, "frac_hbm": gbs / hbm_peak}
            zo.zo_perturb(cs, +1, EPS, 3)
            zo.zo_perturb_range(cs, 0, elems, out_s)
            pe2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            pe2[0].record(stream)
            for _ in range(5):
                zo.zo_perturb_range(cs, 0, elems, out_s)
            pe2[1].record(stream)
            torch.cuda.synchronize()
            zo.zo_restore(cs)
            us = 1e3 * pe2[0].elapsed_time(pe2[1]) / 5
            gbs = 2 * esz * elems / (us * 1e-6) / 1e9
            ent["perturb"] = {"us": us, "GBps": gbs, "frac_hbm": gbs / hbm_peak}
            cs.close()
            streaming[dt] = ent
            del th_s, out_s

    # end to end through the public API with host buffers: D copied in, losses copied out
    D_host = torch.from_numpy(D_np[first:first + count]).pin_memory()
    L_host = torch.zeros(2 * n + 1, dtype=torch.float64).pin_memory()
    e2e_steps = max(3, min(args.steps, 30))

    def e2e_step():
        if world == 1:  # pipelined: step k+1's copy of D overlaps step k's kernels
            zo.zo_quad_step_host_async(ctx, D_host, n, EPS, LR, DAMPING, True, L_host)
            return
        D.copy_(D_host, non_blocking=True)  # this rank's slice of D
        tot = zdist.element_parallel_step(n, partial_losses, apply_step, dev)
        L_host.copy_(tot)  # synchronous device -> host read
    e2e_step()  # staging allocation
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    torch.cuda.synchronize()
    e2e_s = time.perf_counter() - t0
    if world > 1:
        t = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = float(t.item())
    e2e_value = e2e_steps / e2e_s

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            M_sample = 1 << 20
            times = time_oracle(M_sample, 2)
            per = sum(times) / len(times)
            cpu = {"value": (M_sample / M_FULL) / per, "unit": "steps/s", "cores": 1,
                   "kind": "oracle",
                   "sample": "2 oracle steps on the first 2^20 of 2^24 parameters; steps/s scaled by 1/16",
                   "host": host_cpu()}
            import oracle.timing
            ac, P = oracle_all_cores(M_sample, 0, 1)
            cpu["all_cores"] = {
                "value": ac, "unit": "steps/s", "cores": P,
                "sample": f"{P} concurrent single-threaded oracle processes, one step each on its "
                          "own 2^20-element sample; steps/s scaled by 1/16"}
            rates = oracle.timing.element_rates(1 << 22, 1 << 20, (16, 32, 64, 160))
            cpu["element_rates"] = {
                "unit": "elements/s", "cores": 1, "perturb": rates["perturb"],
                "update": rates["update"],
                "sample": "oracle perturbation of 2^22 elements (one probe); oracle fp32-order "
                          "update of 2^20 elements with n probes regenerated"}
        # the loss passes (clean loss fused into the first), precond, update; with N ranks the
        # same per rank on its slice (the loss exchange is NCCL's)
        launches_per_step = n_oct + 2
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M_FULL, "n_pert": n, "eps": EPS, "lr": LR,
                       "damping": DAMPING,
                       "parallelism": (f"element-parallel x{world}: theta and D sharded in "
                                       f"contiguous slices, partial losses all-gathered"
                                       if world > 1 else "1 GPU"),
                       "l2": "flushed between steps (256 MiB write, untimed); theta+D = 128 MiB"},
            "roofline": {"kernel": "quad_octet_kernel (the 128 losses L(theta +- eps z_i) of "
                                   "eight probe octets in one pass, perturbation on load, fp64 "
                                   "accumulation)",
                         "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                         "bytes_per_launch": loss_bytes, "avg_launch_us": loss_us,
                         "traffic": None},
            "kernels": {
                "quad_loss_kernel<pair>": {"avg_launch_us": pair_us, "losses_per_launch": 2,
                                           "bytes_per_launch": loss_bytes,
                                           "achieved_GBps": loss_bytes / (pair_us * 1e-6) / 1e9,
                                           "frac_hbm": loss_bytes / (pair_us * 1e-6) / 1e9 / hbm_peak},
                "update_kernel": {"avg_launch_us": upd_us, "bytes_per_launch": upd_bytes,
                                  "achieved_GBps": upd_bytes / (upd_us * 1e-6) / 1e9,
                                  "frac_hbm": upd_bytes / (upd_us * 1e-6) / 1e9 / hbm_peak},
            },
            "streaming": streaming,
            "phases_from": (f"{n_ph} further steps with phase events after the timed steps"
                            if n_ph else "not bracketed (N > 1)"),
            "phases_ms": {"clean_loss": statistics.mean(clean_ms),
                          "probe_losses": statistics.mean(probe_ms),
                          "precond_update": statistics.mean(upd_ms)},
            "tokens_per_s": None,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": 4 * M_FULL,
                    "d2h_bytes_per_step": 8 * (2 * n + 1) * world,
                    "path": "D pinned host -> device every step (each rank its slice), losses "
                            "back (zo_quad_step_host_async at one GPU: copies on the context's "
                            "copy stream overlap the previous step's kernels)"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        line["roofline"]["traffic"] = args.traffic if args.traffic is not None else loss_traffic()
        if loss_traffic() is not None:  # the recorded instruction count is valid: issue roofline
            mhz = (clocks or {}).get("sm_mhz") or 1965.0
            peak_inst = SM_COUNT * ISSUE_PER_SM_CLOCK * mhz * 1e6 / 1e9  # G warp-instr/s
            ach_inst = LOSS_WARP_INSTRUCTIONS / (loss_us * 1e-6) / 1e9
            hbm_view = {k: line["roofline"][k] for k in ("achieved", "peak", "unit", "frac")}
            line["roofline"].update({
                "bound": "alu", "achieved": ach_inst, "peak": peak_inst,
                "unit": "G warp-instructions/s", "frac": ach_inst / peak_inst,
                "peak_kind": f"issue limit: {SM_COUNT} SMs x {ISSUE_PER_SM_CLOCK} per clock at "
                             f"{mhz:.0f} MHz",
                "warp_instructions_per_launch": LOSS_WARP_INSTRUCTIONS, "hbm_view": hbm_view})
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ decoder workloads

def decoder_cfg(name):
    import synth
    return synth.QWEN_CONFIGS[name] if name.startswith("qwen") else synth.OPT_CONFIGS[name]


def init_decoder_params(theta, cfg, seed):
    """Synthetic initialisation on the device (too large for host numpy at 30B): matrices
    N(0, 0.02) in bf16, biases 0, norm gains 1 and shifts 0."""
    import torch

    import synth
    g = torch.Generator(device=theta.device)
    g.manual_seed(seed)
    o = 0
    segs = synth.qwen_segments if cfg.get("family") == "qwen3" else synth.opt_segments
    for kind, n in segs(cfg):
        seg = theta[o:o + n]
        if kind == "matrix":
            step = 1 << 28
            for a in range(0, n, step):
                seg[a:a + step].normal_(0.0, 0.02, generator=g)
        elif kind == "gain":
            seg.fill_(1.0)
        else:
            seg.zero_()
        o += n


def decoder_arm(args):
    import torch

    import synth
    import zero_order_forward_b200 as zo

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    name = args.workload
    cfg = decoder_cfg(name)
    qwen = cfg.get("family") == "qwen3"
    w = dict(DECODER_WORKLOADS[name])
    if args.n_pert:
        w["n_pert"] = args.n_pert
    B, S, k, n = w["batch"], w["seq"], w["n_micro"], w["n_pert"]
    M = zo.zo_model_param_count(cfg)
    theta = torch.empty(M, dtype=torch.bfloat16, device=dev)
    init_decoder_params(theta, cfg, seed=rank)
    stream = torch.cuda.current_stream(dev)
    ctx = zo.zo_create(theta, seed=rank, stream=stream.cuda_stream)
    model = zo.zo_model_create(ctx, cfg, B * S)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    tokens = torch.randint(0, cfg["vocab"], (k, B, S), dtype=torch.int32, device=dev, generator=gen)
    labels = torch.randint(0, 2, (k, B), dtype=torch.int32, device=dev, generator=gen)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device=dev)
    eps, lr, lam = 1e-3, 1e-6, 1e-3

    def step():
        zo.zo_model_step(model, tokens, labels, B, S, k, n, eps, lr, lam, True, losses)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    zo.zo_enable_phase_timing(ctx, args.steps)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    ev[0].record(stream)
    for i in range(args.steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    zo.zo_sync(ctx)
    phases = zo.zo_phase_times(ctx, args.steps)
    zo.zo_enable_phase_timing(ctx, 0)
    total_s = ev[0].elapsed_time(ev[-1]) / 1e3
    upd_ms = float(phases[:, 2].mean())  # preconditioner (one CTA, ~5 us) + update
    upd_bytes = 2 * 2 * M  # bf16 theta read + written once
    peak_mem = torch.cuda.max_memory_allocated(dev)
    free_b, tot_b = torch.cuda.mem_get_info(dev)

    # one clean forward, and each projection GEMM at this micro-batch's shape
    T, d, f = B * S, cfg["d_model"], cfg["d_ffn"]
    fe = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    fe[0].record(stream)
    zo.zo_model_loss(model, tokens[0], labels[0], B, S, 1.0 / B, losses[0:1])
    fe[1].record(stream)
    torch.cuda.synchronize()
    fwd_ms = fe[0].elapsed_time(fe[1])
    peak_b, peak_s, peak_kind = bf16_peaks()
    H = cfg["n_heads"]
    Hk, e = (cfg["n_kv_heads"], cfg["head_dim"]) if qwen else (H, d // H)
    nq, na = (H + 2 * Hk) * e, H * e
    if qwen:  # no biases; SwiGLU's gate and up projections are one GEMM of width 2f
        shapes = {"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "gate_up": (T, 2 * f, d, 0),
                  "down": (T, d, f, 2)}
    else:
        shapes = {"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "fc1": (T, f, d, 1),
                  "fc2": (T, d, f, 2)}
    gemm = {}
    A = torch.randn(T * max(K for _, _, K, _ in shapes.values()), dtype=torch.bfloat16, device=dev)
    Wt = torch.randn(max(N * K for _, N, K, _ in shapes.values()), dtype=torch.bfloat16,
                     device=dev) * 0.02
    max_n = max(N for _, N, _, _ in shapes.values())
    bias = None if qwen else torch.zeros(max_n, dtype=torch.bfloat16, device=dev)
    out_b = torch.empty(T * max_n, dtype=torch.bfloat16, device=dev)
    out_f = torch.zeros(T * d, dtype=torch.float32, device=dev)
    flops_layer = 0
    for key, (Mm, N, K, epi) in shapes.items():
        out = out_f if epi == 2 else out_b
        for _ in range(2):
            zo.zo_gemm_bf16(ctx, A, Wt, bias, out, Mm, N, K, N, epi)
        reps = 5
        ge = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ge[0].record(stream)
        for _ in range(reps):
            zo.zo_gemm_bf16(ctx, A, Wt, bias, out, Mm, N, K, N, epi)
        ge[1].record(stream)
        torch.cuda.synchronize()
        us = 1e3 * ge[0].elapsed_time(ge[1]) / reps
        fl = 2.0 * Mm * N * K
        flops_layer += fl
        gemm[key] = {"shape": [Mm, N, K], "avg_launch_us": us, "tflops": fl / us / 1e6,
                     "frac_burst": fl / us / 1e6 / peak_b}
    # causal attention at this micro-batch's shape (mma.sync path)
    qkv = torch.randn(T * nq, dtype=torch.bfloat16, device=dev)
    att = torch.empty(T * na, dtype=torch.bfloat16, device=dev)
    for _ in range(2):
        zo.zo_attention_gqa(ctx, qkv, att, B, S, H, Hk, e)
    ae = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ae[0].record(stream)
    for _ in range(5):
        zo.zo_attention_gqa(ctx, qkv, att, B, S, H, Hk, e)
    ae[1].record(stream)
    torch.cuda.synchronize()
    attn_us = 1e3 * ae[0].elapsed_time(ae[1]) / 5
    attn_flops = 2.0 * B * H * S * S * e  # causal half of 4 B H S^2 e
    zo.zo_sync(ctx)
    gemm_us = sum(g["avg_launch_us"] for g in gemm.values())
    gemm_tflops = flops_layer / gemm_us / 1e6
    fwds = (2 * n + 1) * k
    tokens_per_step = fwds * T
    value = args.steps / total_s
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        # the oracle's forward of one layer at the real width (vocabulary cut to 4096: it only
        # feeds the gather and the 2-row head), one thread; the step extrapolated from it
        red = dict(cfg, n_layers=1, vocab=4096)
        seq = 64
        tps = oracle_workers([("forward", "qwen3" if qwen else "opt", json.dumps(red), seq)])[0][
            "tokens_per_s"]
        cpu_step_s = fwds * B * S * cfg["n_layers"] / tps
        cpu = {"value": 1.0 / cpu_step_s, "unit": "steps/s", "cores": 1, "kind": "oracle",
               "extrapolated": True,
               "sample": f"oracle fp64 forward of 1 layer at the real width, 1 x {seq} tokens "
                         f"(vocabulary cut to 4096): {tps:.1f} tokens/s; the step extrapolated "
                         f"linearly in layers and tokens ({fwds} forwards of {B * S} tokens x "
                         f"{cfg['n_layers']} layers), attention's quadratic term at the full "
                         f"length not included"}
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{name}-shaped decoder, micro-batch {B}x{S}, {k} micro-batches, "
                               f"n_pert={n}, 1.5-SPSA", "layers": cfg["n_layers"], "d_model": d,
                   "params": M},
        "tokens_per_s": tokens_per_step * args.steps / total_s,
        "forward_ms": fwd_ms,
        "forwards_per_step": fwds,
        "roofline": {"kernel": "gemm_bf16_kernel (tcgen05, 4 projections of one layer)",
                     "bound": "tensor", "achieved": gemm_tflops, "peak": peak_b,
                     "unit": "TFLOP/s", "frac": gemm_tflops / peak_b, "peak_kind": peak_kind,
                     "flops_per_layer": flops_layer, "traffic": None},
        "gemm": gemm,
        "attention": {"avg_launch_us": attn_us, "tflops": attn_flops / attn_us / 1e6},
        "phases_ms": {"clean_loss": float(phases[:, 0].mean()),
                      "probe_losses": float(phases[:, 1].mean()), "precond_update": upd_ms},
        "kernels": {"update_kernel": {"n_pert": n, "bytes": upd_bytes,
                                      "achieved_GBps": upd_bytes / (upd_ms * 1e-3) / 1e9,
                                      "frac_hbm": upd_bytes / (upd_ms * 1e-3) / 1e9 / peaks()[0]}},
        "memory": {"peak_allocated_GB": peak_mem / 1e9, "device_used_GB": (tot_b - free_b) / 1e9},
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    model.close()
    ctx.close()
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ conditioning study

STUDY_M, STUDY_N, STUDY_STEPS = 1 << 20, 16, 400
# learning rates in units of 2 n / tr(H) (the SPSA step's stability scale: the estimator's
# noise grows with tr(H) / n), so the sweep means the same at any M
STUDY_LR_UNITS = (0.035, 0.05, 0.07, 0.1, 0.14, 0.2, 0.28, 0.4)


def lowrank_arm(args):
    """The low-rank-plus-diagonal quadratic (per-probe curvature differs, so 1.5-SPSA's
    weights do): steps/s of full 1.5-SPSA steps at M = 2^24, n = 64, and a learning-rate
    sweep of 1SPSA against 1.5-SPSA at M = 2^20, n = 16, 400 steps each."""
    import torch

    import synth
    import zero_order_forward_b200 as zo

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_peak, peak_kind = peaks()
    stream = torch.cuda.current_stream(dev)
    n = N_PERT
    th_np, D_np, lam, vseed = synth.lowrank_problem(M_FULL, seed=0)
    theta = torch.from_numpy(th_np).to(dev)
    D = torch.from_numpy(D_np).to(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device=dev)
    ctx = zo.zo_create(theta, seed=0, stream=stream.cuda_stream)
    lr_time = 1e-9  # timing run: any stable lr

    def step():
        zo.zo_lowrank_step(ctx, D, lam, vseed, n, EPS, lr_time, DAMPING, True, losses)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    zo.zo_enable_phase_timing(ctx, args.steps)
    sampler = ClockSampler(0)
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        step()
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    zo.zo_sync(ctx)
    ph = zo.zo_phase_times(ctx, args.steps)
    zo.zo_enable_phase_timing(ctx, 0)
    total_s = sum(e[0].elapsed_time(e[1]) for e in evs) / 1e3
    # the probe phase: per 64 probes one diagonal table pass (theta and D) and one pass per
    # direction for the dot products (theta only), then the combination
    rank = len(lam)
    passes = ((n + 63) // 64) * (1 + rank)
    loss_us = 1e3 * float(ph[:, 1].mean()) / passes
    pass_bytes = (8 + 4 * rank) * M_FULL / (1 + rank)  # mean algorithmic bytes per pass
    achieved = pass_bytes / (loss_us * 1e-6) / 1e9
    ctx.close()

    # the study: the same problem at M = 2^20, both methods, a learning-rate sweep
    sth, sD, slam, svseed = synth.lowrank_problem(STUDY_M, seed=1)
    trH = float(sD.astype(np.float64).sum()) + sum(slam)
    unit = 2 * STUDY_N / trH
    Dd = torch.from_numpy(sD).to(dev)
    sl = torch.zeros(2 * STUDY_N + 1, dtype=torch.float64, device=dev)
    out = torch.zeros(1, dtype=torch.float64, device=dev)
    rows = []
    for u in STUDY_LR_UNITS:
        lr = u * unit
        row = {"lr": lr, "lr_units": u}
        for name, pre in (("1spsa", False), ("1.5spsa", True)):
            th = torch.from_numpy(sth).to(dev)
            c = zo.zo_create(th, seed=2, stream=stream.cuda_stream)
            zo.zo_lowrank_loss(c, Dd, slam, svseed, out)
            L_init = float(out.item())
            skipped = 0
            for k in range(STUDY_STEPS):
                zo.zo_lowrank_step(c, Dd, slam, svseed, STUDY_N, EPS, lr, DAMPING, pre, sl)
                if k % 50 == 49:  # diverged runs stop early (their losses overflow)
                    zo.zo_lowrank_loss(c, Dd, slam, svseed, out)
                    if not np.isfinite(out.item()) or out.item() > 1e6 * L_init:
                        break
            skipped = zo.zo_sync(c, raise_nonfinite=False)
            zo.zo_lowrank_loss(c, Dd, slam, svseed, out)
            ratio = float(out.item()) / L_init
            ok = bool(np.isfinite(ratio)) and ratio < 1.0 and not skipped
            row[name] = ratio if ok else None  # None: diverged
            if pre and ok:  # the weights of the last step: their spread is the preconditioning
                w = zo.zo_get_precond(c, STUDY_N)[2]
                row["w_min_max"] = [float(w.min()), float(w.max())]
            c.close()
        rows.append(row)
    stable = {m: max([r["lr"] for r in rows if r[m] is not None], default=None)
              for m in ("1spsa", "1.5spsa")}
    line = {
        "metric": METRIC, "value": args.steps / total_s, "unit": "steps/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": "low-rank-plus-diagonal quadratic, M=2^24 fp32, rank 4, "
                               f"n_pert={n}, 1.5-SPSA", "M": M_FULL, "n_pert": n,
                   "l2": "flushed between steps (256 MiB write, untimed)"},
        "roofline": {"kernel": "quad_octet_kernel (diagonal and dot-product table passes, 64 "
                               "probes each; issue-bound like the diagonal quadratic's pass)",
                     "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "bytes_per_launch": pass_bytes, "avg_launch_us": loss_us, "traffic": None},
        "phases_ms": {"clean_loss": float(ph[:, 0].mean()), "probe_losses": float(ph[:, 1].mean()),
                      "precond_update": float(ph[:, 2].mean())},
        "study": {"M": STUDY_M, "n_pert": STUDY_N, "steps": STUDY_STEPS, "eps": EPS,
                  "lr_unit": unit, "trace_H": trH,
                  "damping": DAMPING, "alpha": 0.1, "eigenvalues_over_trD": list(synth.LOWRANK_SCALES),
                  "final_over_initial_loss": rows, "largest_stable_lr": stable},
        "gpu_launches": (passes + 3) * args.steps,  # passes, combination, precond, update
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ MLP workload

def mlp_arm(args):
    import torch

    import synth
    import zero_order_forward_b200 as zo

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    n, eps, lr, lam, B = 16, 1e-3, 1e-2, 1e-3, synth.MLP_BATCH
    theta = torch.from_numpy(synth.mlp_params(0)).to(dev)
    teacher = synth.mlp_params(0, tag="teacher")
    batches = [synth.mlp_batch(0, k, teacher) for k in range(args.warmup + args.steps)]
    Xs = [torch.from_numpy(x).to(dev) for x, _ in batches]
    ys = [torch.from_numpy(y).to(dev) for _, y in batches]
    stream = torch.cuda.current_stream(dev)
    ctx = zo.zo_create(theta, seed=0, stream=stream.cuda_stream)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device=dev)
    for k in range(args.warmup):
        zo.zo_mlp_step(ctx, Xs[k], ys[k], B, 64, 256, 10, n, eps, lr, lam, True, losses)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(stream)
    for k in range(args.warmup, args.warmup + args.steps):
        zo.zo_mlp_step(ctx, Xs[k], ys[k], B, 64, 256, 10, n, eps, lr, lam, True, losses)
    ev[1].record(stream)
    torch.cuda.synchronize()
    zo.zo_sync(ctx)
    total_s = ev[0].elapsed_time(ev[1]) / 1e3
    line = {"metric": METRIC, "value": args.steps / total_s, "unit": "steps/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": "MLP 64-256-10 fp32 (M=19,210), batch 64, teacher labels, "
                                   "n_pert=16, eps=1e-3, lr=1e-2, damping=1e-3, 1.5-SPSA"},
            "final_loss": float(losses[0].item()),
            # all 33 losses from one staged-parameter launch and its batch sums, then the
            # preconditioner and the update
            "gpu_launches": 4 * args.steps}
    if not args.no_cpu_baseline:
        ts = oracle_workers([("mlp", 4)])[0]["times"]
        line["cpu_baseline"] = {"value": 1.0 / statistics.mean(ts), "unit": "steps/s", "cores": 1,
                                "kind": "oracle",
                                "sample": "4 full oracle steps of this workload after one untimed "
                                          "step, one thread", "host": host_cpu()}
        # every host core running the same steps in its own single-threaded process
        P = max(1, min(host_cores(), 32))
        res = oracle_workers([("mlp", 4)] * P)
        wall = max(r["t_end"] for r in res) - min(r["t_start"] for r in res)
        line["cpu_baseline"]["all_cores"] = {
            "value": sum(len(r["times"]) for r in res) / wall, "unit": "steps/s", "cores": P,
            "sample": f"{P} concurrent single-threaded oracle processes, 4 timed steps each; "
                      "total steps / the union of their timed phases"}
    ctx.close()
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 300 for the quadratic workloads and the MLP, 3 "
                         "for the decoders)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the loss kernel, if measured")
    ap.add_argument("--workload", default="quadratic",
                    choices=["quadratic", "mlp", "lowrank"] + sorted(DECODER_WORKLOADS))
    ap.add_argument("--n-pert", type=int, default=None, help="override n_pert (decoder workloads)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 3 if args.workload in DECODER_WORKLOADS else 300
    if args.warmup < 3 and args.workload == "quadratic":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args)
    if args.workload == "mlp":
        return mlp_arm(args)
    if args.workload == "lowrank":
        return lowrank_arm(args)
    if args.workload != "quadratic":
        return decoder_arm(args)
    return gpu_arm(args)


if __name__ == "__main__":
    sys.exit(main())
