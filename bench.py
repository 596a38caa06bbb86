#!/usr/bin/env python
"""Benchmark of one 1.5-SPSA step on B200: by default the OPT-30B-shaped decoder.

Default workload (one GPU): OPT-30B-shaped decoder (48 layers, d 7168, 56 heads, FFN 28672,
vocabulary 50272, learned positions, pre-LN; 29.97 B bf16 parameters N(0, 0.02), trained in
place), batch 8 x 2048 uniform tokens, 2-class last-token cross-entropy with Bernoulli(0.5)
labels; n_pert = 16, eps = 1e-3, lr = 1e-6, damping = 1e-3.  One step = the clean forward +
2 n_pert perturbed forwards (each layer's perturbed weights materialised into one layer
window) + the preconditioner + the update of all 29.97 B parameters, through zo_model_step of
libzo.so.  The same run measures the diagonal-quadratic workload (M = 2^24 fp32, n_pert = 64)
as a sub-record.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload opt-30b|opt-1.3b|opt-125m|qwen3-1.7b|qwen3-8b|quadratic|mlp|lowrank]

Prints ONE JSON line (rank 0).  With N > 1 (torchrun, one rank per GPU) the decoder runs
probe-parallel: every rank holds a full replica of theta (same seed), evaluates its share of
the probes and of the clean batch, the losses are all-gathered over NCCL, and every rank
applies the same update, so the replicas stay bit-identical ("scaling": "strong"; the step
time is the max over ranks).  `--impl reference` times the CPU oracle on bounded samples of
the same workload.
"""
import argparse
import hashlib
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
DEFAULT_WORKLOAD = "opt-30b"
M_FULL = 1 << 24
N_PERT, EPS, LR, DAMPING = 64, 1e-3, 4e-7, 1e-3
WORKLOAD = ("diagonal quadratic L=1/2*sum D_j theta_j^2, M=2^24 fp32, D log-uniform [1e-3,1e3], "
            "theta0~N(0,1); 1.5-SPSA n_pert=64 eps=1e-3 lr=4e-7 damping=1e-3")
FALLBACK_HBM_GBS = 6650.0
SM_COUNT, ISSUE_PER_SM_CLOCK = 148, 4

# Counters of single ncu captures, reported beside the live timings.  Each record holds the
# SHA-256 of the kernel's sources at the time of the capture and is reported (as taken from
# that capture, not from this run) only while the sources still hash to it; otherwise null.
#   quad_octet_kernel, M = 2^24: DRAM bytes (read + write) and warp instructions per launch.
LOSS_TRAFFIC = {"sources": ("zo_loss.cu", "zo_internal.cuh"),
                "sources_sha256": "347def2504d19bf9fb19393e6166cf4226ca58880a5027e41e6f1770ef8b1a8b",
                "bytes": 138.50e6, "warp_instructions": 89.22e6}
#   update_kernel on 2^28 elements (the streaming sweep), per dtype and probe count: warp
#   instructions per launch (`bench.py --streaming-only` under ncu).
UPDATE_INSTR = {"sources": ("zo_step.cu", "zo_internal.cuh"),
                "sources_sha256": "e9bb413b69819c1a09adbe59f72eca7616d2ec92b53c210f213d25589e5224b2",
                "warp_instructions": {
                    "f32": {"1": 127.80e6, "2": 127.87e6, "4": 127.87e6, "8": 127.91e6,
                            "16": 184.14e6, "32": 297.79e6, "64": 523.93e6, "160": 1196.59e6},
                    "bf16": {"1": 150.25e6, "2": 150.34e6, "4": 150.40e6, "8": 150.48e6,
                             "16": 207.25e6, "32": 323.66e6, "64": 551.14e6, "160": 1238.20e6}}}
#   gemm_pair_kernel at the OPT-30B layer shapes (T = 16384): DRAM bytes (read + write) per
#   launch averaged over the four projections of one layer (the step's other GEMM launches,
#   the pruned last layer's few rows, move a negligible share of its bytes).  Captured with
#   contiguous A operands; inside the step the FC2 GEMM reads its A (the FFN intermediate)
#   with a padded row stride, which measured about 8 GB less per FC2 launch at this shape.
GEMM_TRAFFIC = {"sources": ("zo_gemm.cu", "zo_tc.cuh"),
                "sources_sha256": "39166dc3dd0be582ecf2af1142e38a68cc4c27363793ed105cafc578f837207f",
                "bytes": 11.69e9}


def sources_sha256(names):
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "zero_order_forward_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured(record, key):
    """record[key] if the kernel's sources are unchanged since the capture, else None."""
    try:
        ok = record["sources_sha256"] is not None and sources_sha256(record["sources"]) == record["sources_sha256"]
    except OSError:
        ok = False
    return record[key] if ok else None


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
    oracle_all_cores.last_wall_s = wall
    return P * steps * (M_sample / M_FULL) / wall, P


def quad_config(world):
    """The `config` object of the quadratic line (the same for the GPU and the reference arm)."""
    return {"workload": WORKLOAD, "M": M_FULL, "n_pert": N_PERT, "eps": EPS, "lr": LR,
            "damping": DAMPING,
            "parallelism": (f"element-parallel x{world}: theta and D sharded in contiguous slices, "
                            f"partial losses all-gathered" if world > 1 else "1 GPU"),
            "l2": "flushed between steps (256 MiB write, untimed); theta+D = 128 MiB"}


def decoder_reference_arm(args):
    """The oracle as it stands on the machine's host cores (numpy's BLAS threads), on the decoder
    workload's config: each of the W + K steps is a bounded sample, the oracle's fp64 forward of
    one layer at the real width on one 64-token sequence (vocabulary cut to 4096, which only
    feeds the embedding gather and the 2-row head); the full step's time is extrapolated
    linearly in layers and tokens and labelled as such."""
    import oracle
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    name = args.workload
    cfg = decoder_cfg(name)
    w = decoder_workload(name, args.n_pert)
    B, S, k, n = w["batch"], w["seq"], w["n_micro"], w["n_pert"]
    qwen = cfg.get("family") == "qwen3"
    M = (oracle.qwen if qwen else oracle.opt).param_count(cfg)
    red = dict(cfg, n_layers=1, vocab=4096)
    seq = 64
    P = host_cores()
    res = oracle_workers([("forward_samples", "qwen3" if qwen else "opt", json.dumps(red), seq,
                           args.warmup, args.steps)], threads=P)[0]
    sample_s = statistics.mean(res["times"])
    fwds = (2 * n + 1) * k
    step_s = fwds * B * S * cfg["n_layers"] * sample_s / seq  # extrapolated full step
    value = 1.0 / step_s
    sample = (f"each step: the oracle's fp64 forward of 1 layer at the real width on 1 x {seq} "
              f"tokens (vocabulary cut to 4096), {P} BLAS threads, {sample_s:.3f} s per sample; "
              f"the full step ({fwds} forwards of {B * S} tokens x {cfg['n_layers']} layers) "
              f"extrapolated linearly in layers and tokens (attention's quadratic term at the full "
              f"length not included)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * step_s, "extrapolated": True,
            "timed_region_s": sum(res["times"]), "sample_ms_per_step": 1e3 * sample_s,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decoder_config(name, w, M, world),
            "tokens_per_s": fwds * B * S / step_s,
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": P, "kind": "oracle",
                             "extrapolated": True, "sample": sample, "host": host_cpu()},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def reference_arm(args):
    if args.workload in DECODER_WORKLOADS:
        return decoder_reference_arm(args)
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
            "ms_per_step": 1e3 / value, "extrapolated": True,
            "timed_region_s": oracle_all_cores.last_wall_s,
            "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": quad_config(world),
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


# ------------------------------------------------------------------ streaming kernels

def streaming_sweep(zo, torch, dev, stream, flush, hbm_peak):
    """The update (n = 1 .. 160) and the window perturbation on 2^28-element vectors (1 GiB
    fp32, 512 MiB bf16: far larger than L2, and L2 flushed before every timed launch), fp32
    then bf16; per launch class 1 untimed + 5 timed launches.  Each update entry carries two
    rooflines: the HBM fraction of its algorithmic bytes, and its instruction-issue fraction,
    the recorded ncu warp-instruction count of that (dtype, n) (UPDATE_INSTR, while the
    sources are unchanged) per second against 148 SMs x 4 per clock at the median SM clock
    sampled over the sweep; `bound` names the larger."""
    elems = 1 << 28
    reps = 5

    def timed_reps(fn):
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            fn()
            ev[1].record(stream)
            torch.cuda.synchronize()
            tot += ev[0].elapsed_time(ev[1])
        return 1e3 * tot / reps

    instr = captured(UPDATE_INSTR, "warp_instructions")
    out = {}
    cs_clock = ClockSampler(torch.cuda.current_device())
    for dt, esz in (("f32", 4), ("bf16", 2)):
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        th_s = torch.empty(elems, dtype=torch.float32 if dt == "f32" else torch.bfloat16, device=dev)
        th_s.normal_(generator=g)
        out_s = torch.empty_like(th_s)
        cs = zo.zo_create(th_s, seed=7, stream=stream.cuda_stream)
        ent = {"elements": elems, "l2": "flushed before every timed launch", "update": {}}
        for nn in (1, 2, 4, 8, 16, 32, 64, 160):
            cz = torch.zeros(nn, dtype=torch.float32, device=dev)  # theta unchanged
            zo.zo_update(cs, cz, nn)
            us = timed_reps(lambda: zo.zo_update(cs, cz, nn))
            gbs = 2 * esz * elems / (us * 1e-6) / 1e9
            ent["update"][str(nn)] = {"us": us, "GBps": gbs, "frac_hbm": gbs / hbm_peak}
        zo.zo_perturb(cs, +1, EPS, 3)
        zo.zo_perturb_range(cs, 0, elems, out_s)
        us = timed_reps(lambda: zo.zo_perturb_range(cs, 0, elems, out_s))
        zo.zo_restore(cs)
        gbs = 2 * esz * elems / (us * 1e-6) / 1e9
        ent["perturb"] = {"us": us, "GBps": gbs, "frac_hbm": gbs / hbm_peak}
        cs.close()
        out[dt] = ent
        del th_s, out_s
    clk = cs_clock.stop()
    mhz = clk["sm_mhz"] if clk else None
    for dt, ent in out.items():
        for nn, e in ent["update"].items():
            wi = instr.get(dt, {}).get(nn) if instr else None
            if wi is None or not mhz:
                e["frac_issue"], e["bound"] = None, None
                continue
            e["warp_instructions"] = wi
            e["frac_issue"] = wi / (e["us"] * 1e-6) / (SM_COUNT * ISSUE_PER_SM_CLOCK * mhz * 1e6)
            e["bound"] = "issue" if e["frac_issue"] > e["frac_hbm"] else "hbm"
    out["sm_mhz"] = mhz
    out["instructions_from"] = ("ncu capture of these launches (smsp__inst_executed.sum), "
                                "not this run" if instr else None)
    torch.cuda.empty_cache()
    return out


def streaming_arm(args):
    """Only the streaming sweep (the command its instruction-count capture profiles)."""
    import torch

    import zero_order_forward_b200 as zo
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    hbm_peak, kind = peaks()
    print(json.dumps({"streaming_only": True, "peak_kind": kind,
                      "streaming": streaming_sweep(zo, torch, dev, stream, flush, hbm_peak)}),
          flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def gpu_arm(args, sub=False):
    """The diagonal-quadratic workload; returns rank 0's JSON line (None elsewhere).  sub=True
    (the sub-record of the decoder line) leaves out the CPU baseline."""
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

    def timed_reps(fn, reps):
        """Mean CUDA-event duration (us) of fn() over reps launches, L2 flushed before each
        (the flush is outside the timed events)."""
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            fn()
            ev[1].record(stream)
            torch.cuda.synchronize()
            tot += ev[0].elapsed_time(ev[1])
        return 1e3 * tot / reps

    # single-kernel timing of the update (same stream), for its own roofline
    coef = torch.from_numpy(synth.coefficients(n, seed=1) * 0).to(dev)  # zero: theta unchanged
    upd_us = timed_reps(lambda: zo.zo_update(ctx, coef, n), 10)

    streaming = streaming_sweep(zo, torch, dev, stream, flush, hbm_peak) if world == 1 else {}

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
        if world == 1 and not args.no_cpu_baseline and not sub:
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
            "config": quad_config(world),
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
        # The pass reads theta and D once (8 B per element): its roofline is HBM, against the
        # algorithmic bytes.  It is bound by instruction issue in practice, so the issue-rate
        # view is kept beside it, from the instruction count of the recorded capture.
        line["roofline"]["traffic"] = (args.traffic if args.traffic is not None
                                       else captured(LOSS_TRAFFIC, "bytes"))
        line["roofline"]["traffic_from"] = ("--traffic" if args.traffic is not None else
                                            "ncu capture of this kernel's current sources (not this run)"
                                            if line["roofline"]["traffic"] is not None else None)
        inst = captured(LOSS_TRAFFIC, "warp_instructions")
        if inst is not None:
            mhz = (clocks or {}).get("sm_mhz") or 1965.0
            peak_inst = SM_COUNT * ISSUE_PER_SM_CLOCK * mhz * 1e6 / 1e9  # G warp-instr/s
            ach_inst = inst / (loss_us * 1e-6) / 1e9
            line["roofline"]["issue_view"] = {
                "achieved": ach_inst, "peak": peak_inst, "unit": "G warp-instructions/s",
                "frac": ach_inst / peak_inst,
                "peak_kind": f"issue limit: {SM_COUNT} SMs x {ISSUE_PER_SM_CLOCK} per clock at "
                             f"{mhz:.0f} MHz (the sampled median)",
                "warp_instructions_per_launch": inst,
                "instructions_from": "ncu capture of this kernel's current sources (not this run)"}
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    del theta, D, flush
    torch.cuda.empty_cache()
    return line


# ------------------------------------------------------------------ decoder workloads

DEC_EPS, DEC_LR, DEC_DAMPING = 1e-3, 1e-6, 1e-3
MEMORY_TARGET_GB = 80.0


def decoder_cfg(name):
    import synth
    return synth.QWEN_CONFIGS[name] if name.startswith("qwen") else synth.OPT_CONFIGS[name]


def decoder_workload(name, n_pert=None):
    w = dict(DECODER_WORKLOADS[name])
    if n_pert:
        w["n_pert"] = n_pert
    return w


def decoder_config(name, w, M, world):
    """The `config` object of a decoder line (the same for the GPU and the reference arm)."""
    cfg = decoder_cfg(name)
    B, S, k, n = w["batch"], w["seq"], w["n_micro"], w["n_pert"]
    fam = "Qwen3" if cfg.get("family") == "qwen3" else "OPT"
    heads = (f"{cfg['n_heads']} query / {cfg['n_kv_heads']} key-value heads of {cfg['head_dim']}"
             if fam == "Qwen3" else f"{cfg['n_heads']} heads")
    return {
        "workload": (f"{name}-shaped {fam} decoder ({cfg['n_layers']} layers, d={cfg['d_model']}, "
                     f"{heads}, FFN {cfg['d_ffn']}, vocab {cfg['vocab']}; {M} bf16 params "
                     f"N(0,0.02)), micro-batch {B}x{S} uniform tokens x {k}, 2-class last-token "
                     f"CE; 1.5-SPSA n_pert={n}, eps={DEC_EPS:g}, lr={DEC_LR:g}, "
                     f"damping={DEC_DAMPING:g}, trained in place"),
        "params": M, "batch": B, "seq": S, "n_micro": k, "n_pert": n, "eps": DEC_EPS,
        "lr": DEC_LR, "damping": DEC_DAMPING,
        "parallelism": (f"probe-parallel x{world}: full theta replica per GPU, probes and the clean "
                        f"batch split across ranks, losses all-gathered (NCCL)" if world > 1
                        else "1 GPU"),
        "l2": "inputs larger than L2: every forward streams all the weights (and the perturbed "
              "layer windows) from HBM",
    }


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


def add_kernel_times(tot, kt):
    for c, v in kt.items():
        for key in ("ms", "launches", "work"):
            tot[c][key] += v[key]


def kernel_summary(tot, hbm_peak, bf16_burst, bf16_sustained):
    """Per kernel class of the timed region: launches, mean launch duration, achieved rate
    from the algorithmic work, and its fraction of the measured peak."""
    out = {}
    for c, v in tot.items():
        if not v["launches"]:
            continue
        sec = v["ms"] * 1e-3
        e = {"launches": v["launches"], "total_ms": v["ms"], "avg_launch_us": 1e3 * v["ms"] / v["launches"],
             "share_of_kernel_time": None}
        if c in ("gemm", "attention"):
            tf = v["work"] / sec / 1e12
            e.update({"flops_per_launch": v["work"] / v["launches"], "tflops": tf,
                      "frac_bf16_sustained": tf / bf16_sustained, "frac_bf16_burst": tf / bf16_burst})
        else:
            gb = v["work"] / sec / 1e9
            e.update({"bytes_per_launch": v["work"] / v["launches"], "GBps": gb,
                      "frac_hbm": gb / hbm_peak})
        out[c] = e
    total = sum(v["ms"] for v in tot.values())
    for c in out:
        out[c]["share_of_kernel_time"] = tot[c]["ms"] / total if total else None
    return out


def decoder_arm(args):
    """Whole 1.5-SPSA steps of a decoder workload through zo_model_step (one GPU) or the
    probe-parallel driver (N ranks); prints rank 0's JSON line."""
    import datetime

    import torch
    import torch.distributed as dist

    import zero_order_forward_b200 as zo
    from zero_order_forward_b200 import dist as zdist

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    name = args.workload
    cfg = decoder_cfg(name)
    qwen = cfg.get("family") == "qwen3"
    w = decoder_workload(name, args.n_pert)
    B, S, k, n = w["batch"], w["seq"], w["n_micro"], w["n_pert"]
    hbm_peak, hbm_kind = peaks()
    peak_b, peak_s, bf16_kind = bf16_peaks()

    # the diagonal-quadratic workload, measured first in the same run (its memory is freed
    # before the decoder's weights are allocated)
    quad = None
    if world == 1 and name == DEFAULT_WORKLOAD and not args.no_quadratic:
        quad = gpu_arm(args, sub=True)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=900),
                                device_id=dev)

    M = zo.zo_model_param_count(cfg)
    theta = torch.empty(M, dtype=torch.bfloat16, device=dev)
    init_decoder_params(theta, cfg, seed=0)  # the same weights on every rank: replicas
    stream = torch.cuda.current_stream(dev)
    ctx = zo.zo_create(theta, seed=0, stream=stream.cuda_stream)
    model = zo.zo_model_create(ctx, cfg, B * S)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000)
    tokens = torch.randint(0, cfg["vocab"], (k, B, S), dtype=torch.int32, device=dev, generator=gen)
    labels = torch.randint(0, 2, (k, B), dtype=torch.int32, device=dev, generator=gen)
    losses = torch.zeros(2 * n + 1, dtype=torch.float64, device=dev)
    eps, lr, lam = DEC_EPS, DEC_LR, DEC_DAMPING
    scale = 1.0 / (k * B)

    if world == 1:
        def step():
            zo.zo_model_step(model, tokens, labels, B, S, k, n, eps, lr, lam, True, losses)
    else:
        b0, nb = zdist.batch_share(B, rank, world)

        def loss_at(sign, probe, out):
            zo.zo_perturb(ctx, sign, eps, probe)
            for j in range(k):
                zo.zo_model_loss(model, tokens[j], labels[j], B, S, scale, out, j > 0)
            zo.zo_restore(ctx)

        def clean(out):  # this rank's share of the clean batch
            if nb == 0:
                out.zero_()
            for j in range(k if nb else 0):
                zo.zo_model_loss(model, tokens[j, b0:b0 + nb], labels[j, b0:b0 + nb], nb, S,
                                 scale, out, j > 0)

        def apply_step(Lp, Lm, L0):
            zo.zo_step(ctx, Lp, Lm, n, L0, lr, eps, lam)

        def step():
            L0, Lp, Lm = zdist.probe_parallel_step(n, loss_at, clean, apply_step, dev,
                                                   clean_shared=True)
            losses[0:1].copy_(L0)
            losses[1:1 + n].copy_(Lp)
            losses[1 + n:].copy_(Lm)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    zo.zo_sync(ctx)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    # timed region: K steps; every launch of the GEMM, attention, window-perturbation and
    # update kernels is bracketed by CUDA events on the context's stream (drained after each
    # step, which synchronises between steps)
    tot = {c: {"ms": 0.0, "launches": 0, "work": 0.0} for c in zo.KERNEL_CLASSES}
    dropped = 0
    zo.zo_enable_kernel_timing(ctx, True)
    zo.zo_kernel_times(ctx)
    if world == 1:
        zo.zo_enable_phase_timing(ctx, args.steps)
    launches0 = zo.zo_launch_count(ctx)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    ev[0].record(stream)
    for i in range(args.steps):
        step()
        ev[i + 1].record(stream)
        kt, dr = zo.zo_kernel_times(ctx)
        add_kernel_times(tot, kt)
        dropped += dr
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    launches = zo.zo_launch_count(ctx) - launches0
    zo.zo_enable_kernel_timing(ctx, False)
    zo.zo_sync(ctx)
    step_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
    total_s = ev[0].elapsed_time(ev[-1]) / 1e3
    phases = None
    if world == 1:
        ph = zo.zo_phase_times(ctx, args.steps)
        zo.zo_enable_phase_timing(ctx, 0)
        phases = {"clean_loss": float(ph[:, 0].mean()), "probe_losses": float(ph[:, 1].mean()),
                  "precond_update": float(ph[:, 2].mean())}
    if world > 1:
        t = torch.tensor([total_s, float(launches)], dtype=torch.float64, device=dev)
        mx = t.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        sm = t.clone()
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
        total_s, launches = float(mx[0].item()), int(sm[1].item())
    free_b, tot_b = torch.cuda.mem_get_info(dev)
    used_gb = (tot_b - free_b) / 1e9
    peak_alloc_gb = torch.cuda.max_memory_allocated(dev) / 1e9
    value = args.steps / total_s
    fwds = (2 * n + 1) * k
    T = B * S
    kernels = kernel_summary(tot, hbm_peak, peak_b, peak_s)

    # each projection GEMM and attention alone at this micro-batch's shape (one GPU)
    gemm_shapes, attn_alone = {}, None
    if world == 1:
        d, f = cfg["d_model"], cfg["d_ffn"]
        H = cfg["n_heads"]
        Hk, e = (cfg["n_kv_heads"], cfg["head_dim"]) if qwen else (H, d // H)
        nq, na = (H + 2 * Hk) * e, H * e
        if qwen:  # no biases; SwiGLU's gate and up projections are one GEMM of width 2f
            shapes = {"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "gate_up": (T, f, d, 3),
                      "down": (T, d, f, 2)}
        else:
            shapes = {"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "fc1": (T, f, d, 1),
                      "fc2": (T, d, f, 2)}
        A = torch.randn(T * max(K for _, _, K, _ in shapes.values()), dtype=torch.bfloat16, device=dev)
        Wt = torch.randn(max((2 if epi == 3 else 1) * N * K for _, N, K, epi in shapes.values()),
                         dtype=torch.bfloat16, device=dev) * 0.02
        max_n = max(N for _, N, _, _ in shapes.values())
        bias = None if qwen else torch.zeros(max_n, dtype=torch.bfloat16, device=dev)
        out_b = torch.empty(T * max_n, dtype=torch.bfloat16, device=dev)
        out_f = torch.zeros(T * d, dtype=torch.float32, device=dev)
        for key, (Mm, N, K, epi) in shapes.items():
            out = out_f if epi == 2 else out_b
            bb = None if epi == 3 else bias
            for _ in range(2):
                zo.zo_gemm_bf16(ctx, A, Wt, bb, out, Mm, N, K, N, epi)
            ge = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            clk = ClockSampler(local_rank)
            ge[0].record(stream)
            for _ in range(5):
                zo.zo_gemm_bf16(ctx, A, Wt, bb, out, Mm, N, K, N, epi)
            ge[1].record(stream)
            torch.cuda.synchronize()
            clk = clk.stop()
            us = 1e3 * ge[0].elapsed_time(ge[1]) / 5
            fl = 2.0 * Mm * N * K * (2 if epi == 3 else 1)
            gemm_shapes[key] = {"shape": [Mm, N, K], "avg_launch_us": us, "tflops": fl / us / 1e6,
                                "frac_bf16_burst": fl / us / 1e6 / peak_b,
                                "sm_mhz": clk["sm_mhz"] if clk else None}
        del A, Wt, out_b, out_f
        qkv = torch.randn(T * nq, dtype=torch.bfloat16, device=dev)
        att = torch.empty(T * na, dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            zo.zo_attention_gqa(ctx, qkv, att, B, S, H, Hk, e)
        ae = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        clk = ClockSampler(local_rank)
        ae[0].record(stream)
        for _ in range(5):
            zo.zo_attention_gqa(ctx, qkv, att, B, S, H, Hk, e)
        ae[1].record(stream)
        torch.cuda.synchronize()
        clk = clk.stop()
        attn_us = 1e3 * ae[0].elapsed_time(ae[1]) / 5
        attn_flops = 4.0 * e * B * H * S * (S + 1) / 2
        attn_alone = {"avg_launch_us": attn_us, "tflops": attn_flops / attn_us / 1e6,
                      "frac_bf16_burst": attn_flops / attn_us / 1e6 / peak_b,
                      "sm_mhz": clk["sm_mhz"] if clk else None,
                      "note": "timed after the steps, at the clock the power cap leaves; "
                              "`bench.py --kernels-only` times it on a cool GPU"}
        del qkv, att
        zo.zo_sync(ctx)

    # end to end through the C ABI with host buffers: every step copies its tokens and labels
    # from pinned host memory to the device and reads the 2n + 1 losses back to the host
    e2e_steps = max(1, min(args.steps, 2))
    tok_host = tokens.cpu().pin_memory()
    lab_host = labels.cpu().pin_memory()
    L_host = torch.zeros(2 * n + 1, dtype=torch.float64).pin_memory()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        if world == 1:
            zo.zo_model_step_host(model, tok_host, lab_host, B, S, k, n, eps, lr, lam, True, L_host)
        else:
            tokens.copy_(tok_host, non_blocking=True)
            labels.copy_(lab_host, non_blocking=True)
            step()
            L_host.copy_(losses)  # synchronous device -> host read
    torch.cuda.synchronize()
    e2e_s = time.perf_counter() - t0
    if world > 1:
        t = torch.tensor([e2e_s], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_s = float(t.item())
    zo.zo_sync(ctx)
    e2e = {"value": e2e_steps / e2e_s, "unit": "steps/s",
           "h2d_bytes_per_step": 4 * (k * B * S + k * B) * world,
           "d2h_bytes_per_step": 8 * (2 * n + 1) * world,
           "steps": e2e_steps, "tokens_per_s": e2e_steps * fwds * T / e2e_s,
           "path": ("zo_model_step_host: tokens and labels from pinned host memory, the 2n+1 "
                    "losses copied back, synchronised every step" if world == 1 else
                    "each rank copies the step's tokens and labels from pinned host memory, "
                    "runs the probe-parallel step and reads the losses back")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decoder_cpu_baseline(name, cfg, w, fwds)

    line = None
    if rank == 0:
        g = kernels.get("gemm", {})
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "gpu_launches": launches,
            "config": decoder_config(name, w, M, world),
            "tokens_per_s": fwds * T * args.steps / total_s,
            "tokens_per_step": fwds * T,
            "forwards_per_step": fwds,
            "step_ms": step_ms,
            "roofline": {
                "kernel": "gemm_pair_kernel (tcgen05 on CTA pairs, TMEM accumulators, TMA-fed: "
                          "the QKV, output and feed-forward projections of every forward)",
                "bound": "tensor", "achieved": g.get("tflops"), "peak": peak_s,
                "unit": "TFLOP/s", "frac": (g.get("tflops") or 0.0) / peak_s,
                "peak_kind": f"{bf16_kind} sustained bf16 GEMM (the kernel runs inside a "
                             f"seconds-long step under the power cap)",
                "frac_of_burst": (g.get("tflops") or 0.0) / peak_b,
                "flops_per_launch": g.get("flops_per_launch"),
                "avg_launch_us": g.get("avg_launch_us"),
                "timed": "CUDA events around every GEMM launch of the timed steps, on the "
                         "context's stream",
                "traffic": captured(GEMM_TRAFFIC, "bytes"),
                "traffic_from": ("ncu capture of this kernel's current sources at the four "
                                 "layer shapes (not this run)"
                                 if captured(GEMM_TRAFFIC, "bytes") is not None else None)},
            "kernels": kernels,
            "kernel_timing_dropped": dropped,
            "gemm_shapes_alone": gemm_shapes,
            "attention_alone": attn_alone,
            "phases_ms": phases,
            "memory": {"device_used_GB": used_gb, "torch_peak_allocated_GB": peak_alloc_gb,
                       "theta_GB": 2 * M / 1e9, "target_GB": MEMORY_TARGET_GB,
                       "within_target": used_gb < MEMORY_TARGET_GB,
                       "measured": "cudaMemGetInfo after the timed steps (every buffer of the "
                                   "step is allocated once and kept; nothing grows per probe)"},
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "peaks": {"hbm_GBps": hbm_peak, "hbm_kind": hbm_kind, "bf16_burst_tflops": peak_b,
                      "bf16_sustained_tflops": peak_s, "bf16_kind": bf16_kind},
        }
        if quad is not None:
            line["quadratic"] = quad
        if used_gb >= MEMORY_TARGET_GB:
            print(f"warning: device memory {used_gb:.1f} GB is above the {MEMORY_TARGET_GB} GB "
                  f"target", file=sys.stderr)
    model.close()
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def kernels_arm(args):
    """Each hot kernel of a decoder workload alone, at the workload's shapes and without the
    model's weights (for profiling and quick measurement): the four projection GEMMs and the
    causal attention of one micro-batch, the perturbation of one layer window, and the update
    of a 2^30-element bf16 slice at the workload's n_pert; for the OPT shapes also each
    projection with the perturbation fused into its operand path against the window path.  L2 is flushed before every timed
    launch.  Prints one JSON line of per-kernel timings (not the benchmark's contract line)."""
    import torch

    import zero_order_forward_b200 as zo

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    name = args.workload
    cfg = decoder_cfg(name)
    qwen = cfg.get("family") == "qwen3"
    w = decoder_workload(name, args.n_pert)
    B, S, n = w["batch"], w["seq"], w["n_pert"]
    T, d, f, H = B * S, cfg["d_model"], cfg["d_ffn"], cfg["n_heads"]
    Hk, e = (cfg["n_kv_heads"], cfg["head_dim"]) if qwen else (H, d // H)
    nq, na = (H + 2 * Hk) * e, H * e
    hbm_peak, _ = peaks()
    peak_b, peak_s, _ = bf16_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    reps = args.steps

    def timed(fn):
        """Average launch time (us) with L2 flushed before each launch, and the median SM
        clock sampled over the timed launches."""
        tot = 0.0
        fn()
        torch.cuda.synchronize()
        cs = ClockSampler(0)
        for _ in range(reps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            fn()
            ev[1].record(stream)
            torch.cuda.synchronize()
            tot += ev[0].elapsed_time(ev[1])
        clk = cs.stop()
        clocks[0] = clk["sm_mhz"] if clk else None
        return 1e3 * tot / reps

    clocks = [None]
    out = {}
    # the streaming kernels first, before the GEMMs heat the GPU up to its power cap
    import synth
    segs = (synth.qwen_segments if qwen else synth.opt_segments)(dict(cfg, n_layers=1))
    lead = 1 if qwen else 2
    layer = sum(c for _, c in segs[lead:-(1 if qwen else 2)])
    th = torch.empty(layer, dtype=torch.bfloat16, device=dev).normal_(0, 0.02)
    win = torch.empty_like(th)
    c2 = zo.zo_create(th, seed=0, stream=stream.cuda_stream)
    zo.zo_perturb(c2, +1, 1e-3, 3)
    us = timed(lambda: zo.zo_perturb_range(c2, 0, layer, win))
    zo.zo_restore(c2)
    gb = 4.0 * layer / (us * 1e-6) / 1e9
    out["perturb_window"] = {"elements": layer, "us": us, "GBps": gb, "frac_hbm": gb / hbm_peak,
                             "sm_mhz": clocks[0]}
    c2.close()
    del th, win
    # the update at this n_pert on a 2^30-element bf16 slice
    Mu = 1 << 30
    th = torch.empty(Mu, dtype=torch.bfloat16, device=dev).normal_(0, 0.02)
    c3 = zo.zo_create(th, seed=0, stream=stream.cuda_stream)
    coef = torch.zeros(n, dtype=torch.float32, device=dev)
    us = timed(lambda: zo.zo_update(c3, coef, n))
    gb = 4.0 * Mu / (us * 1e-6) / 1e9
    out["update"] = {"elements": Mu, "n_pert": n, "us": us, "GBps": gb, "frac_hbm": gb / hbm_peak,
                     "sm_mhz": clocks[0]}
    zo.zo_sync(c3)
    c3.close()
    del th, coef

    small = torch.zeros(1024, dtype=torch.bfloat16, device=dev)
    ctx = zo.zo_create(small, seed=0, stream=stream.cuda_stream)
    shapes = ({"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "gate_up": (T, f, d, 3), "down": (T, d, f, 2)}
              if qwen else
              {"qkv": (T, nq, d, 0), "out": (T, d, na, 2), "fc1": (T, f, d, 1), "fc2": (T, d, f, 2)})
    A = torch.randn(T * max(K for _, _, K, _ in shapes.values()), dtype=torch.bfloat16, device=dev)
    Wt = torch.randn(max((2 if epi == 3 else 1) * N * K for _, N, K, epi in shapes.values()),
                     dtype=torch.bfloat16, device=dev) * 0.02
    max_n = max(N for _, N, _, _ in shapes.values())
    bias = torch.zeros(max_n, dtype=torch.bfloat16, device=dev)
    out_b = torch.empty(T * max_n, dtype=torch.bfloat16, device=dev)
    out_f = torch.zeros(T * d, dtype=torch.float32, device=dev)
    for key, (Mm, N, K, epi) in shapes.items():
        o = out_f if epi == 2 else out_b
        bb = None if (epi == 3 or qwen) else bias
        us = timed(lambda: zo.zo_gemm_bf16(ctx, A, Wt, bb, o, Mm, N, K, N, epi))
        fl = 2.0 * Mm * N * K * (2 if epi == 3 else 1)
        out["gemm_" + key] = {"shape": [Mm, N, K], "us": us, "tflops": fl / us / 1e6,
                              "frac_bf16_burst": fl / us / 1e6 / peak_b, "sm_mhz": clocks[0]}
    if not qwen:
        # the perturbation fused into the GEMM's operand path (single-CTA form: every row tile
        # regenerates the signs of the weight tiles it reads) against the window path (the
        # layer's weights perturbed into a window once, then the GEMM on the window)
        cw = zo.zo_create(Wt, seed=0, stream=stream.cuda_stream)
        zo.zo_perturb(cw, +1, 1e-3, 3)
        win = torch.empty(max(N * K for _, N, K, _ in shapes.values()), dtype=torch.bfloat16, device=dev)
        fused = {}
        for key, (Mm, N, K, epi) in shapes.items():
            o = out_f if epi == 2 else out_b
            us_f = timed(lambda: zo.zo_gemm_bf16_perturbed(cw, A, 0, bias, o, Mm, N, K, N, epi))
            mhz_f = clocks[0]
            us_w = timed(lambda: (zo.zo_perturb_range(cw, 0, N * K, win),
                                  zo.zo_gemm_bf16(ctx, A, win, bias, o, Mm, N, K, N, epi)))
            fused[key] = {"shape": [Mm, N, K], "fused_us": us_f, "window_then_gemm_us": us_w,
                          "fused_over_window": us_f / us_w, "sm_mhz": [mhz_f, clocks[0]]}
        zo.zo_restore(cw)
        zo.zo_sync(cw)
        cw.close()
        del win
        out["fused_perturbation"] = fused
    del A, Wt, out_b, out_f
    qkv = torch.randn(T * nq, dtype=torch.bfloat16, device=dev)
    att = torch.empty(T * na, dtype=torch.bfloat16, device=dev)
    us = timed(lambda: zo.zo_attention_gqa(ctx, qkv, att, B, S, H, Hk, e))
    fl = 4.0 * e * B * H * S * (S + 1) / 2
    out["attention"] = {"us": us, "tflops": fl / us / 1e6, "frac_bf16_burst": fl / us / 1e6 / peak_b,
                        "sm_mhz": clocks[0]}
    del qkv, att
    ctx.close()
    print(json.dumps({"kernels_only": name, "batch": B, "seq": S, "reps": reps,
                      "l2": "flushed before every timed launch", "kernels": out}), flush=True)
    return 0


def decoder_cpu_baseline(name, cfg, w, fwds):
    """The oracle's fp64 forward of one layer at the real width (1 x 64 tokens, vocabulary
    cut to 4096: it only feeds the embedding gather and the 2-row head), one thread; the full
    step extrapolated linearly in layers and tokens."""
    B, S = w["batch"], w["seq"]
    qwen = cfg.get("family") == "qwen3"
    red = dict(cfg, n_layers=1, vocab=4096)
    seq = 64
    tps = oracle_workers([("forward", "qwen3" if qwen else "opt", json.dumps(red), seq)])[0]["tokens_per_s"]
    cpu_step_s = fwds * B * S * cfg["n_layers"] / tps
    return {"value": 1.0 / cpu_step_s, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "extrapolated": True,
            "sample": f"oracle fp64 forward of 1 layer at the real width, 1 x {seq} tokens "
                      f"(vocabulary cut to 4096): {tps:.2f} tokens/s on one thread; the step "
                      f"extrapolated linearly in layers and tokens ({fwds} forwards of {B * S} "
                      f"tokens x {cfg['n_layers']} layers); attention's quadratic term at the "
                      f"full length not included",
            "host": host_cpu()}


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
                    help="timed steps (default: 3 for the decoders, 300 for the quadratic "
                         "workloads and the MLP)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quadratic", action="store_true",
                    help="leave out the quadratic sub-record of the default workload's line")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the quadratic's loss kernel, if measured")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=["quadratic", "mlp", "lowrank"] + sorted(DECODER_WORKLOADS))
    ap.add_argument("--n-pert", type=int, default=None, help="override n_pert (decoder workloads)")
    ap.add_argument("--streaming-only", action="store_true",
                    help="only the streaming sweep (update over n_pert, window perturbation); "
                         "prints a diagnostic line")
    ap.add_argument("--kernels-only", action="store_true",
                    help="time each hot kernel of a decoder workload alone at its shapes "
                         "(--steps = timed launches per kernel); prints a diagnostic line")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 3 if args.workload in DECODER_WORKLOADS else 300
    if args.warmup < 3 and args.workload in ("quadratic",) + tuple(DECODER_WORKLOADS):
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args)
    if args.streaming_only:
        return streaming_arm(args)
    if args.kernels_only:
        if args.workload not in DECODER_WORKLOADS:
            ap.error("--kernels-only needs a decoder workload")
        return kernels_arm(args)
    if args.workload == "mlp":
        return mlp_arm(args)
    if args.workload == "lowrank":
        return lowrank_arm(args)
    if args.workload != "quadratic":
        return decoder_arm(args)
    line = gpu_arm(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
