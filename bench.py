#!/usr/bin/env python
"""Throughput of beam-parallel Gated DeltaNet decode (projection replay) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stress]
    python bench.py --impl reference ...        # the FP64 CPU oracle on the host cores

One bench step = one whole decode of the workload: ola_reset and T ola_step calls over
every request, beam and head (plan kernel + fused tensor-core replay kernel per call), with
all inputs resident in HBM. The metric is beam-head decode steps per second, R*H*B*T per
bench step, summed over ranks (requests are independent: every rank decodes its own batch
of requests, weak scaling, no collective on the data path; barrier + max over ranks for the
timing). Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "beam-head decode steps/s (GDN projection replay) and % of roofline, 1×B200"
UNIT = "beam-head-steps/s"


# ----------------------------------------------------------------------------- roofline

def algorithmic_bytes_per_step(w: wl.Workload, parents: np.ndarray) -> list:
    """Compulsory HBM bytes of each decode step t (one ola_step launch), summed over requests
    and heads: the shared state read once, q/k/v/g/beta read, o written, the new record
    (w_t fp32, k_t, alpha_t) written, every distinct ancestor record read once, the parent
    row read and the chain row written."""
    e = w.elem_bytes
    dk, dv, B, H = w.d_k, w.d_v, w.B, w.H
    U = wl.distinct_ancestor_counts(parents)          # [T, R]
    rec = 4 * dv + e * dk + 4
    out = []
    for t in range(w.T):
        per_rh = 4 * dv * dk + B * ((2 * dk + dv) * e + 8) + 4 * B * dv + B * rec
        total = w.R * H * per_rh + H * int(U[t].sum()) * rec + w.R * 4 * B * (t + 2)
        out.append(total)
    return out


def state_and_record_bytes_per_step(w: wl.Workload, parents: np.ndarray) -> list:
    """The part of each step's compulsory bytes that the method itself names: the shared state
    read once per (request, head), the new records written and the distinct ancestor records
    read (no q/k/v/g/beta, o, parent or chain bytes)."""
    dk, dv, B, H = w.d_k, w.d_v, w.B, w.H
    U = wl.distinct_ancestor_counts(parents)
    rec = 4 * dv + w.elem_bytes * dk + 4
    return [w.R * H * (4 * dv * dk + B * rec) + H * int(U[t].sum()) * rec for t in range(w.T)]


def tensor_flops_per_step(w: wl.Workload) -> int:
    return 4 * w.d_v * w.d_k * w.B * w.R * w.H


def algorithmic_flops_per_step(w: wl.Workload) -> list:
    """Floating-point operations the projection replay performs at each decode step t, counted
    per beam as the method states them (a multiply-add is two): the two shared-state
    contractions S_ctx q and S_ctx k (4 d_v d_k), the t - 1 ancestors' key products with k and q
    (4 d_k each) and their accumulation into u and o (4 d_v each), and the new record and the
    output (8 d_v)."""
    dk, dv = w.d_k, w.d_v
    return [w.R * w.H * w.B * (4 * dv * dk + 4 * t * (dk + dv) + 8 * dv) for t in range(w.T)]


def fullstate_flops_per_step(w: wl.Workload) -> list:
    """Floating-point operations of the FullState recurrence per step: per beam S k, the rank-1
    update alpha (S - beta u k^T) + beta v k^T and S q, 8 d_v d_k."""
    return [w.R * w.H * w.B * 8 * w.d_v * w.d_k for _ in range(w.T)]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("ola_replay_mma.cu", "ola_plan.cu", "ola_device.cuh"):
        h.update(open(os.path.join(ROOT, "linear_attention_beam_gdn_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the replay kernel from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "replay_mma_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_src_sha") != kernel_source_hash() or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        # nvidia-smi needs a moment before its first sample: start the timed region only once
        # it is sampling, so that a short region (tens of ms) still gets samples of its own
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": mx,
                "samples": len(sms), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- oracle baseline

def _oracle_unit_prefill(args):
    import oracle
    k, v, g, b = args
    return oracle.prefill(k, v, g, b)


def _oracle_unit_decode(args):
    import oracle
    S, q, k, v, g, b, par = args
    return oracle.full_state_decode(S, q, k, v, g, b, par)


def _pool(cores):
    import multiprocessing as mp
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
    os.environ.setdefault("MKL_NUM_THREADS", "1")
    return mp.get_context("spawn").Pool(cores)


def oracle_sample(w: wl.Workload, prompt_units, step_units, parents, pool, cores):
    """Time the oracle's full-state decode on the sampled (r, h) units (its own fp64 prefill
    of their prompts runs first, untimed). Returns (seconds, beam-head-steps)."""
    S = pool.map(_oracle_unit_prefill, prompt_units)
    jobs = [(S[i],) + tuple(step_units[i]) + (parents[i],) for i in range(len(S))]
    t0 = time.perf_counter()
    pool.map(_oracle_unit_decode, jobs)
    dt = time.perf_counter() - t0
    return dt, len(jobs) * w.B * w.T


def host_units(w, prompt, steps, parents, units):
    import oracle
    pu, su, pa = [], [], []
    for r, h in units:
        pu.append(tuple(oracle.as_f64(prompt[x][r, :, h]) for x in ("k", "v", "g", "beta")))
        su.append(tuple(np.stack([oracle.as_f64(s[x][r, :, h]) for s in steps])
                        for x in ("q", "k", "v", "g", "beta")))
        pa.append(parents[:, r])
    return pu, su, pa


def sample_units(w, n, seed=7):
    rng = np.random.default_rng(seed)
    allu = [(r, h) for r in range(w.R) for h in range(w.H)]
    idx = rng.permutation(len(allu))[:n]
    return [allu[i] for i in idx]


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cores = len(os.sched_getaffinity(0))
    pool = _pool(cores)
    for name in args.workload.split(","):
        reference_line(wl.WORKLOADS[name], args, pool, cores)
    pool.close()
    return 0


def reference_line(w: wl.Workload, args, pool, cores) -> None:
    """The oracle on the host cores, timed on a bounded sample of workload `w`."""
    n_units = min(w.R * w.H, args.cpu_units or max(2, 2 * cores))
    units = sample_units(w, n_units)
    import torch
    prompt = wl.make_prompt(w.scaled(R=max(r for r, _ in units) + 1), "cpu")
    steps = [wl.make_step_inputs(w, t, "cpu", R=max(r for r, _ in units) + 1)
             for t in range(w.T)]
    parents = wl.make_parents(w)
    pu, su, pa = host_units(w, prompt, steps, parents, units)
    for _ in range(args.warmup):
        oracle_sample(w, pu[:cores], su[:cores], pa[:cores], pool, cores)
    times, work = [], 0
    for _ in range(args.steps):
        dt, n = oracle_sample(w, pu, su, pa, pool, cores)
        times.append(dt)
        work = n
    total = sum(times)
    value = work * args.steps / total
    sample = (f"{n_units} of {w.R * w.H} (request, head) units, all {w.B} beams x {w.T} steps; "
              f"fp64 prefill of those units untimed")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": describe(w), "parallelism": "host cores (process pool)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def describe(w: wl.Workload) -> str:
    cap = f", <= {w.max_children} children" if w.max_children else ""
    return (f"{w.name}: R={w.R} requests x H={w.H} heads, d_k={w.d_k}, d_v={w.d_v}, "
            f"prompt P={w.P}, B={w.B} beams, T={w.T} decode steps, {w.parent_law}"
            f"({w.zipf_s}) parents{cap}, {w.dtype} q/k/v, fp32 S_ctx")


# ----------------------------------------------------------------------------- ranks

def rank_workload(base: wl.Workload, rank: int) -> wl.Workload:
    """Weak scaling: every rank decodes its own batch of base.R requests (its own seeds)."""
    return base.scaled(seed=base.seed + 7919 * rank)


def job_value(world: int, units_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed in `steps` bench steps, over the
    slowest rank's time (ms)."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank number over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    tt = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    import linear_attention_beam_gdn_b200 as ola

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(x: float) -> float:
        return max_over_ranks(x, world, dev)

    cores = len(os.sched_getaffinity(0))
    pool = None
    do_cpu = (not args.no_cpu_baseline) and rank == 0 and world == 1
    if do_cpu:
        pool = _pool(cores)                              # spawn before the first GPU call
    ctx = dict(torch=torch, ola=ola, world=world, rank=rank, local=local, dev=dev,
               barrier=barrier, max_ranks=max_ranks, cores=cores, pool=pool, do_cpu=do_cpu)
    for name in args.workload.split(","):
        base = wl.WORKLOADS[name]
        if args.requests:
            base = base.scaled(R=args.requests)
        result = bench_workload(rank_workload(base, rank), args, ctx)
        if rank == 0:
            print(json.dumps(result), flush=True)
    if pool is not None:
        pool.close()
        pool.join()
    if world > 1:
        dist.destroy_process_group()
    return 0


def capture_decode(torch, ola, dec, decode, stream):
    """Record one call of `decode` (ola_reset + T ola_step calls through the C ABI, taking the
    current stream) into a CUDA graph on a side stream. Returns (graph, note); graph is None if
    the capture failed here, and the caller then issues decodes eagerly."""
    try:
        cap = torch.cuda.Stream(device=stream.device)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            decode(dec)                           # the handle's last stream becomes `cap`
        cap.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap, capture_error_mode="thread_local"):
            decode(dec)
        graph.replay()
        torch.cuda.synchronize()
        if dec.error() != ola.OLA_OK:
            raise RuntimeError("device error in the captured decode")
        return graph, ("CUDA graph of one whole decode (ola_reset + T ola_step calls through the "
                       "C ABI), replayed K times")
    except Exception as ex:                       # noqa: BLE001 - report and time eagerly
        torch.cuda.synchronize()
        dec.reset()
        return None, f"eager (graph capture failed: {type(ex).__name__})"


def tensor_path_ok(w: wl.Workload) -> bool:
    return w.dtype == "bf16" and w.d_k in (64, 128, 256) and w.d_v in (64, 128, 256)


def replay_kernel_label(w: wl.Workload) -> str:
    """The kernels one ola_step launches on the tensor path for this geometry."""
    if w.d_k in (64, 128, 256) and w.d_v in (64, 128, 256) and w.B <= 1024 and w.T <= 12:
        return f"ola::plan_units_kernel + ola::replay_mma_kernel<{w.d_k}, {w.d_v}>"
    if w.d_v == 128 and w.d_k <= 128:
        return f"ola::plan_units_kernel + ola::replay_pipe_kernel<{w.d_k}>"
    if w.d_v == 64 and w.d_k <= 128:
        return f"ola::plan_kernel + ola::replay_pos_kernel<{w.d_k}, {w.d_v}, 64>"
    return "ola::plan_kernel + ola::replay_tc_kernel"


def bench_workload(w: wl.Workload, args, ctx) -> dict:
    """One bench line: the timed decode of workload `w` and its side measurements."""
    torch, ola, dev = ctx["torch"], ctx["ola"], ctx["dev"]
    world, rank, local = ctx["world"], ctx["rank"], ctx["local"]
    barrier, max_ranks = ctx["barrier"], ctx["max_ranks"]
    cores, pool, do_cpu = ctx["cores"], ctx["pool"], ctx["do_cpu"]

    # ---- inputs resident in HBM; shared state by the library's prefill kernel
    prompt = wl.make_prompt(w, dev)
    S = ola.prefill(prompt["k"], prompt["v"], prompt["g"], prompt["beta"])
    steps = [wl.make_step_inputs(w, t, dev) for t in range(w.T)]
    parents = wl.make_parents(w)
    par_dev = [torch.from_numpy(parents[t]).to(dev) for t in range(w.T)]
    units = sample_units(w, min(w.R * w.H, args.cpu_units or max(2, 2 * cores))) if do_cpu else []
    host = host_units(w, prompt, steps, parents, units) if do_cpu else None
    torch.cuda.synchronize()

    outs = [torch.empty((w.R, w.B, w.H, w.d_v), device=dev) for _ in range(w.T)]
    stream = torch.cuda.current_stream()

    def decode(dec, evs=None):
        dec.reset()
        for t in range(w.T):
            s = steps[t]
            if evs is not None:
                evs[t][0].record(stream)
            dec.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par_dev[t], out=outs[t])
            if evs is not None:
                evs[t][1].record(stream)

    # the tensor-core path takes bf16 inputs and widths 64, 128, 256; other workloads (the tiny
    # fp32 one) decode on the fp32 replay path
    tensor = tensor_path_ok(w)
    dec = ola.Decoder(S, B=w.B, T_max=w.T, in_dtype=w.torch_dtype, path=ola.OLA_PATH_REPLAY,
                      math=ola.OLA_MATH_TENSOR if tensor else ola.OLA_MATH_FP32)
    for _ in range(args.warmup):
        decode(dec)
    torch.cuda.synchronize()
    st = dec.error()
    if st != ola.OLA_OK:
        raise RuntimeError(f"device error during warm-up: {ola.ola_strerror(st)}")

    K = args.steps
    # One bench step = one whole decode. By default the decode (ola_reset + T ola_step calls,
    # issued through the C ABI on a side stream) is recorded once into a CUDA graph and the timed
    # region replays it K times, so that the host's per-call work (argument checks, tensor maps,
    # launches) is not on the device timeline; every kernel of every step still runs.
    graph, timing = None, "eager: K decodes issued through the C ABI"
    if not args.no_graph:
        graph, timing = capture_decode(torch, ola, dec, decode, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for k in range(K):
            if graph is not None:
                graph.replay()
            else:
                decode(dec)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    st = dec.error()
    if st != ola.OLA_OK:
        raise RuntimeError(f"device error in the timed region: {ola.ola_strerror(st)}")
    ms = max_ranks(e0.elapsed_time(e1))
    # per-step breakdown (not the metric): eager decodes with CUDA events around every ola_step
    K2 = min(K, 20)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(w.T)]
           for _ in range(K2)]
    for k in range(K2):
        decode(dec, evs[k])
    torch.cuda.synchronize()
    step_ms = np.array([[evs[k][t][0].elapsed_time(evs[k][t][1]) for t in range(w.T)]
                        for k in range(K2)])
    per_launch_ms = step_ms.mean(axis=0)               # ola_step t, averaged over K2
    units_per_step = w.R * w.H * w.B * w.T
    value = job_value(world, units_per_step, K, ms)

    # ---- roofline of the step kernel
    peaks = measured_peaks()
    bytes_t = algorithmic_bytes_per_step(w, parents)
    lit_t = state_and_record_bytes_per_step(w, parents)
    # one decode's algorithmic bytes over its device time in the timed region (plan kernels
    # included)
    achieved = sum(bytes_t) / (ms / K / 1e3) / 1e9
    flops = tensor_flops_per_step(w) * w.T
    tensor_time = flops / (peaks["bf16_tflops"] * 1e12) if tensor else 0.0
    hbm_time = sum(bytes_t) / (peaks["hbm_gbs"] * 1e9)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "traffic": recorded_traffic(w.name),
                "kernel": "ola_step = " + (replay_kernel_label(w) if tensor else
                                           "ola::replay_simt_kernel"),
                "algorithmic_bytes_per_decode": int(sum(bytes_t)),
                "frac_state_and_records_only": sum(lit_t) / (ms / K / 1e3) / 1e9 /
                                               peaks["hbm_gbs"],
                "algorithmic_bytes_per_launch": [int(b) for b in bytes_t],
                "launch_ms_eager": [round(float(x), 4) for x in per_launch_ms],
                "timed_over": "one decode of the timed region (K graph replays / K)",
                "t_roof_ms": 1e3 * max(tensor_time, hbm_time),
                "peak_source": peaks["source"] + " (MEASURED_PEAKS.json hbm_gbs)"}

    result = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
              "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
              "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if tensor else "f32",
              "data": "synthetic",
              "config": {"workload": describe(w), "R": w.R, "H": w.H, "d_k": w.d_k,
                         "d_v": w.d_v, "B": w.B, "T": w.T, "P": w.P,
                         "path": ("replay, tcgen05 tensor cores (bf16 hi/lo S_ctx, fp32 "
                                  "accumulate and epilogue)" if tensor else
                                  "replay, fp32 on CUDA cores"),
                         "l2": ("no flush: each decode step streams %.2f GB (> 126 MB L2)"
                                % (max(bytes_t) / 1e9) if max(bytes_t) > 126e6 else
                                "no flush: each decode step streams %.0f MB, inside the 126 MB "
                                "L2 (a small configuration; its time is launch- and "
                                "latency-bound)" % (max(bytes_t) / 1e6)),
                         "parallelism": f"replicas x{world} (requests sharded, no collective)",
                         "timing": timing},
              "roofline": roofline, "clocks": clocks,
              "gpu_launches": (2 if tensor else 1) * w.T * K}

    # ---- in-library comparisons on the same inputs (not part of the metric)
    comps = {}
    if not args.no_compare:
        for name, p, m, reps in (("replay_fp32", ola.OLA_PATH_REPLAY, ola.OLA_MATH_FP32, 2),
                                 ("fullstate", ola.OLA_PATH_FULLSTATE, ola.OLA_MATH_FP32, 2),
                                 ("replayssm", ola.OLA_PATH_REPLAYSSM, ola.OLA_MATH_FP32, 2)):
            try:
                d2 = ola.Decoder(S, B=w.B, T_max=w.T, in_dtype=w.torch_dtype, path=p, math=m)
            except ola.OlaError as ex:
                comps[name] = {"skipped": str(ex)}
                continue
            decode(d2)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                decode(d2)
            b.record(stream)
            torch.cuda.synchronize()
            mms = max_ranks(a.elapsed_time(b)) / reps
            comps[name] = {"ms_per_step": mms, "value": world * units_per_step / (mms / 1e3),
                           "replay_tensor_speedup": mms / (ms / K)}
            d2.close()
            del d2
            torch.cuda.empty_cache()
    result["compare"] = comps

    # ---- end to end through the host-buffer entry point (pinned memory)
    if not args.no_e2e:
        hs = [{k: v.cpu().pin_memory() for k, v in s.items()} for s in steps]
        hp = [torch.from_numpy(parents[t]).pin_memory() for t in range(w.T)]
        houts = [torch.empty((w.R, w.B, w.H, w.d_v), dtype=torch.float32).pin_memory()
                 for _ in range(w.T)]
        h2d = sum(v.numel() * v.element_size() for s in hs for v in s.values()) + \
            sum(p.numel() * 4 for p in hp)
        d2h = sum(o.numel() * 4 for o in houts)

        def decode_host():
            # pipelined: a step's o is copied back while the next step's inputs go in
            dec.reset()
            for t in range(w.T):
                s = hs[t]
                dec.step_host_async(s["q"], s["k"], s["v"], s["g"], s["beta"], hp[t], houts[t])
            dec.host_sync()

        decode_host()
        barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            decode_host()
        dt = max_ranks(time.perf_counter() - t0)
        result["e2e"] = {"value": world * units_per_step * args.e2e_steps / dt, "unit": UNIT,
                         "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                         "ms_per_step": 1e3 * dt / args.e2e_steps,
                         "via": "ola_step_host_async + ola_host_sync (pinned host buffers; one "
                                "cudaMemcpyAsync per tensor; copy-in and copy-out on two streams)"}
        if dec.error() != ola.OLA_OK:
            raise RuntimeError("device error in the end-to-end run")
        del hs, hp, houts

    dec.close()

    # ---- CPU oracle baseline (rank 0, N = 1)
    if do_cpu:
        pu, su, pa = host
        dt, n = oracle_sample(w, pu, su, pa, pool, cores)
        result["cpu_baseline"] = {
            "value": n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(pu)} of {w.R * w.H} (request, head) units of this workload, all "
                      f"{w.B} beams x {w.T} steps, fp64 full-state recurrence; the units' "
                      f"fp64 prefill untimed", "seconds": dt}

    # ---- the prompt prefill on its own (after the oracle's host processes have finished:
    # the chunked form waits for its kernel inside the call, so host load would show)
    pf_ms = time_prefill(prompt)
    pf_bytes = prefill_bytes(w)
    result["prefill"] = {
        "what": "shared state from the prompt (once per request batch, outside the timed "
                "decode steps); chunked tensor-core form for 128x128 bf16, else token by token",
        "ms": pf_ms, "algorithmic_bytes": pf_bytes,
        "achieved_gbs": pf_bytes / (pf_ms / 1e3) / 1e9,
        "hbm_frac": pf_bytes / (pf_ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    del S, steps, par_dev, outs, prompt
    torch.cuda.empty_cache()
    return result


# ----------------------------------------------------------------------------- operator sweep

SWEEP_GEOMETRIES = tuple((dk, dv) for dk in (64, 128, 256) for dv in (64, 128, 256))
SWEEP_REQUESTS = (1, 2, 8, 32, 64)
SWEEP_BEAMS = (64, 256, 512)
SWEEP_STEPS = (2, 4, 8)
SWEEP_FULLSTATE_LIMIT = 96 << 30      # bytes of FullState ping-pong state the sweep allocates


def prefill_bytes(w: wl.Workload) -> int:
    """Bytes the prefill must move: the prompt's k, v (input dtype), g and beta (fp32) read
    once, the fp32 state of every (request, head) written once."""
    e = 2 if w.dtype == "bf16" else 4
    return w.R * w.P * w.H * ((w.d_k + w.d_v) * e + 8) + w.R * w.H * w.d_v * w.d_k * 4


def time_prefill(prompt, reps: int = 5) -> float:
    """Median device time (ms, CUDA events) of ola.prefill on the resident prompt."""
    import torch
    import linear_attention_beam_gdn_b200 as ola
    for _ in range(2):                                   # warm-up
        ola.prefill(prompt["k"], prompt["v"], prompt["g"], prompt["beta"])
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        ola.prefill(prompt["k"], prompt["v"], prompt["g"], prompt["beta"])
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return float(np.median(ts))


def fullstate_bytes_per_step(w: wl.Workload, parents: np.ndarray) -> list:
    """Compulsory HBM bytes of each FullState step: every distinct parent's state read once
    (step 1: the shared state), every beam's state written (fp32 d_v x d_k each), plus the
    step inputs and o."""
    e = w.elem_bytes
    state = 4 * w.d_v * w.d_k
    per_beam = state + (2 * w.d_k + w.d_v) * e + 8 + 4 * w.d_v
    out = []
    for t in range(w.T):
        n_par = 1 if t == 0 else sum(len(np.unique(parents[t, r])) for r in range(w.R)) / w.R
        out.append(int(w.R * w.H * (w.B * per_beam + n_par * state)))
    return out


def sweep_shapes(args):
    """The sweep's grid (or the subset the --sweep-* options select), as (d_k, d_v, R, B, T)."""
    geoms = SWEEP_GEOMETRIES if not args.sweep_geometry else \
        tuple(tuple(int(x) for x in g.split("x")) for g in args.sweep_geometry.split(","))
    Rs = SWEEP_REQUESTS if not args.sweep_requests else \
        tuple(int(x) for x in args.sweep_requests.split(","))
    Bs = SWEEP_BEAMS if not args.sweep_beams else tuple(int(x) for x in args.sweep_beams.split(","))
    Ts = SWEEP_STEPS if not args.sweep_steps else tuple(int(x) for x in args.sweep_steps.split(","))
    return [(dk, dv, R, B, T) for dk, dv in geoms for R in Rs for B in Bs for T in Ts]


def run_sweep_model(args):
    """Host-side models of every sweep shape, no GPU: each path's compulsory bytes and FLOPs per
    decode, their ratio (arithmetic intensity, FLOP per byte) against the machine balance of
    the measured peaks (dense bf16 tensor FLOP/s over HBM bytes/s), and the capacity bytes. The
    workloads and parent tables are those the timed sweep uses (same seeds)."""
    peaks = measured_peaks()
    balance = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    for dk, dv, R, B, T in sweep_shapes(args):
        w = wl.Workload(f"sweep_dk{dk}_dv{dv}_R{R}_B{B}_T{T}", R=R, H=16, d_k=dk, d_v=dv,
                        P=1024, B=B, T=T, parent_law="zipf", zipf_s=1.0, seed=1005)
        parents = wl.make_parents(w)
        rb, rf = sum(algorithmic_bytes_per_step(w, parents)), sum(algorithmic_flops_per_step(w))
        fb, ff = sum(fullstate_bytes_per_step(w, parents)), sum(fullstate_flops_per_step(w))
        print(json.dumps({
            "d_k": dk, "d_v": dv, "R": R, "H": w.H, "B": B, "T": T,
            "replay": {"bytes": int(rb), "flops": int(rf), "flop_per_byte": rf / rb},
            "fullstate": {"bytes": int(fb), "flops": int(ff), "flop_per_byte": ff / fb},
            "machine_balance_flop_per_byte": balance,
            "capacity": {"replay_record_bytes_per_beam_head_step": 4 * dv + w.elem_bytes * dk + 4,
                         "replay_shared_state_bytes_per_request_head": 4 * dv * dk,
                         "fullstate_bytes_per_beam_head": 4 * dv * dk}}), flush=True)
    return 0


def run_sweep(args):
    """The operator sweep: nine (d_k, d_v) geometries x request counts x beam widths x decode
    lengths (405 shapes), H = 16 heads, bf16 inputs, Zipf(1.0) parents, a shared state from a
    1K-token prompt. Per shape: replay (tensor path) and FullState time per decode (CUDA-graph
    replays of one decode, as in the bench; --no-graph for eager calls), capacity
    bytes, algorithmic DRAM bytes and the fraction of the measured HBM bandwidth, and the
    largest |o| difference between the two paths. One JSON line per shape."""
    import torch
    import linear_attention_beam_gdn_b200 as ola

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    shapes = sweep_shapes(args)
    geoms = tuple(dict.fromkeys((dk, dv) for dk, dv, _, _, _ in shapes))
    Rs = tuple(dict.fromkeys(R for _, _, R, _, _ in shapes))
    Bs = tuple(dict.fromkeys(B for _, _, _, B, _ in shapes))
    Ts = tuple(dict.fromkeys(T for _, _, _, _, T in shapes))
    stream = torch.cuda.current_stream()

    def timed(dec, steps, par, outs, reps, warm):
        def decode(d):
            d.reset()
            for t in range(len(steps)):
                s = steps[t]
                d.step(s["q"], s["k"], s["v"], s["g"], s["beta"], par[t], out=outs[t])
        for _ in range(warm):
            decode(dec)
        torch.cuda.synchronize()
        graph = None
        if not args.no_graph and reps > 0:
            graph, _ = capture_decode(torch, ola, dec, decode, stream)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            if graph is not None:
                graph.replay()
            else:
                decode(dec)
        b.record(stream)
        torch.cuda.synchronize()
        if dec.error() != ola.OLA_OK:
            raise RuntimeError(f"device error: {ola.ola_strerror(dec.error())}")
        del graph
        return a.elapsed_time(b) / max(reps, 1)

    for dk, dv in geoms:
        for R in Rs:
            base = wl.Workload(f"sweep_dk{dk}_dv{dv}_R{R}", R=R, H=16, d_k=dk, d_v=dv, P=1024,
                               B=max(Bs), T=max(Ts), parent_law="zipf", zipf_s=1.0, seed=1005)
            prompt = wl.make_prompt(base, dev)
            S = ola.prefill(prompt["k"], prompt["v"], prompt["g"], prompt["beta"])
            del prompt
            for B in Bs:
                for T in Ts:
                    w = base.scaled(name=f"sweep_dk{dk}_dv{dv}_R{R}_B{B}_T{T}", B=B, T=T)
                    steps = [wl.make_step_inputs(w, t, dev) for t in range(T)]
                    parents = wl.make_parents(w)
                    par = [torch.from_numpy(parents[t]).to(dev) for t in range(T)]
                    outs = [torch.empty((R, B, w.H, dv), device=dev) for _ in range(T)]
                    row = {"d_k": dk, "d_v": dv, "R": R, "H": w.H, "B": B, "T": T}
                    bh_steps = R * w.H * B * T
                    dec = ola.Decoder(S, B=B, T_max=T, in_dtype=w.torch_dtype,
                                      path=ola.OLA_PATH_REPLAY, math=ola.OLA_MATH_TENSOR)
                    t1 = timed(dec, steps, par, outs, 1, args.sweep_warmup)
                    reps = max(1, min(args.sweep_reps, int(200.0 / max(t1, 1e-3))))
                    ms = timed(dec, steps, par, outs, reps, 0)
                    dec.close()
                    rb = sum(algorithmic_bytes_per_step(w, parents))
                    rf = sum(algorithmic_flops_per_step(w))
                    row["replay"] = {"ms": ms, "beam_head_steps_per_s": bh_steps / (ms / 1e3),
                                     "bytes": int(rb), "gbs": rb / (ms / 1e3) / 1e9,
                                     "hbm_frac": rb / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                                     "flops": int(rf), "flop_per_byte": rf / rb}
                    o_rep = [o.clone() for o in outs] if args.sweep_check else None
                    fsb = 2 * R * w.H * B * dv * dk * 4
                    row["capacity"] = {
                        "replay_record_bytes_per_beam_head_step": 4 * dv + w.elem_bytes * dk + 4,
                        "replay_shared_state_bytes_per_request_head": 4 * dv * dk,
                        "fullstate_bytes_per_beam_head": 4 * dv * dk,
                        "fullstate_pingpong_bytes": fsb}
                    if fsb <= SWEEP_FULLSTATE_LIMIT and not args.sweep_no_fullstate:
                        dec = ola.Decoder(S, B=B, T_max=T, in_dtype=w.torch_dtype,
                                          path=ola.OLA_PATH_FULLSTATE, math=ola.OLA_MATH_FP32)
                        t1 = timed(dec, steps, par, outs, 1, min(args.sweep_warmup, 1))
                        reps = max(1, min(args.sweep_reps, int(200.0 / max(t1, 1e-3))))
                        fms = timed(dec, steps, par, outs, reps, 0)
                        dec.close()
                        fb = sum(fullstate_bytes_per_step(w, parents))
                        ff = sum(fullstate_flops_per_step(w))
                        row["fullstate"] = {"ms": fms, "bytes": int(fb), "flops": int(ff),
                                            "flop_per_byte": ff / fb,
                                            "gbs": fb / (fms / 1e3) / 1e9,
                                            "hbm_frac": fb / (fms / 1e3) / 1e9 / peaks["hbm_gbs"],
                                            "replay_speedup": fms / ms}
                        if o_rep is not None:
                            row["max_abs_diff_replay_vs_fullstate"] = max(
                                float((a - b).abs().max()) for a, b in zip(o_rep, outs))
                    else:
                        row["fullstate"] = {"skipped": f"{fsb / 2**30:.1f} GiB of ping-pong state"}
                    print(json.dumps(row), flush=True)
                    del steps, par, outs, o_rep
                    torch.cuda.empty_cache()
            del S
            torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="stress",
                    help="workload name, or several separated by commas (one JSON line each): "
                         + ", ".join(sorted(wl.WORKLOADS)))
    ap.add_argument("--cpu-units", type=int, default=0,
                    help="(request, head) units of the CPU oracle sample (default 2 x cores)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-compare", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eagerly issued decodes instead of CUDA-graph replays")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--requests", type=int, default=0,
                    help="override the workload's request count (profiling a smaller case)")
    ap.add_argument("--sweep", action="store_true",
                    help="run the operator sweep (one JSON line per shape) instead of the bench")
    ap.add_argument("--sweep-geometry", default="", help="e.g. 128x128,256x64 (d_k x d_v)")
    ap.add_argument("--sweep-requests", default="")
    ap.add_argument("--sweep-beams", default="")
    ap.add_argument("--sweep-steps", default="")
    ap.add_argument("--sweep-reps", type=int, default=10)
    ap.add_argument("--sweep-warmup", type=int, default=2)
    ap.add_argument("--sweep-check", action="store_true",
                    help="also report the largest |o| difference between replay and FullState")
    ap.add_argument("--sweep-no-fullstate", action="store_true")
    ap.add_argument("--sweep-model", action="store_true",
                    help="print the sweep's byte, FLOP and capacity models per shape (no GPU)")
    args = ap.parse_args()
    for name in args.workload.split(","):
        if name not in wl.WORKLOADS:
            ap.error(f"unknown workload {name}")
    if args.sweep_model:
        return run_sweep_model(args)
    if args.sweep:
        return run_sweep(args)
    if args.warmup < 3 and args.impl == "ours":
        print("warm-up raised to 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
