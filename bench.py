#!/usr/bin/env python
"""Benchmark of the fused chunked top-K KL loss (forward + backward) on B200.

One step = one fused forward+backward call of the whole path over one batch
of synthetic inputs (teacher-cache preparation, logits + online log-sum-exp
+ teacher gather, lse merge and loss, then per chunk the logit recompute
into dZ and the joint dH = dZ W / dW += dZ^T H launch).  Inputs are resident
in HBM before the timed region starts.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config I] [--N TOKENS]
  python bench.py --impl reference ...      # the fp64 CPU oracle, timed on the host
  python bench.py --op teacher-topk ...     # the offline teacher top-K cache writer

For N > 1 it runs under torch.distributed.run, one process per GPU; each
rank computes an independent replica (the path has no exchange step), the
timed region is bracketed by barriers, and the time is the maximum over
ranks.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused top-K KL fwd+bwd tokens/s, TFLOP/s (% bf16 tensor peak); peak HBM GiB"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_CONFIG = 3
L2_BYTES = 126 * 2**20
# Sources of the loss path's kernels (the teacher top-K select is not on it); their hash dates the
# committed DRAM-traffic capture.
KERNEL_SOURCES = ["kd_gemm.cuh", "kd_ptx.cuh", "kd_schedule.h", "kd_small_kernels.cuh", "kd_topk_kl.cu"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dominant_kernel_traffic.txt")


# ---------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "chunked_top_kl_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on this workload, for this kernel and on the current sources."""
    try:
        kv = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if (kv.get("source_hash") != kernel_source_hash() or kv.get("workload") != workload
                or kv.get("kernel") != kernel):
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup(impl: str):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and impl == "cuda":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def reduce_max(value: float, world: int, device) -> float:
    """Maximum of a per-rank scalar over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# Below this many tokens the row compaction and the per-chunk gather/scatter
# launches cost about what skipping the masked rows saves.
AUTO_SKIP_MIN_N = 16384


def launches_per_step(N: int, chunk: int, skip_rows: bool = False) -> int:
    """Kernels this library launches for one fused forward+backward call:
    teacher prep, logits/lse GEMM, lse merge, loss, gradient scale, and per
    chunk the dZ recompute GEMM and the joint dH/dW GEMM; when masked rows are
    skipped, also the row compaction and per chunk a row gather and scatter."""
    if N == 0:
        return 0
    c = math.ceil(N / chunk)
    return 6 + 4 * c if skip_rows else 5 + 2 * c


def per_kernel_times(ev, N, d, V, chunk, kept=None):
    """Live per-kernel totals from the events recorded around every launch of
    the fused call: 0 teacher prep, 1 logits/lse GEMM, 2 lse merge, 3 loss,
    4 gradient scale, then per chunk c the dZ recompute (5+2c) and the joint
    dH/dW GEMM (6+2c).  With skipped rows (`kept` = tokens the backward
    processes): 5 row compaction, then per chunk the row gather (6+4c), dZ
    recompute (7+4c), joint dH/dW GEMM (8+4c) and dH row scatter (9+4c); the
    GEMMs' flops count the kept rows of each chunk only."""
    names = {0: ("teacher_prep", 0.0), 1: ("forward_gemm", 2.0 * N * d * V), 2: ("lse_merge", 0.0),
             3: ("loss", 0.0), 4: ("grad_scale", 0.0)}
    if kept is not None:
        names[5] = ("row_compaction", 0.0)
    out = {}
    for row in ev:
        for j in range(len(row) - 1):
            if j in names:
                key, flops = names[j]
            elif kept is None:
                c = (j - 5) // 2
                cc = min(chunk, N - c * chunk)
                key, flops = (("dz_recompute", 2.0 * cc * d * V) if (j - 5) % 2 == 0
                              else ("grads_dH_dW", 4.0 * cc * d * V))
            else:
                c, r = divmod(j - 6, 4)
                cc = max(0, min(chunk, kept - c * chunk))
                key, flops = [("row_gather", 0.0), ("dz_recompute", 2.0 * cc * d * V),
                              ("grads_dH_dW", 4.0 * cc * d * V), ("row_scatter", 0.0)][r]
            k = out.setdefault(key, {"launches": 0, "ms": 0.0, "flops": 0.0})
            k["launches"] += 1
            k["ms"] += row[j].elapsed_time(row[j + 1])
            k["flops"] += flops
    total = sum(k["ms"] for k in out.values())
    for k in out.values():
        k["avg_ms"] = k["ms"] / k["launches"]
        k["share"] = k["ms"] / total if total > 0 else None
        k["tflops"] = k["flops"] / (k["ms"] / 1e3) / 1e12 if k["flops"] > 0 else None
    return out


def blas_threads() -> int:
    try:
        import numpy  # noqa: F401  (load the BLAS so threadpoolctl can see it)
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(x, cfg, n_tokens: int):
    """Time the fp64 oracle (as it stands) on the first n_tokens tokens of the
    workload: forward + backward of those tokens against the full W."""
    import oracle
    sub = {k: (v[:n_tokens] if k != "W" else v) for k, v in x.items()}
    t0 = time.perf_counter()
    oracle.kd_topk_kl(sub["H"], sub["W"], sub["topk_idx"], sub["topk_logit"], sub["mask"], cfg.T)
    return time.perf_counter() - t0


def sample_tokens(cfg, flop_budget: float) -> int:
    return int(max(1, min(cfg.N, round(flop_budget / (8.0 * cfg.d * cfg.V)))))


# ---------------------------------------------------------------- arms

def run_reference(args, cfg, world, rank):
    if rank != 0:
        return 0
    x = workloads.make_inputs(cfg)
    n = sample_tokens(cfg, args.ref_flops)
    for _ in range(args.warmup):
        oracle_sample(x, cfg, n)
    times = [oracle_sample(x, cfg, n) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    cores = blas_threads()
    flops = 8.0 * n * cfg.d * cfg.V * args.steps
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "tflops": flops / total / 1e12,
        "config": config_block(cfg, 1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {n} of {cfg.N} tokens per step (full W, fwd+bwd, fp64)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(cfg, world):
    return {"workload": cfg.name, "N": cfg.N, "d": cfg.d, "V": cfg.V, "K": cfg.K, "T": cfg.T,
            "chunk": cfg.chunk, "seed": cfg.seed, "mask": cfg.mask, "teacher": cfg.teacher,
            "global_batch": cfg.N * world, "seq_len": cfg.N,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (W is %.2f GB > 126 MB L2); no flush" % (2 * cfg.V * cfg.d / 1e9)}


def executed_flops(cfg, n_kept=None) -> float:
    """Tensor-core flops a step runs: the forward GEMM over every token (2NdV)
    and the backward's three (6 n d V) over the tokens it processes (all, or
    the kept ones when masked rows are skipped)."""
    nb = cfg.N if n_kept is None else n_kept
    return 2.0 * cfg.N * cfg.d * cfg.V + 6.0 * nb * cfg.d * cfg.V


def measure_config(kd, cfg, dev, steps: int, warmup: int, backward_rows: str = "auto"):
    """Device-timed fused steps of one workload on its own inputs (made here,
    copied to the device before timing, freed after): ms per step, peak HBM
    GiB of the step over inputs, outputs and workspace, and live per-kernel
    times.  Used for the secondary workloads of the default run."""
    x = workloads.make_inputs(cfg)
    N, d, V, K, T, chunk = cfg.N, cfg.d, cfg.V, cfg.K, cfg.T, cfg.chunk
    n_kept = int(((x["mask"] != 0) & (x["topk_idx"] != -1).any(dim=1)).sum())
    skip = backward_rows == "kept" or (backward_rows == "auto" and n_kept < N and N >= AUTO_SKIP_MIN_N)
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(dev)
    base_mem = torch.cuda.memory_allocated(dev)
    g = {k: v.to(dev) for k, v in x.items()}
    del x
    ws = kd.alloc_workspace(N, d, V, K, chunk, dev)
    dH = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((V, d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nl = kd.forward_backward_launches(N, chunk, skip)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record(stream)

    def step(events=None):
        kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk,
                            workspace=ws, dH=dH, dW=dW, events=events, skip_masked_rows=skip)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    st, _ = kd.check(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up ({cfg.name}): {kd.kd_status_string(st)}")
    peak_gib = (torch.cuda.max_memory_allocated(dev) - base_mem) / 2**30
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(steps):
        step(ev[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end) / steps
    kern = per_kernel_times(ev, N, d, V, chunk, n_kept if skip else None)
    del g, ws, dH, dW
    torch.cuda.empty_cache()
    return {"ms": ms, "peak_gib": peak_gib, "kern": kern, "n_kept": n_kept if skip else None}


def secondary_block(kd, dev, args, peaks):
    """The other workloads on which the target is stated, measured in the
    same run: the Llama-shaped 8K head (V = 128,256) and every point of the
    long-context sweep (d = 2048, V = 128,256, 4K to 256K tokens) with its
    peak HBM and a least-squares line through peak GiB against N."""
    out = {}
    peak, peak_sus = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]

    def entry(cfg, r):
        tf = 8.0 * cfg.N * cfg.d * cfg.V / (r["ms"] / 1e3) / 1e12
        tfx = executed_flops(cfg, r["n_kept"]) / (r["ms"] / 1e3) / 1e12
        dom = max((v for v in r["kern"].values() if v["flops"] > 0), key=lambda v: v["ms"])
        return {"N": cfg.N, "d": cfg.d, "V": cfg.V, "chunk": cfg.chunk, "ms_per_step": r["ms"],
                "tokens_per_s": cfg.N / (r["ms"] / 1e3), "tflops": tf, "tflops_executed": tfx,
                "pct_bf16_peak": tf / peak, "pct_bf16_peak_sustained": tf / peak_sus,
                "peak_hbm_gib": r["peak_gib"],
                "kernel_tflops": {k: v["tflops"] for k, v in r["kern"].items() if v["tflops"]},
                "dominant_kernel_frac_sustained": dom["tflops"] / peak_sus}

    cfg2 = workloads.get_config(2)
    out[cfg2.name] = entry(cfg2, measure_config(kd, cfg2, dev, args.secondary_steps, 3))
    sweep = []
    cfg4 = workloads.get_config(4)
    for n in cfg4.sweep:
        c = workloads.get_config(4, n)
        sweep.append(entry(c, measure_config(kd, c, dev, args.secondary_steps, 3)))
    out[cfg4.name] = {"points": sweep,
                      "peak_gib_fit": line_fit([e["N"] for e in sweep], [e["peak_hbm_gib"] for e in sweep])}
    return out


def line_fit(ns, gib):
    """Least-squares line through peak GiB against tokens: its slope in bytes
    per token, its intercept in GiB and the largest relative residual."""
    mn, mg = sum(ns) / len(ns), sum(gib) / len(gib)
    slope = sum((a - mn) * (b - mg) for a, b in zip(ns, gib)) / sum((a - mn) ** 2 for a in ns)
    icpt = mg - slope * mn
    resid = max(abs(b - (icpt + slope * a)) / b for a, b in zip(ns, gib))
    return {"slope_bytes_per_token": slope * 2**30, "intercept_gib": icpt, "max_rel_residual": resid}


def run_cuda(args, cfg, world, rank, local):
    import chunked_top_kl_b200 as kd

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rcfg = cfg if rank == 0 else cfg.__class__(**{**cfg.__dict__, "seed": cfg.seed + 1000 * rank})
    x = workloads.make_inputs(rcfg)
    N, d, V, K, T, chunk = cfg.N, cfg.d, cfg.V, cfg.K, cfg.T, cfg.chunk

    torch.cuda.reset_peak_memory_stats(dev)
    base_mem = torch.cuda.memory_allocated(dev)
    g = {k: v.to(dev) for k, v in x.items()}
    ws = kd.alloc_workspace(N, d, V, K, chunk, dev)
    dH = torch.empty((N, d), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((V, d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    n_kept = int(((x["mask"] != 0) & (x["topk_idx"] != -1).any(dim=1)).sum())
    skip = args.backward_rows == "kept" or (args.backward_rows == "auto" and n_kept < N and N >= AUTO_SKIP_MIN_N)
    kept = n_kept if skip else None

    def step():
        loss, _, _, _ = kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T,
                                            chunk, workspace=ws, dH=dH, dW=dW, skip_masked_rows=skip)
        return loss

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, nbad = kd.check(ws)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {kd.kd_status_string(st)}")
    peak_gib = (torch.cuda.max_memory_allocated(dev) - base_mem) / 2**30
    ws_gib = ws.numel() / 2**30

    # ---- kernel-only timed region (inputs resident in HBM).  Each step is one
    # fused forward+backward call that records an event before each of its
    # kernel launches and after the last (same kernels and work as without
    # events), which gives live per-kernel durations on the launching stream.
    nl = kd.forward_backward_launches(N, chunk, skip)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(args.steps)]
    for row in ev:
        for e in row:
            e.record(stream)                 # creates the CUDA event behind each object
    sampler = ClockSampler(local) if not args.no_clocks else None
    barrier(world)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        kd.forward_backward(g["H"], g["W"], g["topk_idx"], g["topk_logit"], g["mask"], T, chunk,
                            workspace=ws, dH=dH, dW=dW, events=ev[i], skip_masked_rows=skip)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms_local = start.elapsed_time(end)
    kern = per_kernel_times(ev, N, d, V, chunk, kept)
    ms = reduce_max(ms_local, world, dev)
    st, _ = kd.check(ws)
    if st != 0:
        raise RuntimeError(f"device status after timing: {kd.kd_status_string(st)}")

    # ---- end to end through the public API with host buffers.  Every step copies
    # its inputs from pinned host memory and reads its loss back.  Serial: copy,
    # compute, read back, in one stream.  Pipelined (the reported value): two
    # device input sets; the copies of step k + 1 run on a second stream while
    # step k computes, as a data loader would feed them.  Both timed regions
    # start before the first copy and end after the last loss read.
    e2e = None
    if not args.no_e2e:
        host = {k: v.pin_memory() for k, v in x.items()}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        loss_host = torch.empty((), dtype=torch.float32).pin_memory()
        g2 = {k: torch.empty_like(v) for k, v in g.items()}
        copy_stream = torch.cuda.Stream(dev)

        def step_on(buf):
            loss, _, _, _ = kd.forward_backward(buf["H"], buf["W"], buf["topk_idx"], buf["topk_logit"], buf["mask"],
                                                T, chunk, workspace=ws, dH=dH, dW=dW, skip_masked_rows=skip)
            return loss

        def serial(n):
            for _ in range(n):
                for k in g:
                    g[k].copy_(host[k], non_blocking=True)
                loss_host.copy_(step_on(g), non_blocking=True)

        def pipelined(n):
            bufs = (g, g2)
            copied = [torch.cuda.Event(), torch.cuda.Event()]
            freed = [torch.cuda.Event(), torch.cuda.Event()]
            copy_stream.wait_stream(stream)

            def load(i):
                b = i % 2
                with torch.cuda.stream(copy_stream):
                    if i >= 2:
                        copy_stream.wait_event(freed[b])          # step i - 2 has used this set
                    for k in bufs[b]:
                        bufs[b][k].copy_(host[k], non_blocking=True)
                    copied[b].record(copy_stream)

            load(0)
            for i in range(n):
                if i + 1 < n:
                    load(i + 1)
                stream.wait_event(copied[i % 2])
                loss = step_on(bufs[i % 2])
                freed[i % 2].record(stream)
                loss_host.copy_(loss, non_blocking=True)

        def timed(fn):
            fn(max(1, args.warmup))
            barrier(world)
            torch.cuda.synchronize(dev)
            s2 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            s2.record(stream)
            fn(args.steps)
            e2.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            return reduce_max(s2.elapsed_time(e2), world, dev)

        serial_ms = timed(serial)
        e2e_ms = timed(pipelined)
        e2e = {"value": N * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(loss_host.element_size()),
               "ms_per_step": e2e_ms / args.steps,
               "copies": ("every input (H, W, teacher cache, mask) copied in from pinned host memory each "
                          "step, step k+1's on a second stream during step k (two device input sets); "
                          "only the loss is read back: dH and dW stay on the device for the optimizer, "
                          "as in a training step"),
               "serial_ms_per_step": serial_ms / args.steps}
        del g2

    if rank != 0:
        return 0

    peaks, peaks_src = load_peaks()
    secondary = None
    if world == 1 and not args.no_secondary:
        del g, ws, dH, dW
        torch.cuda.empty_cache()
        secondary = secondary_block(kd, dev, args, peaks)
    ms_step = ms / args.steps
    flops_step = 8.0 * N * d * V
    tflops = flops_step * world / (ms_step / 1e3) / 1e12
    tflops_exec = executed_flops(cfg, kept) * world / (ms_step / 1e3) / 1e12
    # Roofline of the dominant kernel (largest share of the step's kernel time).
    dom_name, dom = max(((k, v) for k, v in kern.items() if v["flops"] > 0), key=lambda kv: kv[1]["ms"])
    dom_ach = dom["tflops"]
    fwd_avg = sum(kern[k]["ms"] for k in ("teacher_prep", "forward_gemm", "lse_merge", "loss")) / args.steps
    bwd_avg = sum(v["ms"] for k, v in kern.items()
                  if k not in ("teacher_prep", "forward_gemm", "lse_merge", "loss")) / args.steps
    peak_sus = peaks["bf16_tflops_sustained"]
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n = sample_tokens(cfg, args.cpu_flops)
        t = oracle_sample(x, cfg, n)
        cpu = {"value": n / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {n} of {N} tokens (full W), fwd+bwd in fp64, one run of {t:.1f} s"}
    line = {
        "metric": METRIC, "value": N * world * args.steps / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; H~N(0,1), W~N(0,0.02^2) bf16, Zipf-shaped top-K teacher cache)",
        "tflops": tflops,
        "pct_bf16_peak": tflops / world / peaks["bf16_tflops"],
        "pct_bf16_peak_sustained": tflops / world / peak_sus,
        "tflops_executed": tflops_exec,
        "pct_bf16_peak_executed": tflops_exec / world / peaks["bf16_tflops"],
        "flops_note": ("tflops counts 8 N d V per step (the metric's count); tflops_executed counts the "
                       "tensor-core work the step runs (2 N d V forward + 6 n d V backward over the "
                       "n tokens it processes)"),
        "peak_hbm_gib": peak_gib, "workspace_gib": ws_gib,
        "fwd_ms": fwd_avg, "bwd_ms": bwd_avg,
        "config": {**config_block(cfg, world), "backward_rows": "kept tokens only" if skip else "all tokens"},
        "clocks": clocks,
        "gpu_launches": launches_per_step(N, chunk, skip) * args.steps,
        "roofline": {"bound": "tensor", "kernel": dom_name,
                     "achieved": dom_ach, "peak": peak_sus, "unit": "TFLOP/s", "frac": dom_ach / peak_sus,
                     "peak_kind": f"bf16_tflops_sustained ({peaks_src})",
                     "frac_of_burst": dom_ach / peaks["bf16_tflops"],
                     "flops_per_launch": dom["flops"] / dom["launches"],
                     "avg_launch_ms": dom["avg_ms"], "share": dom["share"],
                     "traffic": committed_traffic(cfg.name, dom_name)},
        "kernels": {k: {kk: v[kk] for kk in ("launches", "avg_ms", "share", "tflops")} for k, v in kern.items()},
        "roofline_step": {"bound": "tensor", "achieved": tflops / world, "peak": peak_sus,
                          "unit": "TFLOP/s", "frac": tflops / world / peak_sus,
                          "flops_per_step": flops_step},
        "e2e": e2e,
        "cpu_baseline": cpu,
        "secondary": secondary,
    }
    print(json.dumps(line), flush=True)
    return 0


TOPK_METRIC = "teacher top-K cache write tokens/s (logits GEMM + exact top-K select)"


def topk_launches_per_call(N: int, chunk: int) -> int:
    """Kernel launches of one kd_teacher_topk call: per chunk, the logits GEMM and the select."""
    return 0 if N == 0 else 2 * ((N + chunk - 1) // chunk)


def run_teacher_topk(args, cfg, world, rank, local):
    """The offline cache writer: a teacher head [V, d] over N hidden states,
    top-K (index, logit) per token.  One step = one kd_teacher_topk call over
    the whole batch; the workload's H and W stand in for the teacher's."""
    import chunked_top_kl_b200 as kd

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rcfg = cfg if rank == 0 else cfg.__class__(**{**cfg.__dict__, "seed": cfg.seed + 1000 * rank})
    x = workloads.make_inputs(rcfg)
    N, d, V, K, chunk = cfg.N, cfg.d, cfg.V, cfg.K, args.topk_chunk
    Ht, Wt = x["H"].to(dev), x["W"].to(dev)
    n_ws = kd.kd_teacher_topk_workspace_size(N, d, V, K, chunk)
    ws = torch.empty(n_ws, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        kd.teacher_topk(Ht, Wt, K, chunk=chunk, workspace=ws)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local) if not args.no_clocks else None
    barrier(world)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.start()
        time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        idx, val = kd.teacher_topk(Ht, Wt, K, chunk=chunk, workspace=ws)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    ms = reduce_max(start.elapsed_time(end), world, dev)

    # End to end through the public API with host buffers: every call copies Ht
    # and Wt in from pinned host memory and reads the cache back.  Serial: copy,
    # compute, read back, in one stream.  Pipelined (the reported value): two
    # device input sets, the copies of call k + 1 on a second stream while call
    # k computes.
    e2e = None
    if not args.no_e2e:
        host = {"H": x["H"].pin_memory(), "W": x["W"].pin_memory()}
        oi = torch.empty((N, K), dtype=torch.int32).pin_memory()
        ov = torch.empty((N, K), dtype=torch.float32).pin_memory()
        bufs = ({"H": Ht, "W": Wt}, {"H": torch.empty_like(Ht), "W": torch.empty_like(Wt)})
        copy_stream = torch.cuda.Stream(dev)

        def call_on(buf):
            i, v = kd.teacher_topk(buf["H"], buf["W"], K, chunk=chunk, workspace=ws)
            oi.copy_(i, non_blocking=True)
            ov.copy_(v, non_blocking=True)

        def serial(n):
            for _ in range(n):
                for k in bufs[0]:
                    bufs[0][k].copy_(host[k], non_blocking=True)
                call_on(bufs[0])

        def pipelined(n):
            copied = [torch.cuda.Event(), torch.cuda.Event()]
            freed = [torch.cuda.Event(), torch.cuda.Event()]
            copy_stream.wait_stream(stream)

            def load(i):
                b = i % 2
                with torch.cuda.stream(copy_stream):
                    if i >= 2:
                        copy_stream.wait_event(freed[b])          # call i - 2 has used this set
                    for k in bufs[b]:
                        bufs[b][k].copy_(host[k], non_blocking=True)
                    copied[b].record(copy_stream)

            load(0)
            for i in range(n):
                if i + 1 < n:
                    load(i + 1)
                stream.wait_event(copied[i % 2])
                call_on(bufs[i % 2])
                freed[i % 2].record(stream)

        def timed(fn):
            fn(max(1, args.warmup))
            barrier(world)
            torch.cuda.synchronize(dev)
            s2 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            s2.record(stream)
            fn(args.steps)
            e2.record(stream)
            torch.cuda.synchronize(dev)
            barrier(world)
            return reduce_max(s2.elapsed_time(e2), world, dev)

        serial_ms = timed(serial)
        e2e_ms = timed(pipelined)
        e2e = {"value": N * world * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(sum(v.numel() * v.element_size() for v in host.values())),
               "d2h_bytes_per_step": int(oi.numel() * 4 + ov.numel() * 4), "ms_per_step": e2e_ms / args.steps,
               "serial_ms_per_step": serial_ms / args.steps,
               "copies": "Ht and Wt copied in from pinned host memory every call, call k+1's on a second stream "
                         "during call k (two device input sets); the cache (indices and logits) read back"}
    if rank != 0:
        return 0

    peaks, peaks_src = load_peaks()
    ms_step = ms / args.steps
    gemm_tflops = 2.0 * N * d * V / (ms_step / 1e3) / 1e12
    peak_sus = peaks["bf16_tflops_sustained"]
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        n = int(max(1, min(N, args.topk_cpu_rows)))
        t0 = time.perf_counter()
        oracle.teacher_topk(x["H"][:n], x["W"], K)
        t = time.perf_counter() - t0
        cpu = {"value": n / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"first {n} of {N} tokens (full teacher head), fp64 logits + stable sort, {t:.1f} s"}
    line = {
        "metric": TOPK_METRIC, "value": N * world * args.steps / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 -> f32",
        "data": "synthetic (seeded; Ht~N(0,1), Wt~N(0,0.02^2) bf16)",
        "config": {"workload": f"teacher_topk_{cfg.name}", "N": N, "d": d, "V": V, "K": K, "chunk": chunk,
                   "seed": cfg.seed, "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (Wt > 126 MB); no flush"},
        "clocks": clocks,
        "gpu_launches": topk_launches_per_call(N, chunk) * args.steps,
        "roofline": {"bound": "tensor", "kernel": "whole call (logits GEMM + select)",
                     "achieved": gemm_tflops, "peak": peak_sus, "unit": "TFLOP/s", "frac": gemm_tflops / peak_sus,
                     "peak_kind": f"bf16_tflops_sustained ({peaks_src})",
                     "flops_per_call": 2.0 * N * d * V, "traffic": None},
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG)
    ap.add_argument("--N", type=int, default=None, help="override the token count (config 4 sweep)")
    ap.add_argument("--V", type=int, default=None, help="override the vocabulary (a smaller case to profile)")
    ap.add_argument("--d", type=int, default=None, help="override the hidden size (a smaller case to profile)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the Llama-shaped head and the long-context sweep measured after the main workload")
    ap.add_argument("--secondary-steps", type=int, default=5, help="timed steps per secondary workload")
    ap.add_argument("--backward-rows", choices=["auto", "all", "kept"], default="auto",
                    help="backward over every token, or over the tokens with a non-zero dZ row only "
                         "(same results; auto: kept when some token is masked and N >= %d)" % AUTO_SKIP_MIN_N)
    ap.add_argument("--cpu-flops", type=float, default=4e12, help="oracle work for cpu_baseline")
    ap.add_argument("--ref-flops", type=float, default=1.2e12, help="oracle work per reference step")
    ap.add_argument("--op", choices=["loss", "teacher-topk"], default="loss",
                    help="loss: the fused loss step (default); teacher-topk: the offline cache writer")
    ap.add_argument("--topk-chunk", type=int, default=4096, help="tokens per chunk of the cache writer")
    ap.add_argument("--topk-cpu-rows", type=int, default=256, help="oracle tokens for its cpu_baseline")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.op == "teacher-topk" and args.impl == "reference":
        ap.error("--op teacher-topk times the library; its oracle is timed in cpu_baseline")
    cfg = workloads.get_config(args.config, args.N)
    if args.V is not None or args.d is not None:
        import dataclasses
        V = args.V if args.V is not None else cfg.V
        d = args.d if args.d is not None else cfg.d
        cfg = dataclasses.replace(cfg, V=V, d=d, name=f"{cfg.name}_at_N{cfg.N}_d{d}_V{V}")
    world, rank, local = dist_setup(args.impl)
    if world != args.gpus and args.impl == "cuda":
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    try:
        if args.impl == "reference":
            return run_reference(args, cfg, world, rank)
        if args.op == "teacher-topk":
            return run_teacher_topk(args, cfg, world, rank, local)
        return run_cuda(args, cfg, world, rank, local)
    finally:
        if world > 1 and args.impl == "cuda":
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
