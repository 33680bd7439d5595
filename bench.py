"""Benchmark of the block-quantized-weight GEMM hot path on B200.

Default workload (one "step"): the Q8_0 27B FFN at decode width B = 64 -- qgemm_run on the
gate [17408, 5120], up [17408, 5120] and down [5120, 17408] matrices, fp32 outputs.  Steps
are timed as replays of a CUDA graph holding the three calls.  The
metric is weight GB/s: packed weight bytes read per step / step time (the pages' weight-
streaming bound for widths <= 64).  Weights cycle through a ring of distinct copies so that
no step finds its weights in L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent replica of the
same workload ("replicas only": the path has no exchange step); value = all ranks' bytes /
max-over-ranks device time.  --impl reference times the CPU oracle on a bounded sample of
the same workload (rank 0 only).  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HIDDEN, INTER = 5120, 17408
FMT = "q8_0"
BATCH = 64
RING = 4  # copies of each matrix: 3 x 4 x 94.7 MB = 1.14 GB of Q8_0 weights > L2
METRIC = "qGEMM weight GB/s (B≤64) & TFLOP/s (prefill) as % of B200 roofline"
WORKLOAD = "Q8_0 27B FFN decode step: gate+up W[17408,5120] and down W[5120,17408], B=64"
KERNEL = "qgemm_pair_kernel<Q8_0, f16 operands> (CTA pairs, tcgen05.mma.cta_group::2)"
SM_MAX_FALLBACK = 1965.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--batch", type=int, default=BATCH)
    ap.add_argument("--fmt", default=FMT)
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def matrices():
    # (name, N, K, weight seed, activation width K, activation seed)
    return [("gate", INTER, HIDDEN, 0), ("up", INTER, HIDDEN, 2), ("down", HIDDEN, INTER, 3)]


def weight_bytes(fmt, N, K):
    if fmt == "q8_0":
        return N * K + N * (K // 32) * 2
    if fmt == "nvfp4":
        return N * K // 2 + N * (K // 16)
    return N * K // 2 + N * (K // 32)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() in ("active", "1", "yes"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_sample(fmt, batch, target_s=12.0):
    """Times the oracle (dequantise + fp64 GEMM) on the first rows of each matrix of the step,
    sized to roughly `target_s` seconds.  Returns (GB/s of weight bytes, description, threads)."""
    import numpy as np
    import oracle
    from block_quantized_weight_qgemm_b200 import inputs
    threads = oracle.default_threads()

    def run(rows):
        t_total, nbytes = 0.0, 0
        for name, N, K, seed in matrices():
            W = inputs.weights(rows, K, seed=seed).numpy()
            codes, scales, ts = oracle.pack(fmt, W)
            x = inputs.bf16_bits(inputs.activations(batch, K, seed=1))
            t0 = time.perf_counter()
            Wd = oracle.dequant(fmt, codes, scales, ts, rows, K)
            oracle.gemm(x, Wd, nthreads=threads)
            t_total += time.perf_counter() - t0
            nbytes += weight_bytes(fmt, rows, K)
        return t_total, nbytes

    t, nb = run(64)
    rows = int(max(64, min(HIDDEN, 64 * target_s / max(t, 1e-3))))
    rows = (rows // 32) * 32
    t, nb = run(rows)
    desc = "first %d rows of each of gate/up/down (%.1f MB of packed weights), B=%d, dequant+fp64 GEMM" % (
        rows, nb / 1e6, batch)
    return nb / t / 1e9, desc, threads, t


def run_reference(args, rank, world):
    if rank != 0:
        return
    gbs, desc, threads, t = cpu_oracle_sample(args.fmt, args.batch, target_s=6.0)
    steps_t = []
    # each step: one bounded sample of the workload through the oracle (as it stands)
    for _ in range(args.warmup):
        pass
    per_step_s = t
    value = gbs
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step_s * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "fmt": args.fmt, "B": args.batch,
                   "sample": desc},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(v: float, device, world: int) -> float:
    """The largest value of v over all ranks (every rank calls this, in the same order)."""
    if world <= 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(bytes_per_rank_step: float, ms_max: float, world: int) -> float:
    """Whole-job GB/s: every rank processes bytes_per_rank_step per step; the job's step time
    is the slowest rank's."""
    return world * bytes_per_rank_step / (ms_max * 1e-3) / 1e9


def launches_per_call(fmt, N, K, B):
    """Kernels one qgemm_run launches: the x conversion (widths <= 256), the GEMM, and the
    split-K reduction when the K split is above 1."""
    from block_quantized_weight_qgemm_b200 import qgemm
    if B > 256:
        return 1
    return 2 + (1 if qgemm.split_k(fmt, N, K) > 1 else 0)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    if world > 1:
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=timedelta(seconds=120))
    if args.impl == "reference":
        run_reference(args, rank, world)
        if world > 1:
            dist.destroy_process_group()
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from block_quantized_weight_qgemm_b200 import inputs, qgemm
    qgemm.lib()

    fmt, B = args.fmt, args.batch
    # weight rings, activations, outputs, workspaces
    calls = []
    for name, N, K, seed in matrices():
        ring = []
        for i in range(RING):
            W = inputs.weights(N, K, seed=seed + 1000 * i).to(dev)
            ring.append(qgemm.pack(fmt, W))
            del W
        x = inputs.activations(B, K, seed=1 if name != "down" else 4).to(dev)
        y = torch.empty(B, N, device=dev)
        ws = torch.empty(max(qgemm.workspace_size(fmt, N, K, B), 16), dtype=torch.uint8, device=dev)
        calls.append(dict(name=name, N=N, K=K, ring=ring, x=x, y=y, ws=ws))
    torch.cuda.synchronize()
    step_bytes = sum(weight_bytes(fmt, c["N"], c["K"]) for c in calls)

    def step(i, events=None, stream=None):
        for j, c in enumerate(calls):
            if events is not None:
                qgemm.profile_events(*events[j])
            qgemm.run(c["x"], c["ring"][i % RING], y=c["y"], workspace=c["ws"], stream=stream)
        if events is not None:
            qgemm.profile_events(None, None)

    # one CUDA graph per weight copy of the ring: a step is the replay of graph[i % RING]
    gstream = torch.cuda.Stream(device=dev)
    graphs = []
    with torch.cuda.stream(gstream):
        for r in range(RING):
            step(r, stream=gstream)
        torch.cuda.synchronize()
        for r in range(RING):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=gstream):
                step(r, stream=gstream)
            graphs.append(g)
    torch.cuda.synchronize()

    for i in range(args.warmup):
        graphs[i % RING].replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # ---- device-timed region: K graph replays between CUDA events -----------------------
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(args.steps):
        graphs[i % RING].replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / args.steps

    # ---- the dominant kernel alone: events around each GEMM launch (stream launches) ----
    kev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in calls] for _ in range(args.steps)]
    for pairs in kev:  # torch creates the CUDA events lazily, on first record
        for a, b in pairs:
            a.record()
            b.record()
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(i, kev[i])
    torch.cuda.synchronize()
    kernel_ms = [[a.elapsed_time(b) for (a, b) in kev[i]] for i in range(args.steps)]
    per_launch = []
    for i in range(args.steps):
        for j, c in enumerate(calls):
            per_launch.append((weight_bytes(fmt, c["N"], c["K"]), kernel_ms[i][j]))
    k_bytes = sum(b for b, _ in per_launch) / len(per_launch)
    k_ms = sum(t for _, t in per_launch) / len(per_launch)

    ms_max = max_over_ranks(ms, dev, world)
    value = job_rate(step_bytes, ms_max, world)

    # ---- end-to-end through the public API with host buffers ---------------------------
    hx = [c["x"].cpu().pin_memory() for c in calls]
    hy = [torch.empty(c["y"].shape, dtype=c["y"].dtype).pin_memory() for c in calls]
    dx = [torch.empty_like(c["x"]) for c in calls]
    h2d = sum(t.numel() * t.element_size() for t in hx)
    d2h = sum(t.numel() * t.element_size() for t in hy)
    stream = torch.cuda.current_stream()

    def e2e_step(i):
        for j, c in enumerate(calls):
            dx[j].copy_(hx[j], non_blocking=True)
            qgemm.run(dx[j], c["ring"][i % RING], y=c["y"], workspace=c["ws"])
            hy[j].copy_(c["y"], non_blocking=True)
        stream.synchronize()

    for i in range(max(2, args.warmup)):
        e2e_step(i)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev, world)
    e2e_value = job_rate(step_bytes, e_ms, world)

    status = qgemm.device_status(reset=True)

    cpu = None
    if rank == 0 and world == 1:
        gbs, desc, threads, _ = cpu_oracle_sample(fmt, B)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": desc}

    peak, peak_kind = peaks()
    achieved = k_bytes / (k_ms * 1e-3) / 1e9
    traffic = _traffic_from_profiles()
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded N(0,0.02) weights, N(0,1) bf16 activations)",
        "config": {"workload": WORKLOAD, "fmt": fmt, "B": B, "accumulate": "f32",
                   "weight_bytes_per_step": step_bytes,
                   "l2": "weights cycle through %d distinct copies per matrix (%.2f GB) > 126 MB L2"
                         % (RING, RING * step_bytes / 1e9),
                   "timing": "step = CUDA-graph replay of the three qgemm_run calls; the kernel "
                             "figure times each GEMM launch between events on its stream",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": KERNEL, "peak_source": peak_kind,
                     "bytes_per_launch": int(k_bytes), "avg_launch_us": round(k_ms * 1e3, 3)},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": sum(launches_per_call(fmt, c["N"], c["K"], B) for c in calls) * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _traffic_from_profiles():
    """DRAM bytes per launch of the timed kernel from the committed ncu summary, if it was
    taken on the current kernel source (else null)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        h = hashlib.sha256()
        for name in sorted(os.listdir(os.path.join(ROOT, "block_quantized_weight_qgemm_b200", "csrc"))):
            with open(os.path.join(ROOT, "block_quantized_weight_qgemm_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if d.get("csrc_sha256") != h.hexdigest():
            return None
        return d.get("dram_bytes_per_launch_scaled")
    except Exception:
        return None


if __name__ == "__main__":
    main()
