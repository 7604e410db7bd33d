#!/usr/bin/env python
"""Benchmark of the fine-grained-scaled FP8 GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one call of the GEMM over one batch of seeded synthetic input (all
of the path: TMA tile loads, FP8 MMA per K-block, FP32 promotion, tile
scheduling, bf16 epilogue).  The default workload is the dense decode shape
M=64, N=2112, K=7168.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
device synchronise on both sides, timed with CUDA events on the launching
stream; the K launches are replayed from one CUDA graph so host launch cost
is not on the device timeline.  When one input set is smaller than twice the
L2 cache, the steps rotate through enough copies of the inputs (in distinct
device buffers) that every step reads HBM.  N > 1 (torchrun): every rank runs
an independent problem of the same shape (weak scaling, no collective on the
data path); the device time is the max over ranks.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle (test
infrastructure) on a bounded row sample of the same workload instead.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_block_scaled_x128_b200 import synth  # noqa: E402

METRIC = "FP8 TFLOPS (bf16 out) and % of B200 FP8/HBM roofline per shape, 1 GPU"
UNIT = "TFLOPS"
DEFAULT_WORKLOAD = "dense_64x2112x7168"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS = 6650.0, 1590.0
FP8_OVER_BF16 = 2.0  # nominal dense FP8 : BF16 tensor throughput (4.5 : 2.25 PFLOP/s)


# --------------------------------------------------------------------------- workload accounting

def workload_inputs(name: str, seed: int):
    return synth.config_inputs(name, seed)


def accounting(d) -> dict:
    """Algorithmic FLOPs and bytes of one step: valid rows only, each input byte
    once, D written once."""
    K = d["K"]
    KB = K // 128
    N = d["N"]
    NB = (N + 127) // 128
    if d["kind"] == "dense":
        M = d["M"]
        rows, b_bytes, sb_bytes = M, N * K, NB * KB * 4
    elif d["kind"] == "contiguous":
        rows = int(np.sum(d["m_indices"] >= 0)) * 128
        used = np.unique(d["m_indices"][d["m_indices"] >= 0])
        b_bytes, sb_bytes = len(used) * N * K, len(used) * NB * KB * 4
    else:
        mm = np.minimum(d["masked_m"], d["Mmax"])
        rows = int(mm.sum())
        active = int(np.sum(mm > 0))
        b_bytes, sb_bytes = active * N * K, active * NB * KB * 4
    flops = 2.0 * rows * N * K
    nbytes = rows * K + rows * KB * 4 + b_bytes + sb_bytes + rows * N * 2
    return dict(flops=flops, bytes=float(nbytes), rows=rows)


def input_bytes(d) -> int:
    return int(d["A"].nbytes + d["sa"].nbytes + d["B"].nbytes + d["sb"].nbytes)


# --------------------------------------------------------------------------- peaks, traffic, clocks

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=1400.0, source="fallback")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "fp8_block_scaled_x128_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values (every rank gets it): a multi-GPU time
    is the slowest replica's, never the wall clock of one of them."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_step: float, steps: int, ms: float) -> float:
    """Aggregate throughput of `world` replicas that each ran `steps` steps in
    at most `ms` milliseconds."""
    return world * flops_per_step * steps / (ms * 1e-3) / 1e12


def kernels_per_call(variant: str) -> int:
    """Kernels one C-ABI call launches: the two-kernel split-K variants run a
    partial-sums kernel and a reduce kernel, all others one kernel."""
    return 2 if "gsplit_2k" in variant else 1


def ncu_traffic(workload: str, variant: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{variant}__{workload}.txt")
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("kernel_source_hash") != kernel_source_hash():
            return None
        return float(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms, stamped on arrival."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    @classmethod
    def disabled(cls):
        obj = cls.__new__(cls)
        obj.samples, obj.proc = [], None
        return obj

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]), parts[3:7]))
            except ValueError:
                pass

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        win = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples[-3:]
        if not win:
            return None
        reasons = sorted({self.REASONS[i] for s in win for i, v in enumerate(s[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(s[1] for s in win), "sm_max_mhz": max(s[2] for s in win),
                "reasons": reasons, "samples": len(win)}


def clocks_rejected(c) -> bool:
    if not c:
        return False
    if set(c["reasons"]) & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    return c["sm_mhz"] < 0.6 * c["sm_max_mhz"] and not c["reasons"]


# --------------------------------------------------------------------------- CPU oracle (test infrastructure)

def oracle_rows_per_second(d, rows: int, nthreads: int):
    import oracle
    rng = np.random.default_rng(0)
    if d["kind"] == "dense":
        pick = np.sort(rng.choice(d["M"], min(rows, d["M"]), replace=False)).astype(np.int32)
        t = time.perf_counter()
        oracle.gemm_nt(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["M"], d["N"], d["K"], rows=pick,
                       nthreads=nthreads)
    elif d["kind"] == "contiguous":
        live = np.nonzero(np.repeat(d["m_indices"] >= 0, 128))[0]
        pick = np.sort(rng.choice(live, min(rows, len(live)), replace=False)).astype(np.int32)
        t = time.perf_counter()
        oracle.m_grouped_contiguous(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], d["m_indices"], d["M"], d["N"],
                                    d["K"], d["G"], rows=pick, nthreads=nthreads)
    else:
        # a masked sample: the same groups with their counts capped so that
        # about `rows` rows are computed in total
        mm = np.minimum(d["masked_m"], d["Mmax"])
        cap = max(1, math.ceil(rows / max(1, int(np.sum(mm > 0)))))
        sub = np.minimum(mm, cap).astype(np.int32)
        pick = np.arange(int(sub.sum()))
        t = time.perf_counter()
        oracle.m_grouped_masked(d["A"], d["sa"], d["ld_sa"], d["B"], d["sb"], sub, d["G"], d["Mmax"], d["N"],
                                d["K"], nthreads=nthreads)
    dt = time.perf_counter() - t
    return len(pick), dt


def cpu_baseline(d, target_s: float = 12.0):
    """Time the oracle as it stands on a bounded row sample; scale to TFLOPS."""
    import oracle
    nthreads = oracle.default_threads()
    acc = accounting(d)
    flop_per_row = acc["flops"] / max(1, acc["rows"])
    n, dt = oracle_rows_per_second(d, nthreads, nthreads)  # one row per thread
    rows = int(min(acc["rows"], max(n, n * target_s / max(dt, 1e-6))))
    n, dt = oracle_rows_per_second(d, rows, nthreads)
    return {"value": n * flop_per_row / dt / 1e12, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": f"{n} of {acc['rows']} output rows of {d['name']}, all N columns, {dt:.2f} s"}


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    import oracle
    d = workload_inputs(args.workload, 0)
    d["name"] = args.workload
    acc = accounting(d)
    flop_per_row = acc["flops"] / max(1, acc["rows"])
    nthreads = oracle.default_threads()
    n1, dt1 = oracle_rows_per_second(d, nthreads, nthreads)  # one row per thread
    per_step_rows = max(1, int(min(acc["rows"], n1 * 1.5 / max(dt1, 1e-6))))  # ~1.5 s per step
    for _ in range(args.warmup):
        oracle_rows_per_second(d, per_step_rows, nthreads)
    total_rows, total_t = 0, 0.0
    for _ in range(args.steps):
        n, dt = oracle_rows_per_second(d, per_step_rows, nthreads)
        total_rows += n
        total_t += dt
    value = total_rows * flop_per_row / total_t / 1e12
    sample = (f"{per_step_rows} of {acc['rows']} output rows of {args.workload} per step "
              f"(all N columns), {args.steps} steps")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": {"workload": args.workload},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------------------- GPU arm

def run_ours(args, rank: int, world: int) -> None:
    import torch
    import torch.distributed as dist

    from fp8_block_scaled_x128_b200 import gemm

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    d = workload_inputs(args.workload, rank)
    d["name"] = args.workload
    acc = accounting(d)
    kind = d["kind"]
    if args.variant is not None:
        gemm.set_variant_override(args.variant)

    # device inputs, rotated through enough copies that each step reads HBM
    per_copy = input_bytes(d)
    copies = 1 if per_copy >= 2 * L2_BYTES else int(math.ceil(2 * L2_BYTES / per_copy))
    host = {k: torch.from_numpy(np.ascontiguousarray(d[k])) for k in ("A", "sa", "B", "sb")}
    if kind == "contiguous":
        host["idx"] = torch.from_numpy(d["m_indices"])
    elif kind == "masked":
        host["idx"] = torch.from_numpy(d["masked_m"])
    sets = [{k: v.to(dev) for k, v in host.items()} for _ in range(copies)]
    if kind == "dense":
        out_shape = (d["M"], d["N"])
    elif kind == "contiguous":
        out_shape = (d["M"], d["N"])
    else:
        out_shape = (d["G"], d["Mmax"], d["N"])
    D = torch.empty(out_shape, dtype=torch.bfloat16, device=dev)

    def step(i: int, s=None):
        t = sets[i % copies]
        if kind == "dense":
            gemm.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"], D=D, stream=s)
        elif kind == "contiguous":
            gemm.m_grouped_fp8_gemm_nt_contiguous(t["A"], t["sa"], t["B"], t["sb"], t["idx"], D=D, stream=s)
        else:
            gemm.m_grouped_fp8_gemm_nt_masked(t["A"], t["sa"], t["B"], t["sb"], t["idx"], d["expected_m"], D=D,
                                              stream=s)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        step(0, stream)  # per-device set-up outside capture
    torch.cuda.synchronize(dev)
    variant = gemm.variant_names()[gemm.last_variant()]

    def capture(nsteps: int, first: int, events: bool):
        g = torch.cuda.CUDAGraph()
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nsteps + 1)] if events else []
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                if events:
                    evs[i].record(stream)
                step(first + i, stream)
            if events:
                evs[nsteps].record(stream)
        return g, evs

    warm_graph, _ = capture(max(1, args.warmup), 0, False)
    # no event nodes between the timed launches: they would stop a launch
    # from overlapping its prologue with the previous one (programmatic
    # dependent launch); the average launch time is the region time / K
    timed_graph, evs = capture(args.steps, args.warmup, args.per_launch_events)

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id) if not args.no_clocks else ClockSampler.disabled()

    def timed_region():
        # graph.replay() launches on torch's current stream: make it `stream`,
        # the stream the timing events are recorded on
        with torch.cuda.stream(stream):
            # keep the GPU busy >= 0.6 s before the timed steps so clock samples see this kernel under load
            soak_t0 = time.time()
            while time.time() - soak_t0 < 0.6:
                warm_graph.replay()
                torch.cuda.synchronize(dev)
            # a graph's first replay also uploads it to the device; do that
            # outside the timed region
            timed_graph.replay()
            torch.cuda.synchronize(dev)
            warm_graph.replay()
            start = torch.cuda.Event(enable_timing=True)
            end = torch.cuda.Event(enable_timing=True)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            start.record(stream)
            timed_graph.replay()
            end.record(stream)
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t_end = time.time()
        ms = start.elapsed_time(end)
        if args.per_launch_events:
            per_launch = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
        else:
            per_launch = [ms / args.steps] * args.steps
        return ms, per_launch, sampler.summary(soak_t0, t_end)

    time.sleep(0.5)
    ms, per_launch, clocks = timed_region()
    remeasured = False
    if clocks_rejected(clocks):
        ms, per_launch, clocks = timed_region()
        remeasured = True
    sampler.stop()
    err = gemm.device_error(clear=True)
    if err:
        raise RuntimeError(f"device error word {err:#x} after the timed region")

    ms_max = max_over_ranks(ms, world, dev)

    # end to end through the public API: pinned host inputs -> device, GEMM, D -> pinned host
    e2e = None
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in host.items()}
        dev_in = sets[0]
        d_host = torch.empty(out_shape, dtype=torch.bfloat16).pin_memory()
        n_e2e = max(3, min(args.steps, 50))

        def e2e_step():
            for k in pin:
                dev_in[k].copy_(pin[k], non_blocking=True)
            step(0, stream)
            d_host.copy_(D, non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(3):
                e2e_step()
            torch.cuda.synchronize(dev)
            if world > 1:
                dist.barrier()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(n_e2e):
                e2e_step()
            s1.record(stream)
            torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / n_e2e, world, dev)
        e2e = {"value": world * acc["flops"] / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(sum(v.nbytes for v in pin.values())),
               "d2h_bytes_per_step": int(d_host.nbytes), "steps": n_e2e,
               "note": "pinned host inputs copied to the device, GEMM through the C ABI, D copied back, every step"}

    if rank != 0:
        return

    pk = peaks()
    ridge = pk["bf16"] * FP8_OVER_BF16 * 1e12 / (pk["hbm"] * 1e9)
    intensity = acc["flops"] / acc["bytes"]
    avg_launch_s = statistics.mean(per_launch) * 1e-3
    if intensity < ridge:
        achieved = acc["bytes"] / avg_launch_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"], "peak_source": f"hbm_gbs of {pk['source']}"}
    else:
        achieved = acc["flops"] / avg_launch_s / 1e12
        peak = pk["bf16"] * FP8_OVER_BF16
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                "peak_source": f"bf16_tflops (burst) of {pk['source']} x {FP8_OVER_BF16} (FP8:BF16 nominal)"}
    roof["traffic"] = ncu_traffic(args.workload, variant)
    roof["kernel"] = variant
    roof["algorithmic_bytes_per_launch"] = acc["bytes"]
    roof["algorithmic_flops_per_launch"] = acc["flops"]
    roof["avg_launch_us"] = avg_launch_s * 1e6
    roof["launch_time_source"] = ("CUDA events around every launch" if args.per_launch_events else
                                  "CUDA events around the K back-to-back launches of the timed region, / K")
    if kernels_per_call(variant) > 1:
        roof["launch_time_source"] += " (a call is the partial-sums kernel and its reduce kernel)"

    value = whole_job_tflops(world, acc["flops"], args.steps, ms_max)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded generator: bf16 N(0,1) draws quantised to e4m3 with 1x128 / 128x128 FP32 scales)",
        "config": {"workload": args.workload, "shape": {k: d[k] for k in ("M", "N", "K", "G", "Mmax") if k in d},
                   "accumulate": "fp32 (per-128-K-block promotion)", "out": "bf16",
                   "l2": (f"inputs rotate over {copies} device copies ({copies * per_copy / 2**20:.0f} MiB > 2x L2)"
                          if copies > 1 else f"inputs {per_copy / 2**20:.0f} MiB >= 2x L2"),
                   "launch": "CUDA graph of the K steps, one C-ABI call each",
                   "variant": variant, "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roof, "gpu_launches": world * args.steps * kernels_per_call(variant), "clocks": clocks,
        "e2e": e2e,
    }
    if remeasured:
        line["clocks_remeasured"] = True
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(d)
    print(json.dumps(line), flush=True)


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(synth.CONFIGS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--variant", type=int, default=None, help="force a kernel variant (tuning)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi clocks (diagnostic)")
    ap.add_argument("--per-launch-events", action="store_true",
                    help="record an event between launches (diagnostic; prevents launch overlap)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0

    import datetime

    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
