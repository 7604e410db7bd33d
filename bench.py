#!/usr/bin/env python
"""Benchmark of the fine-grained-scaled FP8 GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one call of the GEMM over one batch of seeded synthetic input (all
of the path: TMA tile loads, FP8 MMA per K-block, FP32 promotion, tile
scheduling, bf16 epilogue).  The default (headline) workload is the largest
single-GPU configuration of the benchmark table: the contiguous M-grouped
GEMM with 4 experts of 8192 rows, N=4096, K=7168.  The metric is per shape,
so the same JSON line also carries a `per_shape` object with every workload
of the table (dense 128x256x512, dense 64x2112x7168, dense 4096x7168x16384,
contiguous, masked G=16), each timed in the same run with its own roofline,
clock record and CPU-oracle baseline.

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
DEFAULT_WORKLOAD = "contiguous_g4_m8192_n4096_k7168"
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
    # each step a bounded sample: about 1.5 s, less when there are many steps,
    # so that the whole run (warm-up included) takes about a minute at most
    step_s = min(1.5, max(0.2, 60.0 / (args.steps + args.warmup)))
    per_step_rows = max(1, int(min(acc["rows"], n1 * step_s / max(dt1, 1e-6))))
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

# timed launches per shape in the per_shape block (at least --steps): enough
# that each shape's timed region lasts ~10 ms or more
PER_SHAPE_STEPS = {"dense_128x256x512": 400, "dense_64x2112x7168": 400, "dense_4096x7168x16384": 20,
                   "contiguous_g4_m8192_n4096_k7168": 10, "masked_g16_m256_n4096_k7168": 60}


class Shape:
    """One workload on the device: inputs (rotated over enough copies that each
    step reads HBM), output, and a step function calling the C ABI."""

    def __init__(self, name: str, rank: int, dev):
        import torch
        from fp8_block_scaled_x128_b200 import gemm
        self.gemm = gemm
        self.name = name
        self.dev = dev
        d = workload_inputs(name, rank)
        d["name"] = name
        self.d = d
        self.acc = accounting(d)
        self.kind = d["kind"]
        self.per_copy = input_bytes(d)
        self.copies = 1 if self.per_copy >= 2 * L2_BYTES else int(math.ceil(2 * L2_BYTES / self.per_copy))
        self.host = {k: torch.from_numpy(np.ascontiguousarray(d[k])) for k in ("A", "sa", "B", "sb")}
        if self.kind == "contiguous":
            self.host["idx"] = torch.from_numpy(d["m_indices"])
        elif self.kind == "masked":
            self.host["idx"] = torch.from_numpy(d["masked_m"])
        self.sets = [{k: v.to(dev) for k, v in self.host.items()} for _ in range(self.copies)]
        self.out_shape = (d["G"], d["Mmax"], d["N"]) if self.kind == "masked" else (d["M"], d["N"])
        self.D = torch.empty(self.out_shape, dtype=torch.bfloat16, device=dev)

    def step(self, i: int, stream):
        g, t, d = self.gemm, self.sets[i % self.copies], self.d
        if self.kind == "dense":
            g.fp8_gemm_nt(t["A"], t["sa"], t["B"], t["sb"], D=self.D, stream=stream)
        elif self.kind == "contiguous":
            g.m_grouped_fp8_gemm_nt_contiguous(t["A"], t["sa"], t["B"], t["sb"], t["idx"], D=self.D, stream=stream)
        else:
            g.m_grouped_fp8_gemm_nt_masked(t["A"], t["sa"], t["B"], t["sb"], t["idx"], d["expected_m"], D=self.D,
                                           stream=stream)

    def l2_note(self) -> str:
        if self.copies > 1:
            return f"inputs rotate over {self.copies} device copies ({self.copies * self.per_copy / 2**20:.0f} MiB > 2x L2)"
        return f"inputs {self.per_copy / 2**20:.0f} MiB >= 2x L2"


def time_shape(S: Shape, steps: int, warmup: int, stream, sampler, world: int, per_launch_events: bool):
    """Device time of `steps` back-to-back calls replayed from one CUDA graph,
    bracketed by a barrier and a synchronise on both sides (max over ranks).
    Returns (ms, per-launch ms list, clock summary, variant name)."""
    import torch
    import torch.distributed as dist
    dev = S.dev
    with torch.cuda.stream(stream):
        S.step(0, stream)  # per-device set-up outside capture
    torch.cuda.synchronize(dev)
    variant = S.gemm.variant_names()[S.gemm.last_variant()]

    def capture(nsteps: int, first: int, events: bool):
        g = torch.cuda.CUDAGraph()
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nsteps + 1)] if events else []
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                if events:
                    evs[i].record(stream)
                S.step(first + i, stream)
            if events:
                evs[nsteps].record(stream)
        return g, evs

    warm_graph, _ = capture(max(1, warmup), 0, False)
    # no event nodes between the timed launches: they would stop a launch
    # from overlapping its prologue with the previous one (programmatic
    # dependent launch); the average launch time is the region time / K
    timed_graph, evs = capture(steps, warmup, per_launch_events)

    def region():
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
        per_launch = ([evs[i].elapsed_time(evs[i + 1]) for i in range(steps)] if per_launch_events
                      else [ms / steps] * steps)
        return ms, per_launch, sampler.summary(soak_t0, t_end)

    ms, per_launch, clocks = region()
    if clocks_rejected(clocks):
        ms, per_launch, clocks = region()
        if clocks is not None:
            clocks["remeasured"] = True
    err = S.gemm.device_error(clear=True)
    if err:
        raise RuntimeError(f"device error word {err:#x} after the timed region of {S.name}")
    del warm_graph, timed_graph
    return ms, per_launch, clocks, variant


def roofline(acc, avg_launch_s: float, workload: str, variant: str, per_launch_events: bool) -> dict:
    pk = peaks()
    ridge = pk["bf16"] * FP8_OVER_BF16 * 1e12 / (pk["hbm"] * 1e9)
    intensity = acc["flops"] / acc["bytes"]
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
    roof["traffic"] = ncu_traffic(workload, variant)
    roof["kernel"] = variant
    roof["algorithmic_bytes_per_launch"] = acc["bytes"]
    roof["algorithmic_flops_per_launch"] = acc["flops"]
    roof["avg_launch_us"] = avg_launch_s * 1e6
    roof["launch_time_source"] = ("CUDA events around every launch" if per_launch_events else
                                  "CUDA events around the K back-to-back launches of the timed region, / K")
    if kernels_per_call(variant) > 1:
        roof["launch_time_source"] += " (a call is the partial-sums kernel and its reduce kernel)"
    return roof


def e2e_measure(S: Shape, steps: int, stream, world: int) -> dict:
    """The same metric end to end through the public API: pinned host inputs
    copied to the device, the C-ABI call, D copied back to pinned host memory,
    every step."""
    import torch
    import torch.distributed as dist
    dev = S.dev
    pin = {k: v.pin_memory() for k, v in S.host.items()}
    dev_in = S.sets[0]
    d_host = torch.empty(S.out_shape, dtype=torch.bfloat16).pin_memory()
    n_e2e = max(3, min(steps, 50))

    def e2e_step():
        for k in pin:
            dev_in[k].copy_(pin[k], non_blocking=True)
        S.step(0, stream)
        d_host.copy_(S.D, non_blocking=True)

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
    return {"value": world * S.acc["flops"] / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": int(sum(v.nbytes for v in pin.values())),
            "d2h_bytes_per_step": int(d_host.nbytes), "steps": n_e2e,
            "note": "pinned host inputs copied to the device, GEMM through the C ABI, D copied back, every step"}


def measure_extras(dev, stream, sampler, steps: int) -> dict:
    """The pieces around the GEMM, each timed in the same run on seeded
    synthetic inputs larger than L2: the FP8 quantisers, the expert dispatch and
    combine of the contiguous layout (a routing of 8192 tokens x top-4 over 4
    experts, the contiguous workload's 32768 rows), the BF16 GEMM and the FP8
    GEMM with power-of-two scales.  Each
    entry: device time per call (CUDA events over `steps` back-to-back calls
    after warm-up) and its roofline against the measured peaks."""
    import torch
    from fp8_block_scaled_x128_b200 import gemm
    pk = peaks()
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    out = {}

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            torch.cuda.synchronize(dev)
            t0 = time.time()
            while time.time() - t0 < 0.3:
                fn()
                torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0 = time.time()
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps * 1e-3, sampler.summary(s0 - 0.3, time.time())

    def hbm(name, nbytes, fn, what):
        sec, clk = timed(fn)
        gbs = nbytes / sec / 1e9
        out[name] = {"what": what, "us_per_call": sec * 1e6, "roofline": {
            "bound": "hbm", "achieved": gbs, "peak": pk["hbm"], "unit": "GB/s", "frac": gbs / pk["hbm"],
            "algorithmic_bytes_per_call": nbytes, "peak_source": f"hbm_gbs of {pk['source']}"}, "clocks": clk}

    # quantisers: bf16 activations [32768, 7168] and 4 experts' weights [16384, 7168]
    T, K, N, G, topk = 8192, 7168, 4096, 4, 4
    x = torch.randn(4 * T, K, generator=gen, device=dev).to(torch.bfloat16)
    q, sa = gemm.quantize_1x128(x)
    hbm("quantize_1x128_bf16_32768x7168", x.numel() * 3 + sa.numel() * 4,
        lambda: gemm.quantize_1x128(x, q, sa, stream=stream), "activations, one scale per 1x128 group")
    w = (torch.randn(G * N, K, generator=gen, device=dev) * 0.02).to(torch.bfloat16)
    qb, sb = gemm.quantize_128x128(w)
    hbm("quantize_128x128_bf16_16384x7168", w.numel() * 3 + sb.numel() * 4,
        lambda: gemm.quantize_128x128(w, qb, sb, stream=stream), "weights, one scale per 128x128 block")
    del x, q, sa, w, qb, sb
    # expert dispatch + combine around the contiguous GEMM
    xt = torch.randn(T, K, generator=gen, device=dev).to(torch.bfloat16)
    e = torch.stack([torch.randperm(G, generator=gen, device=dev) for _ in range(T)]).to(torch.int32).reshape(-1)
    R = T * topk
    bufs = list(gemm.moe_dispatch(xt, e, topk, G))
    ws = torch.empty((gemm.lib.fp8g_moe_dispatch_workspace_bytes(R, G) + 3) // 4, dtype=torch.int32, device=dev)
    outs = (bufs[0], bufs[1], torch.empty(R, dtype=torch.int32, device=dev), bufs[3], ws)
    hbm("moe_dispatch_8192x4_g4_k7168", T * K * 2 + R * K + R * (K // 128) * 4 + 2 * R * 4,
        lambda: gemm.moe_dispatch(xt, e, topk, G, out=outs, stream=stream),
        "routing -> contiguous layout, tokens quantised into it (counts, ranks, gather, padding)")
    pos = outs[2]
    Dm = torch.randn(bufs[0].shape[0], N, generator=gen, device=dev).to(torch.bfloat16)
    wts = torch.rand(R, generator=gen, device=dev)
    comb = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    hbm("moe_combine_8192x4_n4096", R * N * 2 + T * N * 2 + R * 8,
        lambda: gemm.moe_combine(Dm, pos, wts, T, topk, out=comb, stream=stream),
        "GEMM rows back to tokens, weighted FP32 sum over the top-4 slots")
    del xt, e, bufs, outs, Dm, wts, comb
    # BF16 GEMM 8192^3 against the measured bf16 peak
    Mb = 8192
    A = torch.randn(Mb, Mb, generator=gen, device=dev).to(torch.bfloat16)
    B = (torch.randn(Mb, Mb, generator=gen, device=dev) * 0.05).to(torch.bfloat16)
    Db = torch.empty(Mb, Mb, dtype=torch.bfloat16, device=dev)
    sec, clk = timed(lambda: gemm.bf16_gemm_nt(A, B, Db, stream=stream))
    tf = 2.0 * Mb ** 3 / sec / 1e12
    out["bf16_gemm_8192x8192x8192"] = {"what": "BF16 NT GEMM, FP32 accumulation", "us_per_call": sec * 1e6,
                                       "variant": gemm.variant_names()[gemm.last_variant()], "roofline": {
        "bound": "tensor", "achieved": tf, "peak": pk["bf16"], "unit": "TFLOP/s", "frac": tf / pk["bf16"],
        "peak_source": f"bf16_tflops (burst) of {pk['source']}"}, "clocks": clk}
    del A, B, Db
    # FP8 GEMM with power-of-two scales (block-scaled MMA) on the large dense shape
    M3, N3, K3 = 4096, 7168, 16384
    A = torch.randint(0, 126, (M3, K3), generator=gen, device=dev, dtype=torch.uint8)
    B = torch.randint(0, 126, (N3, K3), generator=gen, device=dev, dtype=torch.uint8)
    sfa = torch.randint(120, 128, (K3 // 128, M3), generator=gen, device=dev, dtype=torch.uint8)
    sfb = torch.randint(120, 128, ((N3 + 127) // 128, K3 // 128), generator=gen, device=dev, dtype=torch.uint8)
    D3 = torch.empty(M3, N3, dtype=torch.bfloat16, device=dev)
    sec, clk = timed(lambda: gemm.fp8_gemm_nt_ue8m0(A, sfa, B, sfb, D3, stream=stream))
    tf = 2.0 * M3 * N3 * K3 / sec / 1e12
    peak = pk["bf16"] * FP8_OVER_BF16
    out["ue8m0_gemm_4096x7168x16384"] = {"what": "FP8 GEMM with power-of-two scales on the block-scaled MMA",
                                         "us_per_call": sec * 1e6, "variant": gemm.variant_names()[gemm.last_variant()],
                                         "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                                                      "frac": tf / peak, "peak_source":
                                                      f"bf16_tflops (burst) of {pk['source']} x {FP8_OVER_BF16}"},
                                         "clocks": clk}
    del A, B, sfa, sfb, D3
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank: int, world: int) -> None:
    import torch

    from fp8_block_scaled_x128_b200 import gemm

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    if args.variant is not None:
        gemm.set_variant_override(args.variant)
    stream = torch.cuda.Stream(device=dev)
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id) if not args.no_clocks else ClockSampler.disabled()
    time.sleep(0.5)
    with_cpu = world == 1 and rank == 0 and not args.no_cpu_baseline
    try:
        # the headline workload: exactly --steps timed steps, e2e, oracle baseline
        S = Shape(args.workload, rank, dev)
        ms, per_launch, clocks, variant = time_shape(S, args.steps, args.warmup, stream, sampler, world,
                                                     args.per_launch_events)
        ms_max = max_over_ranks(ms, world, dev)
        e2e = None if args.no_e2e else e2e_measure(S, args.steps, stream, world)
        head = dict(S=S, ms=ms_max, per_launch=per_launch, clocks=clocks, variant=variant)
        headline_cpu = cpu_baseline(S.d) if with_cpu else None
        head_acc, head_d, head_l2 = S.acc, S.d, S.l2_note()
        del S
        torch.cuda.empty_cache()

        # every workload of the benchmark table, measured in the same run
        per_shape = {}
        if not args.no_per_shape:
            for name in synth.CONFIGS:
                if name == args.workload:
                    ps_ms, ps_launch, ps_clocks, ps_variant, ps_steps, acc = (
                        ms_max, per_launch, clocks, variant, args.steps, head_acc)
                    ps_cpu = headline_cpu
                else:
                    S = Shape(name, rank, dev)
                    ps_steps = max(args.steps, PER_SHAPE_STEPS.get(name, args.steps))
                    ps_ms, ps_launch, ps_clocks, ps_variant = time_shape(S, ps_steps, args.warmup, stream, sampler,
                                                                         world, args.per_launch_events)
                    ps_ms = max_over_ranks(ps_ms, world, dev)
                    acc = S.acc
                    ps_cpu = cpu_baseline(S.d, target_s=4.0) if with_cpu else None
                    del S
                    torch.cuda.empty_cache()
                avg_s = ps_ms / ps_steps * 1e-3
                per_shape[name] = {
                    "value": whole_job_tflops(world, acc["flops"], ps_steps, ps_ms), "unit": UNIT,
                    "us_per_launch": avg_s * 1e6, "steps": ps_steps, "variant": ps_variant,
                    "roofline": roofline(acc, avg_s, name, ps_variant, args.per_launch_events),
                    "gpu_launches": world * ps_steps * kernels_per_call(ps_variant),
                    "clocks": ps_clocks, "cpu_baseline": ps_cpu,
                }
        extras = {} if args.no_extras else measure_extras(dev, stream, sampler, max(args.steps, 10))
    finally:
        sampler.stop()

    if rank != 0:
        return
    avg_launch_s = statistics.mean(head["per_launch"]) * 1e-3
    line = {
        "metric": METRIC, "value": whole_job_tflops(world, head_acc["flops"], args.steps, head["ms"]), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms"] / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic (seeded generator: bf16 N(0,1) draws quantised to e4m3 with 1x128 / 128x128 FP32 scales)",
        "config": {"workload": args.workload,
                   "shape": {k: head_d[k] for k in ("M", "N", "K", "G", "Mmax") if k in head_d},
                   "accumulate": "fp32 (per-128-K-block promotion)", "out": "bf16", "l2": head_l2,
                   "launch": "CUDA graph of the K steps, one C-ABI call each",
                   "variant": head["variant"], "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": roofline(head_acc, avg_launch_s, args.workload, head["variant"], args.per_launch_events),
        "gpu_launches": world * args.steps * kernels_per_call(head["variant"]), "clocks": head["clocks"],
        "e2e": e2e,
    }
    if headline_cpu is not None:
        line["cpu_baseline"] = headline_cpu
    if per_shape:
        line["per_shape"] = per_shape
    if extras:
        line["extras"] = extras
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
    ap.add_argument("--no-per-shape", action="store_true", help="measure the headline workload only")
    ap.add_argument("--no-extras", action="store_true", help="skip the quantiser / MoE / BF16 measurements")
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
