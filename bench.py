"""Q4_0 decode-step benchmark on B200.

One step = one decode step of the workload through the C-ABI layer stack
(q4_layer_stack): every GEMV of every layer, in dependency-group order, with the
weights resident in HBM as Q4_0 planes. The default workload is the 8B-class
Llama layer stack (32 layers, 224 GEMVs, 3.93 GB of Q4_0 per step), batch 1: the
working set is 31x the 126 MB L2, so every step streams its weights from HBM
without any flush.

Prints one JSON line (rank 0): whole-job weight GB/s (value), tokens/s, the
roofline of the GEMV kernel against the measured HBM copy peak, the end-to-end
figure through the C ABI with host buffers (activations copied in and results
copied out every step), the oracle timed on the host cores, sampled SM clocks
and the number of library kernels launched in the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--batch B]
  python bench.py --impl reference ...   # the CPU oracle as the reference arm
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import glob
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Q4_0 decode GEMV weight GB/s (% of B200 HBM peak); layer-stack tokens/s"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def source_digest() -> str:
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "quantized_decode_q4_b200", "csrc", "*")))
    for p in files:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, batch: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    kernel sources as they are now; otherwise None."""
    path = os.path.join(ROOT, "profiles", f"gemv_launches_{workload}_b{batch}.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    s = re.search(r"^source_digest:\s*(\w+)", text, re.M)
    if not m or not s or s.group(1) != source_digest():
        return None
    return float(m.group(1))


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [int(r[1]) for r in rows]
        reasons = sorted({self.NAMES[i] for r in rows for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]),
                "sm_mhz_min": min(sm), "samples": len(rows), "reasons": reasons,
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ---------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """A bounded sample of the workload for the CPU oracle: the first `rows` rows of
    every GEMV of the first layer (the first four dependency groups)."""

    def __init__(self, workload, batch: int, rows: int = 64):
        import oracle
        from quantized_decode_q4_b200 import synth
        self.oracle = oracle
        first_groups = sorted({g.group for g in workload.gemvs})[:4]
        self.items = []
        for i, g in enumerate(workload.gemvs):
            if g.group not in first_groups:
                continue
            r = min(rows, g.n)
            w = synth.matrix_rows(workload.seed, g.w_stream, g.k, range(r), synth.WEIGHT_STD)
            blocks = oracle.q4_pack(w.numpy())
            X = workload.activations(i, batch).numpy()
            self.items.append((blocks, r, g.k, X))
        self.weights = sum(r * k for _, r, k, _ in self.items)
        self.q4_bytes = self.weights * 9 // 16
        self.desc = (f"rows 0..{rows - 1} of each of the {len(self.items)} GEMVs of the first "
                     f"layer ({self.weights / 1e6:.2f} M weights, {self.q4_bytes / 1e6:.2f} MB "
                     f"Q4_0), batch {batch}, binary64 oracle GEMV, 1 thread")

    def run_once(self):
        for blocks, r, k, X in self.items:
            if X.shape[0] == 1:
                self.oracle.q4_gemv(blocks, r, k, X[0])
            else:
                self.oracle.q4_gemv_batched(blocks, r, k, X)

    def time(self, seconds: float):
        self.run_once()
        reps, t0 = 0, time.perf_counter()
        while True:
            self.run_once()
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= seconds:
                return reps, dt

    def time_threads(self, seconds: float, threads: int):
        """Passes of the sample completed by `threads` threads running it side by side
        (the oracle's C calls release the GIL) within `seconds`."""
        import threading
        counts = [0] * threads
        t0 = time.perf_counter()
        deadline = t0 + seconds

        def work(i):
            while time.perf_counter() < deadline:
                self.run_once()
                counts[i] += 1

        ts = [threading.Thread(target=work, args=(i,)) for i in range(threads)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
        return sum(counts), time.perf_counter() - t0


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def step_percentiles(ms: list) -> dict:
    """Median, 10th and 90th percentile (linear interpolation) of single-step times."""
    s = sorted(ms)

    def q(p):
        x = p * (len(s) - 1)
        i = int(x)
        return s[i] if i + 1 >= len(s) else s[i] + (s[i + 1] - s[i]) * (x - i)

    return {"steps": len(s), "median_ms": q(0.5), "p10_ms": q(0.1), "p90_ms": q(0.9)}


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of every rank's value (all ranks must call it, in the same order)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: float, steps: int, ms_max: float) -> float:
    """Whole-job weight GB/s: every rank streams bytes_per_step per step; the job takes the
    slowest rank's time."""
    return world * bytes_per_step * steps / (ms_max / 1e3) / 1e9


def reference_arm(args, workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    sample = OracleSample(workload, args.batch)
    for _ in range(args.warmup):
        sample.run_once()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sample.run_once()
    dt = time.perf_counter() - t0
    gbs = sample.q4_bytes * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload.name, "batch": args.batch,
                   "sample": sample.desc},
        "tokens_per_s": gbs * 1e9 / workload.q4_bytes * args.batch,
        "cpu_baseline": {"value": gbs, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample.desc},
        "e2e": {"value": gbs, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA library
# ---------------------------------------------------------------------------

def time_pack_dequant(peak: float, n: int = 14336, k: int = 4096, reps: int = 10) -> dict:
    """The offline calls: q4_pack (binary32 -> Q4_0 planes) and q4_dequant (planes ->
    binary32) on one 14336 x 4096 matrix (235 MB of binary32, larger than L2), outputs
    preallocated, CUDA events on the current stream after 3 warm-up calls. Bytes per
    call: 4 n k + 9 n k / 16 either way (binary32 side + Q4_0 side)."""
    import torch

    from quantized_decode_q4_b200 import q4, synth
    w = synth.matrix(11, 11, n, k, synth.WEIGHT_STD, device="cuda")
    m = q4.pack(w)
    out = torch.empty(n, k, dtype=torch.float32, device="cuda")
    nbytes = 4 * n * k + 9 * n * k // 16
    res = {"matrix": f"{n} x {k} binary32 ({4 * n * k / 1e6:.0f} MB, larger than L2)",
           "bytes_per_call": nbytes}
    for name, fn in (("pack", lambda: q4.pack(w, out=m)), ("dequant", lambda: q4.dequant(m, out=out))):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        e1.synchronize()
        us = e0.elapsed_time(e1) / reps * 1e3
        res[name] = {"us_per_call": us, "gbs": nbytes / us / 1e3, "frac": nbytes / us / 1e3 / peak}
    del w, m, out
    torch.cuda.empty_cache()
    return res


# Every configuration the workloads define beyond the headline one: (workload, batch).
# Largest batch the CUDA-core kernel takes; more tokens go to the tensor cores.
SMALL_BATCH = 4

CONFIG_CASES = [("single_768", 1), ("gpt2_124m", 1), ("smollm2_360m", 1), ("smollm2_360m", 4),
                ("minimind_26m", 1), ("minimind_26m", 2), ("minimind_26m", 8),
                ("minimind_26m", 16), ("smollm2_135m", 1), ("smollm2_135m", 2),
                ("smollm2_135m", 8), ("smollm2_135m", 16), ("llama8b_class", 2),
                ("llama8b_class", 4)]


def measure_configs(peak: float, shared=None, min_steps: int = 200, max_seconds: float = 4.0) -> dict:
    """Decode-step throughput of every configuration in CONFIG_CASES, L2-cold: R
    byte-identical copies of the packed weights (R x weight bytes >= 4 x the 126 MB
    L2) run in turn, all R steps captured in one CUDA graph; CUDA events on the
    replaying stream around whole replays after 3 warm-up replays. Per configuration:
    weight GB/s (Q4_0 bytes per step / step time), tokens/s (batch / step time), ms per
    step and the roofline fraction of the algorithmic bytes (weights + x + y) against
    the measured HBM peak. `shared` maps a workload name to a DecodeStep whose packed
    weights are reused."""
    import math

    import torch

    from quantized_decode_q4_b200 import q4, synth
    from quantized_decode_q4_b200.decode_step import DecodeStep
    out = {}
    for name, b in CONFIG_CASES:
        try:
            wl = synth.workloads()[name]
            base = (shared or {}).get(name)
            step = DecodeStep(wl, b, mats=base.mats if base is not None else None)
            r = max(1, math.ceil(4 * L2_BYTES / step.q4_bytes))
            stacks = step.weight_copies(r)
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                for st in stacks:            # first use outside the capture
                    q4.layer_stack(st, b, step.ws, stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for st in stacks:
                    q4.layer_stack(st, b, step.ws, stream)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    g.replay()
            stream.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                g.replay()
                e1.record(stream)
            e1.synchronize()
            one = e0.elapsed_time(e1) / 1e3
            reps = max(1, min(math.ceil(min_steps / r), int(max_seconds / max(one, 1e-6))))
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            e1.synchronize()
            sec = e0.elapsed_time(e1) / 1e3 / (reps * r)
            out[f"{name}_b{b}"] = {
                "weight_gbs": step.q4_bytes / sec / 1e9, "tokens_per_s": b / sec,
                "ms_per_step": sec * 1e3, "frac": step.algorithmic_bytes / sec / 1e9 / peak,
                "q4_bytes_per_step": step.q4_bytes, "launches_per_step": step.launches,
                "weight_copies": r, "steps_timed": reps * r,
                "l2": f"cold: {r} weight copies, {r * step.q4_bytes / 1e6:.0f} MB in turn",
                "kernel": "q4k::gemv_b1_kernel" if b <= SMALL_BATCH else "q4k::gemv_tc_kernel"}
            del g, stacks, step
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        except Exception as e:  # reported, never allowed to lose the bench line
            out[f"{name}_b{b}"] = {"error": f"{type(e).__name__}: {e}"}
    return out


def profile_gemv(args):
    """Launches of a single GEMV (synthetic weights packed on the GPU) for profilers."""
    import torch

    from quantized_decode_q4_b200 import q4, synth
    n, k = (int(v) for v in args.profile_gemv.split(","))
    w = synth.matrix(7, 7, n, k, synth.WEIGHT_STD, device="cuda")
    m = q4.pack(w)
    del w
    X = synth.normal(7, 8, 0, args.batch * k, 1.0, device="cuda").view(args.batch, k)
    Y = torch.empty(args.batch, n, device="cuda")
    ws = q4.workspace(q4.workspace_bytes(n, k, args.batch))
    for _ in range(args.warmup + args.steps):
        q4.gemv_batched(m, X, Y, ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile_gemv": [n, k], "batch": args.batch,
                      "launches": args.warmup + args.steps,
                      "status": q4.workspace_status(ws)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="llama8b_class")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--launch", default="graph", choices=["graph", "direct"])
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration throughput table")
    ap.add_argument("--profile-gemv", metavar="N,K", default=None,
                    help="no bench line: run --warmup + --steps launches of one GEMV of this "
                         "shape for --batch tokens (a small case for ncu captures)")
    args = ap.parse_args()
    if args.profile_gemv:
        profile_gemv(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        ap.error("at least 3 warm-up steps")

    from quantized_decode_q4_b200 import synth
    workload = synth.workloads()[args.workload]
    if args.batch not in workload.batches and args.batch not in range(1, 17):
        ap.error("batch must be 1..16")

    if args.impl == "reference":
        reference_arm(args, workload)
        return

    import torch
    import torch.distributed as dist

    from quantized_decode_q4_b200 import q4
    from quantized_decode_q4_b200.decode_step import DecodeStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()


    # every rank holds its own replica of the decode step (independent requests)
    step = DecodeStep(workload, args.batch, dev)
    stream = torch.cuda.Stream(dev)
    graph = step.graph(stream) if args.launch == "graph" else None

    def run_step():
        if graph is not None:
            graph.launch(stream)
        else:
            step.run(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            run_step()
    torch.cuda.synchronize()

    # device-timed region: inputs resident in HBM
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local
    clocks = Clocks(gpu_index)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    c0 = q4.launch_count()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            run_step()
        ev1.record(stream)
    ev1.synchronize()
    launches = q4.launch_count() - c0
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world, dev)
    sec = ms / 1e3

    # distribution of single steps (a separate pass: an event between steps keeps the
    # next step's first launch from overlapping the previous step's last one)
    try:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        with torch.cuda.stream(stream):
            evs[0].record(stream)
            for i in range(args.steps):
                run_step()
                evs[i + 1].record(stream)
        evs[-1].synchronize()
        step_dist = step_percentiles([evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)])
    except Exception as e:  # reported, never allowed to lose the bench line
        step_dist = {"error": f"{type(e).__name__}: {e}"}

    # end to end through the C ABI: per step, activations host -> device from pinned
    # memory, the step, and the results device -> host into pinned memory
    x_host = step.x_all.cpu().pin_memory()
    y_host = torch.empty(step.y_all.numel(), dtype=torch.float32).pin_memory()
    with torch.cuda.stream(stream):
        for _ in range(3):
            step.x_all.copy_(x_host, non_blocking=True)
            run_step()
            y_host.copy_(step.y_all, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            step.x_all.copy_(x_host, non_blocking=True)
            run_step()
            y_host.copy_(step.y_all, non_blocking=True)
        e1.record(stream)
    e1.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

    q4_bytes = step.q4_bytes
    value = whole_job_gbs(world, q4_bytes, args.steps, ms)
    e2e = whole_job_gbs(world, q4_bytes, args.steps, e2e_ms)
    peak, peak_src = hbm_peak()
    per_gpu_alg = step.algorithmic_bytes * args.steps / sec / 1e9
    traffic = recorded_traffic(args.workload, args.batch)

    if rank == 0:
        # the offline calls of the path (pack, dequant), after the timed decode steps
        try:
            offline = time_pack_dequant(peak)
        except Exception as e:  # reported, never allowed to lose the bench line
            offline = {"error": f"{type(e).__name__}: {e}"}
        # every other configuration, L2-cold (one GPU only: keeps scaling runs short)
        configs = (measure_configs(peak, shared={args.workload: step}) if world == 1 and
                   not args.no_configs else {"skipped": "measured at one GPU"})
        # the oracle on the host: one thread, then every core of this process
        cpu = OracleSample(workload, args.batch)
        reps1, dt1 = cpu.time(args.cpu_seconds / 2)
        cores = host_cores()
        reps, dt = cpu.time_threads(args.cpu_seconds / 2, cores)
        cpu_gbs = cpu.q4_bytes * reps / dt / 1e9
        cpu_gbs1 = cpu.q4_bytes * reps1 / dt1 / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if args.batch <= SMALL_BATCH else "bf16", "data": "synthetic",
            "config": {
                "workload": args.workload, "batch": args.batch,
                "arith": ("exact integer block dot products of 4-bit codes with 31-bit block "
                          "fixed-point activations (two 16-bit digit planes, dp2a); a 1024-weight "
                          "slice holding an element the fixed point cannot carry within 2^-14 "
                          "of itself is multiplied in binary32; binary32 scales and sums"
                          if args.batch == 1 else
                          "binary32 on the CUDA cores: each code word unpacked once into exact "
                          "(q - 8) pairs, f32x2 fused multiply-adds per token, binary32 sums"
                          if args.batch <= SMALL_BATCH else
                          "tcgen05 bf16 MMA: (q - 8) exact in bf16, activations as bf16 hi + lo "
                          "(2^-16 relative), binary32 accumulators and sums"),
                "gemvs_per_step": len(workload.gemvs), "q4_bytes_per_step": q4_bytes,
                "weights": "Q4_0 planes (4.5 bits/weight), binary32 activations and sums",
                "launch": ("one CUDA graph per step of PDL-chained group launches"
                           if graph is not None else "PDL-chained group launches"),
                "l2": (f"no flush: the weights of one step ({q4_bytes / 1e9:.2f} GB) are "
                       f"{q4_bytes / L2_BYTES:.0f}x the 126 MB L2"
                       if q4_bytes > 4 * L2_BYTES else
                       "working set within 4x L2: figure is L2-warm"),
                "parallelism": f"replicas x{world} (one decode step per GPU, no collectives)",
            },
            "tokens_per_s": world * args.batch * args.steps / sec,
            "pct_hbm_peak_measured": 100.0 * value / world / peak,
            "pct_hbm_peak_nominal": 100.0 * value / world / NOMINAL_HBM_GBS,
            "roofline": {
                "bound": "hbm", "achieved": per_gpu_alg, "peak": peak, "unit": "GB/s",
                "frac": per_gpu_alg / peak, "traffic": traffic,
                "kernel": ("q4k::gemv_b1_kernel" if args.batch <= SMALL_BATCH else
                           "q4k::gemv_tc_kernel"),
                "peak_source": peak_src,
                "note": ("achieved = algorithmic bytes of a step (Q4_0 weights + x + y) / step "
                         f"time; the step is {step.launches} launches of this one kernel, so "
                         "this equals bytes per launch / mean launch duration"),
            },
            "cpu_baseline": {"value": cpu_gbs, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": (cpu.desc.replace(", 1 thread", "") +
                                        f", {cores} threads side by side: {reps} passes in "
                                        f"{dt:.1f} s"),
                             "single_thread": {"value": cpu_gbs1, "unit": UNIT, "cores": 1,
                                               "passes": reps1, "seconds": round(dt1, 2)}},
            "e2e": {"value": e2e, "unit": UNIT,
                    "h2d_bytes_per_step": step.x_all.numel() * 4,
                    "d2h_bytes_per_step": step.y_all.numel() * 4},
            "gpu_launches": launches,
            "clocks": clock_info,
            "offline_kernels": offline,
            "configs": configs,
            "step_ms_single": step_dist,
        }
        print(json.dumps(line), flush=True)
    if graph is not None:
        graph.close()
    if world > 1:
        barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
