#!/usr/bin/env python
"""Throughput of the fused row-normalisation path on B200 (one JSON line on stdout).

Default workload (one step = one add_rms_norm call through the C ABI):
    add_rms_norm, bfloat16 I/O, x and r [8192, 4096] ~ N(0, 1), w [4096] ~ U(0.5, 1.5),
    eps = 1e-5; outputs y and h = x + r.
Metric: achieved HBM GB/s of algorithmic bytes (4 N s + D s per call, s = 2) and rows/s,
against B200's HBM peak.  Each step is timed with CUDA events on the launching stream.
Steps rotate over device buffer sets and run back to back; between two uses of one set the
other sets move at least 3x L2 through the cache, so no step reads data a previous step
left in L2, and every step pays the write-back of its predecessor's output (workloads
whose buffers are too small for that -- under 3/8 of L2 -- are timed one step at a time
after an L2 flush instead).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --sweep        # add_rms_norm over D x rows x dtype, one line per point

Multi-GPU (torchrun, one process per GPU): rows are independent, so every rank runs its
own batch of the same shape (weak scaling); there is no data-path collective.  The
reported time is the maximum over ranks of the summed per-step device times.

``--impl reference`` times the CPU oracle on a bounded sample of the same workload, on
rank 0 only: the published description of these ops comes with no implementation and no
measurements, so the oracle is the only reference there is.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "add_rms_norm achieved HBM GB/s and rows/s vs 8 TB/s peak (1×B200)"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = {"rows": 8192, "D": 4096, "dtype": "bf16", "eps": 1e-5}
# sources of the timed kernel: recorded ncu traffic is void once these change
KERNEL_SOURCES = ["rope_add_rms_b200/csrc/rms.cuh", "rope_add_rms_b200/csrc/common.cuh"]


# ---- environment --------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, plan):
    """dram bytes per launch recorded from an ncu capture, if neither the kernel's
    sources nor its launch plan have changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    ent = d.get(kernel_key)
    if not ent or ent.get("source_hash") != source_hash() or ent.get("plan") != plan:
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle samples of one GPU while a region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        reasons = sorted({self.NAMES[i] for r in rows for i, v in enumerate(r[2])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---- ranks ------------------------------------------------------------------------------

def shard_seed(rank: int) -> int:
    """Each rank runs its own batch of rows (weak scaling): rank r's inputs use seed r."""
    return rank


def max_over_ranks(values, device="cuda"):
    """Element-wise maximum over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, step_bytes: int, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's time."""
    return world * step_bytes * steps / (max_ms * 1e-3) / 1e9


# ---- workloads ----------------------------------------------------------------------

def algorithmic_bytes(op, rows, D, s, nparts=0):
    if op == "allreduce_add_rms_norm":  # read the parts, r, w; write y, h
        return (nparts + 3) * rows * D * s + D * s
    if op == "add_rms_norm":
        return 4 * rows * D * s + D * s
    if op == "rms_norm":
        return 2 * rows * D * s + D * s
    if op == "layer_norm":
        return 2 * rows * D * s + 2 * D * s
    if op == "norm_rope":
        return 2 * rows * D * s + D * s
    if op == "rms_norm_vjp":          # read x, g, w; write dx, dw
        return 3 * rows * D * s + 2 * D * s
    if op == "layer_norm_vjp":        # read x, g, w; write dx, dw, db
        return 3 * rows * D * s + 3 * D * s
    raise ValueError(op)


def rotation_sets(set_bytes, l2_bytes):
    """Copies of a workload's buffers to rotate over: enough that the other copies, which
    the steps between two uses of one copy touch, hold at least 3x L2 (at least 2 copies,
    at most 9); 1 (and an L2 flush before each step) when even 8 other copies would hold
    less than that."""
    if 8 * set_bytes < 3 * l2_bytes:
        return 1
    return max(2, min(9, 1 + -(-3 * l2_bytes // set_bytes)))


class Case:
    """Device-resident inputs/outputs of one workload and a callable that runs it once.

    Large workloads keep `nsets` copies of their device buffers and step i uses copy
    i % nsets; the other nsets - 1 copies, which the steps in between touch, hold at least
    3x L2, so no line a step reads survives in L2 from the last use of its copy (with 2
    copies of the 268 MB norm_rope set, lines that an L2 bulk prefetch had brought in --
    at normal eviction priority, unlike the streamed rows -- still made up ~5% of a
    step's reads).  Steps run back to back (each then also pays the write-back of the
    previous step's dirty lines, as in a steady stream).  Workloads too small for that
    are timed one step at a time after an L2 flush.
    """

    def __init__(self, op, shape, dtype, seed, **kw):
        from rope_add_rms_b200 import synth
        import rope_add_rms_b200 as nv
        self.op, self.dtype, self.kw = op, dtype, kw
        tdt = synth.DTYPES[dtype]
        self.s = torch.empty((), dtype=tdt).element_size()
        if op == "norm_rope":
            B, H, L, D = shape
            inp = synth.norm_rope_inputs(B, H, L, D, dtype, seed)
            self.rows, self.D, self.L = B * H * L, D, L
        else:
            rows, D = shape
            self.rows, self.D = rows, D
            if op == "add_rms_norm" and rows * D > (1 << 27):
                # hundreds of millions of values: drawn on the device (same recipe)
                inp = {"x": synth.normal_device((rows, D), 0.0, 1.0, seed, synth.X, dtype),
                       "r": synth.normal_device((rows, D), 0.0, 1.0, seed, synth.R, dtype),
                       "w": synth.uniform_device((D,), 0.5, 1.5, seed, synth.W, dtype)}
            elif op == "add_rms_norm":
                inp = synth.add_rms_inputs(rows, D, dtype, seed)
            elif op == "allreduce_add_rms_norm":
                a = synth.allreduce_inputs(rows, D, kw["nparts"], dtype, seed)
                inp = {"r": a["r"], "w": a["w"]}
                inp.update({f"p{i}": p for i, p in enumerate(a["parts"])})
            elif op in ("rms_norm", "rms_norm_vjp"):
                inp = synth.rms_inputs(rows, D, dtype, seed)
            else:
                inp = synth.layer_norm_inputs(rows, D, dtype, seed)
            if op.endswith("_vjp"):
                inp["r"] = synth.normal((rows, D), 0.0, 1.0, seed, synth.R, dtype)  # g
        on_dev = any(v is not None and v.is_cuda for v in inp.values())
        self.host = {k: (v.pin_memory() if v is not None and not on_dev else None)
                     for k, v in inp.items()}
        self.device_drawn = on_dev
        src = inp if on_dev else self.host
        self.nparts = kw.get("nparts", 0)
        self.bytes = algorithmic_bytes(op, self.rows, self.D, self.s, self.nparts)
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        n_row_tensors = 4 if op == "add_rms_norm" else (3 if op.endswith("_vjp") else 2)
        if op == "allreduce_add_rms_norm":
            n_row_tensors = self.nparts + 3
        self.n_row_tensors = n_row_tensors
        self.nsets = rotation_sets(n_row_tensors * self.rows * self.D * self.s, l2)
        self.sets = []
        for _ in range(self.nsets):
            d = {k: (v.clone() if on_dev else v.cuda()) if v is not None else None
                 for k, v in src.items()}
            d["y"] = torch.empty_like(d["r"] if op == "allreduce_add_rms_norm" else d["x"])
            if op == "norm_rope" and kw.get("y_len"):   # a KV cache [B, H, y_len, D]
                d["y"] = torch.empty((self.rows // self.L * kw["y_len"], self.D),
                                     dtype=d["x"].dtype, device="cuda")
            d["h"] = torch.empty_like(d["y"]) if "add_rms_norm" in op else None
            if op.endswith("_vjp"):
                d["dw"] = torch.empty_like(d["w"])
                d["db"] = torch.empty_like(d["w"])
                d["ws"] = torch.empty(max(1, nv.nv_norm_vjp_workspace_size(
                    op[:-4], rows, D)), dtype=torch.uint8, device="cuda")
            self.sets.append(d)
        self.nv = nv
        # explicit frequencies (the Llama 3 or the YaRN scaling) for the general rope call
        self.freqs = None
        if op == "norm_rope" and kw.get("llama3"):
            self.freqs = nv.rope_llama3_freqs(self.D).cuda()
        elif op == "norm_rope" and kw.get("yarn"):
            self.freqs = nv.rope_yarn_freqs(self.D, 10000.0, 8.0, 4096)[0].cuda()
        n_out = 2 if op == "add_rms_norm" else 1
        self.host_out = [] if on_dev or "x" not in self.host else \
            [torch.empty_like(self.host["x"]).pin_memory() for _ in range(n_out)]
        self.plan = None

    @property
    def rotating(self):
        return self.nsets > 1

    def l2_note(self):
        if self.rotating:
            mb = self.nsets * self.n_row_tensors * self.rows * self.D * self.s
            return (f"inputs larger than L2: {self.nsets} buffer sets ({mb / 1e6:.0f} MB) "
                    "rotated, steps back to back, no flush")
        return "L2 flushed before every step (read of 2x L2)"

    def run(self, stream=None, i=0):
        d, nv, k = self.sets[i % self.nsets], self.nv, self.kw
        if self.op == "add_rms_norm":
            nv.nv_add_rms_norm(d["x"], d["r"], d["w"], d["y"], d["h"], k["eps"], stream, self.plan)
        elif self.op == "allreduce_add_rms_norm":
            nv.nv_allreduce_add_rms_norm([d[f"p{j}"] for j in range(self.nparts)], d["r"], d["w"],
                                         d["y"], d["h"], k["eps"], stream=stream)
        elif self.op == "rms_norm":
            nv.nv_rms_norm(d["x"], d["w"], d["y"], k["eps"], stream, self.plan)
        elif self.op == "layer_norm":
            nv.nv_layer_norm(d["x"], d["w"], d["b"], d["y"], k["eps"], stream, self.plan)
        elif self.op == "rms_norm_vjp":
            nv.nv_rms_norm_vjp(d["x"], d["w"], d["r"], d["y"], d["dw"], k["eps"], d["ws"], stream)
        elif self.op == "layer_norm_vjp":
            nv.nv_layer_norm_vjp(d["x"], d["w"], d["r"], d["y"], d["dw"], d["db"], k["eps"],
                                 d["ws"], stream)
        elif k.get("y_len") or self.freqs is not None:
            nv.nv_rope(d["x"], d["w"], d["y"], self.L, k["dims"], k["traditional"], k["base"],
                       k["scale"], k["offset"], 1, k["eps"], freqs=self.freqs,
                       y_len=k.get("y_len", 0), stream=stream, plan=self.plan)
        else:
            nv.nv_norm_rope(d["x"], d["w"], d["y"], self.L, k["dims"], k["traditional"], k["base"],
                            k["scale"], k["offset"], 1, k["eps"], stream, self.plan)

    def run_e2e(self, stream=None, i=0):
        """Host -> device copy of the step's inputs, the call, device -> host of its outputs.
        add_rms_norm goes through the library's host-buffer entry point, which pipelines the
        copies and the compute over row chunks; the other ops copy, call and copy back."""
        d = self.sets[0]
        if self.op == "add_rms_norm":
            self.nv.nv_add_rms_norm_host(self.host["x"], self.host["r"], d["w"],
                                         self.host_out[0], self.host_out[1], d["x"], d["r"],
                                         d["y"], d["h"], self.kw["eps"], 0, stream)
            return
        d["x"].copy_(self.host["x"], non_blocking=True)
        self.run(stream, 0)
        self.host_out[0].copy_(d["y"], non_blocking=True)

    def e2e_bytes(self):
        n = 2 if self.op == "add_rms_norm" else 1
        per = self.rows * self.D * self.s
        return n * per, n * per


def l2_flush_buffer():
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    return torch.zeros(2 * max(l2, 64 << 20), dtype=torch.uint8, device="cuda")


def flush_l2(buf):
    """Evict the cache by reading a buffer of twice its size.  A read leaves clean lines
    behind: writing the buffer instead would leave 2x L2 of dirty lines whose write-back
    the next kernel pays (a 67 MB add_rms_norm step timed 18.5 us after a write flush
    against 12.8 us back to back in steady state)."""
    torch.amax(buf)


class nvtx_range:
    """An NVTX range around a phase of the bench (for nsys timelines and ncu's --nvtx
    filters); a no-op where NVTX is unavailable."""

    def __init__(self, name):
        self.name = name
        self.open = False

    def __enter__(self):
        try:
            torch.cuda.nvtx.range_push(self.name)
            self.open = True
        except Exception:  # noqa: BLE001 -- tracing must never stop the bench
            pass
        return self

    def __exit__(self, *exc):
        if self.open:
            try:
                torch.cuda.nvtx.range_pop()
            except Exception:  # noqa: BLE001
                pass
        return False


def time_span(case, steps, warmup):
    """K back-to-back steps over rotating buffer sets, bracketed by one pair of CUDA
    events on the launching stream; returns the span in ms.  NVTX ranges mark the
    warm-up and the timed steps (one range each: nothing is added between launches)."""
    stream = torch.cuda.current_stream()
    with nvtx_range(f"{case.op} warmup x{warmup}"):
        for i in range(warmup):
            case.run(stream, i)
        torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with nvtx_range(f"{case.op} timed x{steps}"):
        start.record(stream)
        for i in range(steps):
            case.run(stream, i)
        end.record(stream)
        torch.cuda.synchronize()
    return start.elapsed_time(end)


def time_steps(case, steps, warmup, flush, e2e=False):
    """Per-step device times (ms): CUDA events around each call on the launching stream."""
    stream = torch.cuda.current_stream()
    fn = case.run_e2e if e2e else case.run
    use_flush = e2e or not case.rotating
    for i in range(warmup):
        if use_flush:
            flush_l2(flush)
        fn(stream, i)
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if use_flush:
            flush_l2(flush)
        with nvtx_range(f"{case.op}{' e2e' if e2e else ''} step {i}"):
            starts[i].record(stream)
            fn(stream, i)
            ends[i].record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


# ---- arms -----------------------------------------------------------------------------

def cpu_baseline(seconds=10.0, sample_rows=2048):
    """The CPU oracle on a bounded sample of the default workload (rank 0, N = 1)."""
    import oracle
    from rope_add_rms_b200 import synth
    rows, D = sample_rows, WORKLOAD["D"]
    inp = synth.add_rms_inputs(rows, D, "bf16", 0)
    x, r, w = (synth.to_numpy(inp[k]) for k in ("x", "r", "w"))
    o = oracle.get()
    threads = oracle.default_threads()
    o.add_rms_norm(x, r, w, WORKLOAD["eps"], threads=threads)     # warm
    t0 = time.perf_counter()
    reps = 0
    while True:
        o.add_rms_norm(x, r, w, WORKLOAD["eps"], threads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= 1000:
            break
    gbs = algorithmic_bytes("add_rms_norm", rows, D, 2) * reps / el / 1e9
    return {"value": round(gbs, 3), "unit": "GB/s", "cores": o.last_threads, "kind": "oracle",
            "sample": f"{reps} x add_rms_norm bf16 [{rows}, {D}] (of the [8192, 4096] workload), "
                      f"{el:.1f} s wall, fp64 C oracle, rows split over threads",
            "rows_per_s": round(rows * reps / el, 1)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from rope_add_rms_b200 import synth
    rows, D = 512, WORKLOAD["D"]
    inp = synth.add_rms_inputs(rows, D, "bf16", 0)
    x, r, w = (synth.to_numpy(inp[k]) for k in ("x", "r", "w"))
    o = oracle.get()
    threads = oracle.default_threads()
    for _ in range(args.warmup):
        o.add_rms_norm(x, r, w, WORKLOAD["eps"], threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.add_rms_norm(x, r, w, WORKLOAD["eps"], threads=threads)
    el = time.perf_counter() - t0
    nbytes = algorithmic_bytes("add_rms_norm", rows, D, 2)
    gbs = nbytes * args.steps / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "add_rms_norm bf16 [8192,4096] eps 1e-5 (CPU oracle on a "
                               "512-row sample per step)", "rows": rows, "D": D},
        "rows_per_s": round(rows * args.steps / el, 1),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": o.last_threads,
                         "kind": "oracle",
                         "sample": f"{args.steps} steps x add_rms_norm bf16 [{rows}, {D}]"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def other_configs(flush, steps):
    """Fractions of the roofline for the other workloads (reported, not the headline)."""
    peak, peak_src = measured_peak()
    peak_src = f"{peak_src} {peak:g} GB/s"
    out = {}
    cases = {
        "layer_norm bf16 [16384,8192] x~N(0.5,2^2) eps 1e-5":
            Case("layer_norm", (16384, 8192), "bf16", 0, eps=1e-5),
        "norm_rope bf16 [8,32,2048,128] halves offset 0 eps 1e-6":
            Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6, dims=128, traditional=0,
                 base=10000.0, scale=1.0, offset=0),
        "norm_rope bf16 [8,32,2048,128] traditional offset 4096 eps 1e-6":
            Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6, dims=128, traditional=1,
                 base=10000.0, scale=1.0, offset=4096),
        "rms_norm f32 [64,512] eps 1e-6":
            Case("rms_norm", (64, 512), "f32", 0, eps=1e-6),
        "rms_norm_vjp bf16 [8192,4096] eps 1e-5 (dx, dw)":
            Case("rms_norm_vjp", (8192, 4096), "bf16", 0, eps=1e-5),
        "layer_norm_vjp bf16 [16384,8192] eps 1e-5 (dx, dw, db)":
            Case("layer_norm_vjp", (16384, 8192), "bf16", 0, eps=1e-5),
    }
    for name, c in cases.items():
        if c.rotating:
            med = time_span(c, steps, 3) / steps
        else:
            med = statistics.median(time_steps(c, steps, 3, flush))
        gbs = c.bytes / (med * 1e-3) / 1e9
        out[name] = {"median_us": round(med * 1e3, 2), "GB/s": round(gbs, 1),
                     "frac_of_hbm_peak": round(gbs / peak, 4), "peak_source": peak_src,
                     "rows_per_s": round(c.rows / (med * 1e-3), 1)}
        del c
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    import rope_add_rms_b200 as nv
    nv.library()

    case = Case("add_rms_norm", (WORKLOAD["rows"], WORKLOAD["D"]), WORKLOAD["dtype"],
                seed=shard_seed(rank), eps=WORKLOAD["eps"])
    flush = l2_flush_buffer()

    def barrier():
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        torch.cuda.synchronize()

    # warm-up, then the timed steps (back to back, one event pair) with clocks sampled
    barrier()
    with ClockSampler(torch.cuda.current_device()) as clk:
        total_ms = time_span(case, args.steps, args.warmup)
    barrier()
    # per-step distribution, each step bracketed by its own events (informational)
    ts = time_steps(case, min(args.steps, 100), 3, flush)
    barrier()
    e2e_steps = max(3, min(args.steps, 20))
    te = time_steps(case, e2e_steps, 3, flush, e2e=True)
    barrier()
    e2e_ms = sum(te)
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms])

    extras = None
    if rank == 0 and not args.no_extras and world == 1:
        extras = other_configs(flush, max(5, min(args.steps, 50)))
    decode = None
    if rank == 0 and not args.no_extras and world == 1:
        # decode-sized calls are host-bound: the host time inside one C-ABI call next to
        # the kernel time, with the per-pointer driver queries on and off
        decode = {f"{op} {dt} [{r},{d}] checks={'on' if ck else 'off'}":
                  host_cost(op, r, d, dt, checks=ck)
                  for op, r, d, dt in (("rms_norm", 64, 512, "f32"), ("add_rms_norm", 1, 4096, "bf16"))
                  for ck in (True, False)}
    baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        baseline = cpu_baseline(args.cpu_seconds)

    if rank == 0:
        peak, peak_kind = measured_peak()
        step_bytes = case.bytes
        value = job_throughput(world, step_bytes, args.steps, total_ms)
        per_launch_ms = total_ms / args.steps      # average launch duration, back to back
        achieved = step_bytes / (per_launch_ms * 1e-3) / 1e9
        bi, bo = case.e2e_bytes()
        e2e_value = job_throughput(world, step_bytes, e2e_steps, e2e_ms)
        plan = nv.nv_describe_plan("add_rms_norm", WORKLOAD["rows"], WORKLOAD["D"],
                                   torch.bfloat16)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "add_rms_norm bf16 x,r [8192,4096] ~N(0,1), w [4096] "
                                   "~U(0.5,1.5), eps 1e-5 (outputs y, h); per GPU",
                       "rows": WORKLOAD["rows"], "D": WORKLOAD["D"], "global_batch_rows":
                           WORKLOAD["rows"] * world,
                       "l2": case.l2_note(),
                       "parallelism": f"row shards x{world}, no collective",
                       "plan": plan},
            "rows_per_s": round(world * WORKLOAD["rows"] * args.steps / (total_ms * 1e-3), 1),
            "step_us": {"median": round(statistics.median(ts) * 1e3, 3),
                        "p10": round(float(np.percentile(ts, 10)) * 1e3, 3),
                        "p90": round(float(np.percentile(ts, 90)) * 1e3, 3),
                        "how": "each step alone between its own events (not the headline)"},
            "timing": "K steps back to back over rotating buffer sets, one CUDA event pair "
                      "on the launching stream; max over ranks",
            "frac_of_nominal_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": ncu_traffic("add_rms_norm_bf16_8192x4096", plan),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6650 GB/s",
                         "kernel": f"rms_rows_kernel<bf16, VPT={plan['vec_per_thread']}, ADD>",
                         "bytes_per_launch": step_bytes},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": bi,
                    "d2h_bytes_per_step": bo,
                    "ms_per_step": round(e2e_ms / e2e_steps, 4), "steps": e2e_steps,
                    "how": "nv_add_rms_norm_host: pinned host x, r -> device, add_rms_norm, "
                           "y, h -> pinned host, 8 row chunks through copy-in/compute/copy-out streams; "
                           "events on the caller's stream around each step"},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "cpu_baseline": baseline,
            "other_configs": extras,
            "decode_host_us": decode,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


WORKLOADS = {
    "add_rms_norm": lambda: Case("add_rms_norm", (8192, 4096), "bf16", 0, eps=1e-5),
    "rms_norm_small": lambda: Case("rms_norm", (64, 512), "f32", 0, eps=1e-6),
    "rms_norm": lambda: Case("rms_norm", (8192, 4096), "bf16", 0, eps=1e-5),
    "layer_norm": lambda: Case("layer_norm", (16384, 8192), "bf16", 0, eps=1e-5),
    "norm_rope_halves": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6,
                                     dims=128, traditional=0, base=10000.0, scale=1.0, offset=0),
    "norm_rope_traditional": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6,
                                          dims=128, traditional=1, base=10000.0, scale=1.0,
                                          offset=4096),
    # partial rotary: only the first 64 of the 128 features rotate (halves (i, i + 32)), the
    # rest are normalised and weighted only
    "norm_rope_partial": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6,
                                      dims=64, traditional=0, base=10000.0, scale=1.0,
                                      offset=0),
    # NormRope's cache form: the 2048 new positions of every (b, h) written into a KV cache
    # of 8192 positions at offset 4096
    "norm_rope_cache": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6,
                                    dims=128, traditional=0, base=10000.0, scale=1.0,
                                    offset=4096, y_len=8192),
    # NormRope with the Llama 3 scaled frequencies (base 500000), past the original context
    "norm_rope_llama3": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-5,
                                     dims=128, traditional=0, base=500000.0, scale=1.0,
                                     offset=16384, llama3=True),
    # NormRope with YaRN frequencies (factor 8 over an original context of 4096), past it
    "norm_rope_yarn": lambda: Case("norm_rope", (8, 32, 2048, 128), "bf16", 0, eps=1e-6,
                                   dims=128, traditional=0, base=10000.0, scale=1.0,
                                   offset=16384, yarn=True),
    # narrow rows: a per-head RMSNorm (128 features), a 256-feature LayerNorm and its
    # gradient (rows narrower than a warp, several to a warp)
    "rms_norm_per_head": lambda: Case("rms_norm", (524288, 128), "bf16", 0, eps=1e-6),
    "layer_norm_narrow": lambda: Case("layer_norm", (262144, 256), "bf16", 0, eps=1e-5),
    "layer_norm_vjp_narrow": lambda: Case("layer_norm_vjp", (262144, 256), "bf16", 0,
                                          eps=1e-5),
    "rms_norm_vjp": lambda: Case("rms_norm_vjp", (8192, 4096), "bf16", 0, eps=1e-5),
    "layer_norm_vjp": lambda: Case("layer_norm_vjp", (16384, 8192), "bf16", 0, eps=1e-5),
    # a TP8 decoder's all-reduce + residual add + RMSNorm, the 8 partial outputs already
    # in this GPU's memory (the reduction half of a one-shot all-reduce)
    "allreduce_add_rms_norm": lambda: Case("allreduce_add_rms_norm", (8192, 4096), "bf16", 0,
                                           eps=1e-5, nparts=8),
}


def run_workload(args):
    """One named workload (not the headline metric): GB/s of algorithmic bytes."""
    torch.cuda.set_device(dist_env()[2])
    c = WORKLOADS[args.workload]()
    import rope_add_rms_b200 as nv
    if args.plan:
        c.plan = nv.Plan(**json.loads(args.plan))
    flush = l2_flush_buffer()
    peak, peak_src = measured_peak()
    peak_src = f"{peak_src} {peak:g} GB/s"
    if c.rotating:
        ms = time_span(c, args.steps, args.warmup) / args.steps
    else:
        ms = statistics.median(time_steps(c, args.steps, args.warmup, flush))
    gbs = c.bytes / (ms * 1e-3) / 1e9
    plan = c.plan.as_dict() if c.plan is not None else None
    print(json.dumps({"workload": args.workload, "op": c.op, "rows": c.rows, "D": c.D, "plan": plan,
                      "dtype": c.dtype, "us_per_call": round(ms * 1e3, 3), "GB/s": round(gbs, 1),
                      "frac_of_hbm_peak": round(gbs / peak, 4), "peak_source": peak_src,
                      "rows_per_s": round(c.rows / (ms * 1e-3), 1), "l2": c.l2_note()}),
          flush=True)
    return 0


# Forced plans the sweep compares with the automatic one (register path at every vector
# count, with one or two rows per CTA, persistent grids, and the staged path).
SWEEP_PLANS = (
    [{"path": 1, "vec_per_thread": v} for v in (1, 2, 4, 8)]
    + [{"path": 1, "vec_per_thread": v, "rows_per_cta": 2} for v in (2, 4, 8)]
    + [{"path": 1, "vec_per_thread": 4, "ctas_per_sm": c} for c in (2, 4)]
    + [{"path": 3}, {"path": 3, "ctas_per_sm": 2}]
)


def host_cost(op, rows, D, dtype, iters=200, checks=True):
    """Host time inside one C-ABI call and device time per call (tests/c/host_cost.c,
    compiled here with gcc): the decode-size story, where the call's host cost can exceed
    the kernel.  checks=False turns the library's per-pointer driver queries off first.
    None if the program cannot be built."""
    import shutil
    from rope_add_rms_b200 import library_path
    if shutil.which("gcc") is None:
        return None
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = os.path.join(tempfile.gettempdir(), f"nv_host_cost_{os.getpid()}")
    if not os.path.exists(exe):
        libdir = os.path.dirname(library_path)
        cmd = ["gcc", "-std=c99", "-O2", "-I", os.path.join(ROOT, "include"),
               "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c", "host_cost.c"),
               "-o", exe, "-L", libdir, "-lnvnorm", "-L", os.path.join(cuda, "lib64"), "-lcudart",
               f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}"]
        if subprocess.run(cmd, capture_output=True).returncode != 0:
            return None
    res = subprocess.run([exe, "add" if op == "add_rms_norm" else "rms", str(rows), str(D),
                          dtype, str(iters)] + ([] if checks else ["nochecks"]),
                         capture_output=True, text=True, timeout=120)
    if res.returncode != 0:
        return None
    return json.loads(res.stdout)


def run_sweep(args):
    """add_rms_norm over D x rows x dtype (eps 1e-6): one JSON line per point.  Points of
    >= 4096 rows also time every forced plan of SWEEP_PLANS and report the best next to the
    automatic plan; points of <= 256 rows add the host cost of one call through the C ABI
    (latency-bound: the kernel time is not an HBM figure there)."""
    import rope_add_rms_b200 as nv
    torch.cuda.set_device(dist_env()[2])
    flush = l2_flush_buffer()
    peak, _ = measured_peak()

    def timed(c):
        if c.rotating:
            return time_span(c, args.steps, args.warmup) / args.steps
        return statistics.median(time_steps(c, args.steps, args.warmup, flush))

    for dtype in ("bf16", "f32"):
        for D in (2048, 4096, 5120, 8192, 16384):
            for rows in (1, 16, 256, 4096, 65536):
                c = Case("add_rms_norm", (rows, D), dtype, 0, eps=1e-6)
                med = timed(c)
                gbs = c.bytes / (med * 1e-3) / 1e9
                auto = nv.nv_describe_plan("add_rms_norm", rows, D,
                                           torch.bfloat16 if dtype == "bf16" else torch.float32)
                line = {"op": "add_rms_norm", "dtype": dtype, "rows": rows, "D": D,
                        "median_us": round(med * 1e3, 2), "GB/s": round(gbs, 1),
                        "frac": round(gbs / peak, 4),
                        "rows_per_s": round(rows / (med * 1e-3), 1),
                        "bound": "hbm" if rows >= 4096 else "latency", "plan": auto}
                if rows >= 4096 and args.plans:
                    best = None
                    for p in SWEEP_PLANS:
                        c.plan = nv.Plan(**p)
                        try:
                            m = timed(c)
                        except nv.NvError:
                            continue
                        if best is None or m < best[0]:
                            best = (m, p)
                    c.plan = None
                    if best:
                        bg = c.bytes / (best[0] * 1e-3) / 1e9
                        line["best_forced"] = {"plan": best[1], "median_us": round(best[0] * 1e3, 2),
                                               "GB/s": round(bg, 1)}
                        line["auto_over_best"] = round(gbs / bg, 4)
                if rows <= 256:
                    line["host_call"] = host_cost("add_rms_norm", rows, D, dtype)
                    line["host_call_nochecks"] = host_cost("add_rms_norm", rows, D, dtype,
                                                           checks=False)
                print(json.dumps(line), flush=True)
                del c
                torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--plans", action="store_true",
                    help="with --sweep: also time the forced plans at each large point")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=None,
                    help="time one named workload instead of the headline step")
    ap.add_argument("--plan", default=None,
                    help="with --workload: a forced nv_plan as JSON, e.g. '{\"path\": 4}'")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.workload:
        return run_workload(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
