"""Throughput of the 4-bit Shampoo preconditioner step on B200.

One step = update_stats + refresh_roots + precondition over every tile of the
workload (default: the Llama-style layer set, 8 x 4096x11008 + 8 x 4096x4096
cut into 480 tiles of at most 1024 x 1024, 960 factors), with the gradients
already resident in HBM.  Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload 1..5] [--precision tf32|fp32] [--shapes RxC,...]

--shapes replaces the workload's parameter list (its hyper-parameters and
gradient distribution stay), e.g. ``--shapes 4096x4096`` for a small case
with the same 1024 x 1024 factors as the default workload.  The timed steps
run inside an NVTX push/pop range named "timed", so a profiler can select
exactly their launches (ncu --nvtx --nvtx-include "timed/").

The headline roofline is the whole step's algorithmic work by the formulas
of the work model (bit_quantized_shampoo_b200.costmodel): statistics
2mn(m+n) and precondition 2(m^3+n^3) + 2mn(m+n) per tile, refresh
(4t + 2 + 8/3 + 2) d^3 per factor, amortized over the refresh interval --
divided by the step time, against the precision-weighted tensor peak
(Bjorck, statistics, roots and apply at the TF32 rate; the fp32-accurate
subspace step, QR and Rayleigh product at a third of it).

The four smaller workloads are also timed, each at its own refresh interval
(``configs`` in the line), after the main workload's handle is released.

Multi-GPU: one process per GPU (torchrun).  By default the ranks share one
workload and shard its refresh: each rank refreshes the factors it owns (by
d^3 cost) and the ranks exchange codes, scales and eigenvalues by NCCL
broadcasts ("strong" scaling).  --replicas instead runs an independent copy
per rank with no data-path collective ("weak").
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "precond steps/sec & 1024² root refreshes/sec; quant HBM GB/s; TC util"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", type=int, default=5)
    ap.add_argument("--precision", default="tf32", choices=["tf32", "fp32"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-codec", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-graft", action="store_true")
    ap.add_argument("--compressed", action="store_true",
                    help="keep each statistic only as its 4-bit eigenbasis and eigenvalues")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--replicas", action="store_true",
                    help="with N ranks: N independent copies of the workload (weak scaling) instead of the "
                         "default sharded refresh, where each rank refreshes 1/N of the factors (by cost) and "
                         "the ranks exchange codes, scales and eigenvalues (one NCCL broadcast per rank)")
    ap.add_argument("--no-configs", action="store_true", help="skip timing the four smaller workloads")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip timing the codebook and root-method variants on the transformer layer stack")
    ap.add_argument("--cpu-tiles", type=int, default=48,
                    help="tiles of the CPU baseline's sample: every ragged tile, then seeded full ones")
    ap.add_argument("--shapes", default=None, help="comma-separated RxC list replacing the workload's shapes")
    ap.add_argument("--grad-sets", type=int, default=2,
                    help="seeded gradient sets the steps cycle through (1 = the same gradient every step)")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.samples.append([p.strip() for p in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if len(s) > 5 + i and s[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ peaks
def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "sm_max_mhz": 1965.0}, "fallback"


# B200: 148 SMs; per SM and clock 128 fp32 FMA lanes and 64 fp64 FMA lanes.
def alu_peak_tflops(kind: str, mhz: float) -> float:
    lanes = 128 if kind == "fp32" else 64
    return 148 * lanes * 2 * mhz * 1e6 / 1e12


# Dense TF32 runs at 1.1/2.25 of the dense bf16 rate (nominal per-GPU figures),
# so the TF32 denominator is the measured bf16 throughput times that ratio;
# a 3xTF32 product spends three MMAs per useful one.
TF32_OVER_BF16 = 1.1 / 2.25

# What bounds each stage in the current kernels.
STAGE_BOUND = {
    "stats_gemm": "tf32", "bjorck_gram": "tf32", "bjorck_update": "tf32", "roots": "tf32",
    "apply_left": "tf32", "apply_right": "tf32",
    "subspace": "3xtf32", "rayleigh_gemm": "3xtf32", "qr_gram": "3xtf32", "qr_syrk": "3xtf32",
    "qr_trsm_panel": "3xtf32", "qr_solve_update": "3xtf32", "qr_solve_panel": "3xtf32",
    "qr_potrf": "latency", "qr_inverse": "latency", "rayleigh": "hbm", "requant": "hbm", "precond_dequant": "hbm",
    "basis": "hbm", "stats_scan": "hbm", "refresh_scan": "hbm", "qr_convert": "hbm", "precond_mu": "hbm",
    "stats_dequant": "hbm", "stats_rebuild": "tf32", "tables": "latency",
    "newton_elt": "hbm", "newton_gemm": "3xtf32",
}


# DRAM bytes (read + write) of ONE launch of a stage's tensor-core GEMM per
# element of the factors it processes, from an ncu capture of the GEMM on 32
# factors of 1024 x 1024 (one 4096 x 4096 gradient).  A launch over other
# factors of the same kind moves the same bytes per element.  Valid only for
# the GEMM source it was taken on: the figure is dropped (traffic = null) when
# gemm_tc.cu or tc.h has changed since.
TRAFFIC_SOURCE_SHA = "6c7fb2eaf26f9bd9"
# (The QR Gram stage is left out: its first-pass Gram runs in TF32 since
# that capture, and the fp32-accurate second-pass Gram moves 13.18 B per
# element, so no single per-launch figure describes the stage.)
TRAFFIC_PER_ELEMENT = {"stats_gemm": 6.589, "bjorck_gram": 5.469, "bjorck_update": 10.482,
                       "subspace": 32.758}


def gemm_source_sha():
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "tc.h"):
        with open(os.path.join(ROOT, "bit_quantized_shampoo_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stage_traffic(stage, factor_elems):
    """Per-launch DRAM traffic of the stage's GEMM for factors totalling
    factor_elems elements, or None when no capture covers it."""
    b = TRAFFIC_PER_ELEMENT.get(stage)
    if b is None or gemm_source_sha() != TRAFFIC_SOURCE_SHA:
        return None
    return b * factor_elems


def stage_roofline(name, st, pk, pk_src, sustained=True):
    bound = STAGE_BOUND.get(name, "latency")
    ms = st["ms"]
    per_launch = {"launches_per_step": st["launches"], "ms_per_launch": ms / max(1, st["launches"])}
    if bound == "hbm":
        achieved = st["bytes"] / (ms / 1e3) / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
             "peak_source": pk_src + " HBM copy"}
    elif bound in ("tf32", "3xtf32"):
        bf16 = pk.get("bf16_tflops_sustained" if sustained else "bf16_tflops", 1400.0)
        peak = bf16 * TF32_OVER_BF16 / (3.0 if bound == "3xtf32" else 1.0)
        achieved = st["flops"] / (ms / 1e3) / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
             "peak_source": f"{pk_src} bf16 {'sustained' if sustained else 'burst'} x 1.1/2.25"
                            + (" / 3 (3xTF32)" if bound == "3xtf32" else "")}
    else:
        return {"kernel": name, "bound": "latency", "ms_per_step": ms, "per_launch": per_launch}
    r["frac"] = r["achieved"] / r["peak"]
    r["kernel"] = name
    r["per_launch"] = per_launch
    return r


def step_work(dims, bjorck_iters, refresh_every, precision):
    """Algorithmic flops of one optimizer step by the work model, split by
    the arithmetic each part runs in: (flops at the TF32 rate, flops at the
    3xTF32 rate).  dims: the (m, n) of every tile.  The refresh is amortized
    over refresh_every steps.  In FP32 mode every product is 3xTF32."""
    from bit_quantized_shampoo_b200 import costmodel as cm
    single = triple = 0.0
    for m, n in dims:
        single += cm.stats_flops(m, n) + cm.precondition_flops(m, n)
        for d in (m, n):
            bj = 4.0 * bjorck_iters * float(d) ** 3
            single += bj / refresh_every
            triple += (cm.refresh_flops(d, bjorck_iters) - bj) / refresh_every
    if precision == "fp32":
        single, triple = 0.0, single + triple
    return single, triple


def refresh_work(dims, bjorck_iters, precision):
    """(TF32-rate, 3xTF32-rate) algorithmic flops of one refresh of every factor."""
    from bit_quantized_shampoo_b200 import costmodel as cm
    single = triple = 0.0
    for m, n in dims:
        for d in (m, n):
            bj = 4.0 * bjorck_iters * float(d) ** 3
            single += bj
            triple += cm.refresh_flops(d, bjorck_iters) - bj
    if precision == "fp32":
        single, triple = 0.0, single + triple
    return single, triple


def formula_roofline(work, seconds, pk, pk_src, label, sustained=True):
    """Achieved = algorithmic flops / time; peak = the same flops over their
    ideal time at the TF32 rate (single) and a third of it (triple), i.e. the
    precision-weighted peak; frac = ideal time / time."""
    single, triple = work
    bf16 = pk.get("bf16_tflops_sustained" if sustained else "bf16_tflops", 1400.0)
    tf32 = bf16 * TF32_OVER_BF16
    ideal = single / (tf32 * 1e12) + triple / (tf32 / 3.0 * 1e12)
    total = single + triple
    return {"bound": "tensor", "achieved": total / seconds / 1e12, "peak": total / ideal / 1e12,
            "unit": "TFLOP/s", "frac": ideal / seconds, "kernel": label,
            "flops": total, "flops_tf32": single, "flops_3xtf32": triple, "ideal_ms": ideal * 1e3,
            "peak_source": (f"{pk_src} bf16 {'sustained' if sustained else 'burst'} x 1.1/2.25 (TF32), "
                            f"a third of that for 3xTF32; weighted by the flops at each")}


def workload_shapes(wid, shapes=None):
    import dataclasses
    from bit_quantized_shampoo_b200.workloads import WORKLOADS
    w = WORKLOADS[wid]
    if shapes:
        dims = tuple(tuple(int(v) for v in item.lower().split("x")) for item in shapes.split(","))
        if not dims or any(len(d) != 2 or min(d) < 1 for d in dims):
            raise SystemExit(f"--shapes: expected RxC[,RxC...], got {shapes!r}")
        w = dataclasses.replace(w, shapes=dims, name=f"{w.name}; shapes replaced by {shapes}")
    return w


# ------------------------------------------------------------------ CPU oracle leg
def cpu_tile_sample(w, ntiles: int, seed: int = 7):
    """The CPU baseline's tiles: every ragged tile (an edge below max_block),
    then seeded random full tiles up to ntiles in all."""
    from oracle import shampoo4_oracle as O
    blocks = O.partition(w.shapes, w.max_block)
    ragged = [k for k, b in enumerate(blocks) if b.m < w.max_block or b.n < w.max_block]
    full = [k for k in range(len(blocks)) if k not in set(ragged)]
    rng = np.random.default_rng(seed)
    extra = list(rng.permutation(full)[:max(0, ntiles - len(ragged))]) if full else []
    return blocks, sorted(ragged[:ntiles] + [int(k) for k in extra])


def cpu_sample(w, picks, blocks, seed_step: int = 1):
    """Time the oracle on the given tiles (stats + warm refresh of both
    factors with Bjorck + precondition; a first, cold refresh is untimed).
    Returns (seconds per tile, threads)."""
    from oracle import shampoo4_oracle as O
    from bit_quantized_shampoo_b200.workloads import gradient
    grads = {}
    t_total = 0.0
    for k in picks:
        b = blocks[k]
        if b.param not in grads:
            grads[b.param] = gradient(w, b.param, seed_step)
        g = grads[b.param][b.r0:b.r0 + b.m, b.c0:b.c0 + b.n].copy()
        fl = O.Factor(b.m, np.zeros((b.m, b.m), np.float32))
        fr = O.Factor(b.n, np.zeros((b.n, b.n), np.float32))
        for f, side in ((fl, "L"), (fr, "R")):        # untimed: a first basis
            f.S = O.ema_stats(f.S, g, w.beta, side)
            O.refresh_factor(f, w.eps, w.bjorck_iters)
        t0 = time.perf_counter()
        fl.S = O.ema_stats(fl.S, g, w.beta, "L")
        fr.S = O.ema_stats(fr.S, g, w.beta, "R")
        O.refresh_factor(fl, w.eps, w.bjorck_iters)
        O.refresh_factor(fr, w.eps, w.bjorck_iters)
        O.apply_roots(O.factor_root(fl, w.eps), g, O.factor_root(fr, w.eps))
        t_total += time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    return t_total / max(1, len(picks)), threads


def cpu_rate(w, picks, blocks, seed_step=1):
    """(steps/s extrapolated from the sample's mean per-tile time, threads)."""
    tile_s, threads = cpu_sample(w, picks, blocks, seed_step)
    return 1.0 / (tile_s * len(blocks)), threads


# ------------------------------------------------------------------ ranks
def max_over_ranks(ms, device=None):
    """The job's time: every rank passes its own elapsed milliseconds and
    gets the slowest rank's.  Unchanged in a single process."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, units_per_rank, ms):
    """Whole-job throughput: every rank processed units_per_rank units (weak
    scaling, one replica of the workload per rank) in the job's time ms."""
    return world * units_per_rank / (ms / 1e3)


# ------------------------------------------------------------------ main
def run_reference(args, rank, world):
    """The oracle as the reference arm, on the host cores: each step times a
    different slice of 4 tiles of the CPU baseline's sample (every ragged
    tile plus seeded full ones), extrapolated per tile to the workload."""
    if rank != 0:
        return
    w = workload_shapes(args.workload, args.shapes)
    blocks, sample = cpu_tile_sample(w, args.cpu_tiles)
    per_step = 4
    rates = []
    threads = None
    for i in range(args.warmup + args.steps):
        picks = [sample[(per_step * i + j) % len(sample)] for j in range(min(per_step, len(sample)))]
        v, threads = cpu_rate(w, picks, blocks, seed_step=1 + i)
        if i >= args.warmup:
            rates.append(v)
    value = float(len(rates) / np.sum([1.0 / r for r in rates]))      # mean time per step
    desc = (f"each step: 4 tiles of a {len(sample)}-tile sample (all ragged tiles + seeded full ones) of "
            f"{len(blocks)}, stats + warm refresh with Bjorck of both factors + precondition; per-tile time "
            f"extrapolated to the whole workload")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "tiles": len(blocks), "steps_per_refresh": 1},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure_config(wid, dev, args, pk, pk_src, world):
    """One of the smaller workloads at its own refresh interval T: cycles of
    T steps (statistics every step, a refresh on the first step of each
    cycle, precondition every step), gradients resident in HBM, CUDA events
    on the launching stream.  Also the refresh call alone.  Every rank runs
    its own copy (no collective); times are the max over ranks."""
    import torch
    from bit_quantized_shampoo_b200 import api
    from bit_quantized_shampoo_b200.workloads import WORKLOADS, gradient
    w = WORKLOADS[wid]
    T = w.refresh_every
    shapes = list(w.shapes)
    sh = api.Shampoo4(shapes, beta=w.beta, eps=w.eps, max_block=w.max_block, bjorck_iters=w.bjorck_iters,
                      precision=args.precision, device=dev)
    sets = [[torch.from_numpy(gradient(w, i, 1 + s)).to(dev) for i in range(len(shapes))] for s in range(2)]
    out = [torch.empty(s, dtype=torch.float32, device=dev) for s in shapes]
    stream = torch.cuda.current_stream()
    t = [0]

    def step():
        g = sets[t[0] % 2]
        sh.update_stats(g)
        if t[0] % T == 0:
            sh.refresh_roots()
        sh.precondition(g, out=out)
        t[0] += 1

    for _ in range(max(3, T)):
        step()
    while t[0] % T:
        step()
    cycles = max(1, (20 + T - 1) // T) if T > 1 else 20
    torch.cuda.synchronize()
    warmup_flags = sh.status_flags()         # the cold first refresh's, cleared
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(cycles * T):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dev) / (cycles * T)
    # the refresh alone
    reps = 5
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for _ in range(reps):
        sh.refresh_roots()
    r1.record(stream)
    torch.cuda.synchronize()
    rms = max_over_ranks(r0.elapsed_time(r1), dev) / reps
    dims = [tuple(sh.block_info(k)[3:5]) for k in range(sh.nblocks)]
    res = {"workload": w.name, "tiles": sh.nblocks, "factors": sh.nfactors, "refresh_every": T,
           "steps_timed": cycles * T, "ms_per_step": ms, "us_per_step": ms * 1e3,
           "steps_per_s": world * 1e3 / ms, "refresh_ms": rms, "root_refreshes_per_s": world * sh.nfactors * 1e3 / rms,
           "status_flags": sh.status_flags(), "warmup_status_flags": warmup_flags,
           "roofline": formula_roofline(step_work(dims, w.bjorck_iters, T, args.precision), ms / 1e3, pk, pk_src,
                                        f"step at T = {T}, algorithmic flops of the work model"),
           "workspace_bytes": sh.workspace_bytes, "state_bytes": sh.state_bytes}
    del sh, sets, out
    return res


def measure_variant(wid, dev, args, pk, pk_src, world, **kw):
    """Step (refresh every step) and refresh-call times of one handle variant
    (codebook, root method) on a workload; CUDA events on the launching
    stream, max over ranks."""
    import torch
    from bit_quantized_shampoo_b200 import api
    from bit_quantized_shampoo_b200.workloads import WORKLOADS, gradient
    w = WORKLOADS[wid]
    shapes = list(w.shapes)
    sh = api.Shampoo4(shapes, beta=w.beta, eps=w.eps, max_block=w.max_block, bjorck_iters=w.bjorck_iters,
                      precision=args.precision, device=dev, **kw)
    sets = [[torch.from_numpy(gradient(w, i, 1 + s)).to(dev) for i in range(len(shapes))] for s in range(2)]
    out = [torch.empty(s, dtype=torch.float32, device=dev) for s in shapes]
    stream = torch.cuda.current_stream()

    def step(i):
        sh.update_stats(sets[i % 2])
        sh.refresh_roots()
        sh.precondition(sets[i % 2], out=out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    warmup_flags = sh.status_flags()         # the cold first refresh's, cleared
    reps = 5
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    ev[0].record(stream)
    for i in range(reps):
        step(i)
    ev[1].record(stream)
    for _ in range(reps):
        sh.refresh_roots()
    ev[2].record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev[0].elapsed_time(ev[1]), dev) / reps
    rms = max_over_ranks(ev[1].elapsed_time(ev[2]), dev) / reps
    res = {"ms_per_step": ms, "refresh_ms": rms, "root_refreshes_per_s": world * sh.nfactors * 1e3 / rms,
           "state_bytes": sh.state_bytes, "status_flags": sh.status_flags(), "warmup_status_flags": warmup_flags}
    del sh, sets, out
    return res


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist
    from bit_quantized_shampoo_b200 import api, _lib as L
    from bit_quantized_shampoo_b200.workloads import gradient
    import ctypes as C

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)

    w = workload_shapes(args.workload, args.shapes)
    shapes = list(w.shapes)
    # inputs: seeded host draws (one set per gradient step seed), copied to
    # pinned host memory and to HBM; step t uses set t mod grad_sets
    nsets = max(1, args.grad_sets)
    host_sets = [[torch.from_numpy(gradient(w, i, 1 + s)).pin_memory() for i in range(len(shapes))]
                 for s in range(nsets)]
    dev_sets = [[h.to(dev, non_blocking=False) for h in hs] for hs in host_sets]
    host_g = host_sets[0]
    dev_out = [torch.empty(s, dtype=torch.float32, device=dev) for s in shapes]
    host_out = [torch.empty(s, dtype=torch.float32).pin_memory() for s in shapes]
    shard = (not args.replicas) and world > 1
    sh = api.Shampoo4(shapes, beta=w.beta, eps=w.eps, max_block=w.max_block, bjorck_iters=w.bjorck_iters,
                      precision=args.precision, device=dev, compressed=args.compressed,
                      refresh_rank=rank if shard else 0, refresh_world=world if shard else 1)
    stream = torch.cuda.current_stream()

    counter = [0]

    refresh_ev = []                 # (start, end) CUDA events around each timed refresh

    def one_step(g, out, ev=None):
        sh.update_stats(g)
        if ev is not None:
            ev[0].record(stream)
        sh.refresh_roots()
        if ev is not None:
            ev[1].record(stream)
        if shard:
            sh.exchange_roots()
        sh.precondition(g, out=out)

    def step(timed=False):
        g = dev_sets[counter[0] % nsets]
        counter[0] += 1
        ev = None
        if timed:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            refresh_ev.append(ev)
        one_step(g, dev_out, ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # the latched flags of the warm-up (its first refresh is the cold one,
    # from U = I) are read and cleared here, so the line's status_flags
    # describe the steps after it
    warmup_flags = sh.status_flags()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("timed")
        e0.record(stream)
        for _ in range(args.steps):
            step(timed=True)
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    ms_per_step = ms / args.steps
    # replicas: every rank runs a whole step; sharded refresh: the ranks run
    # one step together
    value = args.steps / (ms / 1e3) if shard else job_rate(world, args.steps, ms)

    # per-stage times: the library's launch timing (an event pair around
    # every launch) over separate steps after the timed region, so that the
    # timed steps carry no instrumentation
    tsteps = max(1, min(3, args.steps))
    L.call("shampoo4_timing_enable", sh._h, 1)
    for _ in range(tsteps):
        step()
    torch.cuda.synchronize()
    stages = {}
    launches = 0
    s = 0
    while True:                                      # every stage the library names
        name = L.lib().shampoo4_stage_name(s).decode()
        if name == "unknown":
            break
        t_ms, n, fl, by = C.c_double(), C.c_int64(), C.c_double(), C.c_double()
        L.call("shampoo4_timing_read", sh._h, s, C.byref(t_ms), C.byref(n), C.byref(fl), C.byref(by))
        s += 1
        if n.value:
            stages[name] = {"ms": t_ms.value / tsteps, "launches": n.value // tsteps,
                            "flops": fl.value / tsteps, "bytes": by.value / tsteps}
            launches += n.value // tsteps
    L.call("shampoo4_timing_enable", sh._h, 0)
    status = sh.status_flags()

    pk, pk_src = peaks()
    clocks = clk.summary()
    g_bytes = sum(r * c for r, c in shapes) * 4
    dims = [tuple(sh.block_info(k)[3:5]) for k in range(sh.nblocks)]
    stat_bytes = sum(m * m + n * n for m, n in dims) * 4
    # headline: the whole step by the work model's formulas (refresh on every
    # step here), against the precision-weighted tensor peak
    roof = formula_roofline(step_work(dims, w.bjorck_iters, 1, args.precision), ms_per_step / 1e3, pk, pk_src,
                            "whole step (statistics + refresh + precondition), algorithmic flops of the work model")
    roof["traffic"] = None
    roof["traffic_note"] = "no single-kernel DRAM count for a whole step; per-stage GEMM traffic in rooflines_other"
    refresh_stages = ("refresh_scan", "basis", "bjorck_gram", "bjorck_update", "subspace", "qr_gram", "qr_potrf",
                      "qr_trsm_panel", "qr_syrk", "qr_solve_update", "qr_solve_panel", "qr_convert", "qr_inverse",
                      "rayleigh_gemm", "rayleigh", "requant")
    # the refresh call itself, between CUDA events on the caller's stream
    # (its parts run concurrently on the handle's streams, so summed stage
    # times would overstate it)
    refresh_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in refresh_ev), dev) / args.steps
    stage_sum = sum(stages[k]["ms"] for k in refresh_stages if k in stages)
    others = [formula_roofline(refresh_work(dims, w.bjorck_iters, args.precision), refresh_ms / 1e3, pk, pk_src,
                               "refresh of every factor (a3-a8), algorithmic flops of the work model; time = the "
                               "refresh call between CUDA events on the caller's stream")]
    # per stage: the flops each launch's descriptors carry (the implementation's
    # products, which exceed the work model's count for the QR)
    ranked = sorted(stages, key=lambda k: -stages[k]["ms"])
    for k in ranked[:8]:
        r = stage_roofline(k, stages[k], pk, pk_src)
        t = stage_traffic(k, sum(m * m + n * n for m, n in dims))
        if t is not None:
            r["traffic"] = t
        r["flops_note"] = "implementation flops of the stage's launches (not the work model's count)"
        others.append(r)

    line = {"metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if shard else "weak",
            "vs_baseline": None, "dtype": args.precision if args.precision == "fp32" else "tf32",
            "data": "synthetic",
            "config": {"workload": w.name, "tiles": sh.nblocks, "factors": sh.nfactors,
                       "steps_per_refresh": 1,
                       "refresh_ms_per_step": refresh_ms,
                       "refresh_stage_busy_ms": stage_sum,
                       "statistics": "compressed (4-bit eigenbasis + eigenvalues)" if args.compressed else "fp32",
                       "parallelism": (f"refresh sharded over {world} ranks + NCCL span broadcasts" if shard
                                       else f"{world} independent replica(s)"),
                       "state_bytes": sh.state_bytes, "workspace_bytes": sh.workspace_bytes,
                       "gradients": f"{nsets} seeded set(s), step t uses set t mod {nsets}",
                       "l2": (f"inputs larger than L2 ({g_bytes / 1e9:.2f} GB of G, {stat_bytes / 1e9:.2f} GB "
                              f"of fp32 statistics; L2 is 0.126 GB)")},
            "root_refreshes_per_s": value * sh.nfactors,
            "status_flags": status, "warmup_status_flags": warmup_flags,
            "gpu_launches": launches * args.steps,
            "clocks": clocks, "roofline": roof, "rooflines_other": others,
            "stages_ms": {k: round(v["ms"], 4) for k, v in sorted(stages.items(), key=lambda kv: -kv[1]["ms"])},
            "stages_note": f"launch durations per step over {tsteps} step(s) after the timed region"}

    # the same refresh split into two cost-balanced parts on the handle's
    # two streams (the default is one launch sequence)
    if not shard:
        L.call("shampoo4_debug_refresh_parts", sh._h, 2)
        sh.bind(reset=False)
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(3):
            sh.refresh_roots()
        r1.record(stream)
        torch.cuda.synchronize()
        line["config"]["refresh_ms_two_parts"] = r0.elapsed_time(r1) / 3
        L.call("shampoo4_debug_refresh_parts", sh._h, 1)
        sh.bind(reset=False)

    # end to end through the public API with host buffers: every step copies
    # its gradients in from pinned host memory and its update out to pinned
    # host memory.  The copies run on a second stream, double-buffered, so
    # step t+1's gradients load and step t's update drains while the GPU
    # computes (the first load and the last drain are exposed).
    if not args.no_e2e:
        torch.cuda.synchronize()
        k = max(2, args.steps)
        copy_s = torch.cuda.Stream(device=dev)
        gbuf = [dev_sets[0], dev_sets[1] if nsets > 1 else [torch.empty_like(x) for x in dev_sets[0]]]
        obuf = [dev_out, [torch.empty_like(x) for x in dev_out]]
        hout = [host_out, [torch.empty(s, dtype=torch.float32).pin_memory() for s in shapes]]
        loaded = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def load(i):
            slot = i % 2
            if i >= 2:
                copy_s.wait_event(done[slot])              # step i-2 has finished reading this slot
            with torch.cuda.stream(copy_s):
                for h, d in zip(host_sets[i % nsets], gbuf[slot]):
                    d.copy_(h, non_blocking=True)
            loaded[slot].record(copy_s)

        e2.record(stream)
        copy_s.wait_event(e2)
        load(0)
        for i in range(k):
            slot = i % 2
            stream.wait_event(loaded[slot])
            g = gbuf[slot]
            one_step(g, obuf[slot])
            done[slot].record(stream)
            if i + 1 < k:
                load(i + 1)
            copy_s.wait_event(done[slot])
            with torch.cuda.stream(copy_s):
                for d, h in zip(obuf[slot], hout[slot]):
                    h.copy_(d, non_blocking=True)
        stream.wait_stream(copy_s)
        e3.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e2.elapsed_time(e3), dev)
        bi = sum(h.numel() * 4 for h in host_g)
        bo = sum(h.numel() * 4 for h in host_out)
        line["e2e"] = {"value": k / (ems / 1e3) if shard else job_rate(world, k, ems), "unit": "steps/s", "steps": k,
                       "h2d_bytes_per_step": bi,
                       "d2h_bytes_per_step": bo,
                       "copies": "pinned host buffers, second stream, double-buffered (overlapped with compute)"}
        del gbuf, obuf, hout

    # the same steps captured once in a CUDA graph (two steps, one per gradient
    # buffer) and replayed: launch gaps and host work leave the step
    if not args.no_graph and not shard:
        torch.cuda.synchronize()
        side = torch.cuda.Stream(device=dev)
        graph = torch.cuda.CUDAGraph()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            # thread-local capture: another thread's CUDA calls (a process
            # group's watchdog, say) do not disturb it
            with torch.cuda.graph(graph, stream=side, capture_error_mode="thread_local"):
                for i in range(2):
                    one_step(dev_sets[i % nsets], dev_out)
        stream.wait_stream(side)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        reps = max(1, args.steps // 2)
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e4.record(stream)
        for _ in range(reps):
            graph.replay()
        e5.record(stream)
        torch.cuda.synchronize()
        gms = max_over_ranks(e4.elapsed_time(e5), dev)
        line["graph"] = {"value": job_rate(world, 2 * reps, gms), "unit": "steps/s", "steps": 2 * reps,
                         "ms_per_step": gms / (2 * reps),
                         "note": "the timed steps captured once in a CUDA graph and replayed"}
        del graph

    # stand-alone codec bandwidth on eigenvector-shaped tensors of the workload's size
    if not args.no_codec:
        n_elem = sum(int(b[3]) ** 2 + int(b[4]) ** 2 for b in (sh.block_info(k) for k in range(sh.nblocks)))
        g = torch.Generator(device=dev).manual_seed(3)
        x = torch.randn(n_elem, device=dev, generator=g) * (1.0 / 32)
        codes = torch.empty((n_elem + 1) // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty((n_elem + 63) // 64, dtype=torch.float32, device=dev)
        y = torch.empty_like(x)
        for _ in range(3):
            api.quant4_pack([x], [codes], [scales])
            api.quant4_unpack([codes], [scales], [n_elem], [y])
        torch.cuda.synchronize()
        reps = 5
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        for _ in range(reps):
            api.quant4_pack([x], [codes], [scales])
        ev[1].record(stream)
        for _ in range(reps):
            api.quant4_unpack([codes], [scales], [n_elem], [y])
        ev[2].record(stream)
        torch.cuda.synchronize()
        bpe = 4.0 + 0.5 + 4.0 / 64
        pack_gbs = bpe * n_elem * reps / (ev[0].elapsed_time(ev[1]) / 1e3) / 1e9
        unpack_gbs = bpe * n_elem * reps / (ev[1].elapsed_time(ev[2]) / 1e3) / 1e9
        line["codec"] = {"elements": n_elem, "pack_gbs": pack_gbs, "unpack_gbs": unpack_gbs,
                         "pack_frac": pack_gbs / pk["hbm_gbs"], "unpack_frac": unpack_gbs / pk["hbm_gbs"],
                         "peak_gbs": pk["hbm_gbs"], "peak_source": pk_src}
        del x, y, codes, scales

    # stand-alone grafted weight update (Adam graft) over the workload's parameters,
    # fed this step's gradients and directions
    if not args.no_graft:
        gen = torch.Generator(device=dev).manual_seed(5)
        weights = [torch.randn(s, device=dev, generator=gen) * 0.02 for s in shapes]
        gstate = sh.graft_state("adam")
        g = dev_sets[0]
        t = [0]

        # dev_out is the last precondition's output, unmodified: the update
        # may take ||D|| as that call's apply recorded it (D read once)
        def graft(dir_norms):
            t[0] += 1
            sh.graft_update(gstate, t[0], 1e-3, g, dev_out, weights, kind="adam", dir_norms=dir_norms)

        def time_graft(dir_norms):
            for _ in range(3):
                graft(dir_norms)
            torch.cuda.synchronize()
            reps = 5
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            for _ in range(reps):
                graft(dir_norms)
            ev[1].record(stream)
            torch.cuda.synchronize()
            return ev[0].elapsed_time(ev[1]) / reps

        n_elem = sum(r * c for r, c in shapes)
        bpe = 32.0          # read G, D, W, m, v; write W, m, v (fp32)
        gms = time_graft(True)
        gbs = bpe * n_elem / (gms / 1e3) / 1e9
        line["graft"] = {"kind": "adam", "elements": n_elem, "ms": gms, "launches": 2, "bound": "hbm",
                         "bytes_per_element": bpe, "issued_bytes_per_element": 32.0,
                         "dir_norms": "recorded by the precondition's apply (D read once)",
                         "gbs": gbs, "frac": gbs / pk["hbm_gbs"], "peak_gbs": pk["hbm_gbs"], "peak_source": pk_src,
                         "status_flags": sh.status_flags()}
        gms2 = time_graft(False)
        line["graft"]["reading_d_twice"] = {"ms": gms2, "issued_bytes_per_element": 36.0,
                                           "frac": bpe * n_elem / (gms2 / 1e3) / 1e9 / pk["hbm_gbs"]}
        del weights, gstate

    # bounded workspace layouts of the same step: 48 and 16 tiles per group
    # (the default here is one group, the largest workspace and the fastest)
    layouts_ok = not args.no_configs and args.shapes is None and args.workload == 5 and not shard
    if layouts_ok:
        del sh
        torch.cuda.empty_cache()
        line["layouts"] = {}
        for name, gt in (("48_tiles_per_group", 48), ("16_tiles_per_group", 16)):
            lay = api.Shampoo4(shapes, beta=w.beta, eps=w.eps, max_block=w.max_block, bjorck_iters=w.bjorck_iters,
                               precision=args.precision, device=dev, group_tiles=gt)
            for i in range(3):
                lay.update_stats(dev_sets[i % nsets]); lay.refresh_roots(); lay.precondition(dev_sets[i % nsets], out=dev_out)
            torch.cuda.synchronize()
            l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            l0.record(stream)
            for i in range(3):
                lay.update_stats(dev_sets[i % nsets]); lay.refresh_roots(); lay.precondition(dev_sets[i % nsets], out=dev_out)
            l1.record(stream)
            torch.cuda.synchronize()
            line["layouts"][name] = {"group_tiles": gt, "workspace_bytes": lay.workspace_bytes,
                                     "ms_per_step": max_over_ranks(l0.elapsed_time(l1), dev) / 3}
            del lay
            torch.cuda.empty_cache()

    # the four smaller workloads, each at its own refresh interval
    if not args.no_configs and args.shapes is None and args.workload == 5:
        if not layouts_ok:
            del sh
        torch.cuda.empty_cache()
        line["configs"] = {}
        for wid in (1, 2, 3, 4):
            line["configs"][f"c{wid}"] = measure_config(wid, dev, args, pk, pk_src, world)
            torch.cuda.empty_cache()

    # the alternatives the 4-bit Shampoo abstract compares against, on the
    # transformer layer stack with a refresh every step
    if not args.no_variants and args.shapes is None and args.workload == 5:
        torch.cuda.empty_cache()
        line["variants"] = {"workload": "transformer stack, 12 blocks of d=768, refresh every step"}
        for name, kw in (("eigen_linear_square", {}), ("eigen_dynamic_tree", {"codebook": "dynamic_tree"}),
                         ("newton_fp32_root", {"root": "newton"}), ("newton_4bit_root", {"root": "newton_q4"})):
            line["variants"][name] = measure_variant(4, dev, args, pk, pk_src, world, **kw)
            torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu:
        blocks, sample = cpu_tile_sample(w, args.cpu_tiles)
        v, threads = cpu_rate(w, sample, blocks)
        nrag = sum(1 for k in sample if blocks[k].m < w.max_block or blocks[k].n < w.max_block)
        line["cpu_baseline"] = {"value": v, "unit": "steps/s", "cores": threads, "kind": "oracle",
                                "sample": (f"{len(sample)} of {len(blocks)} tiles ({nrag} ragged + "
                                           f"{len(sample) - nrag} seeded full ones): stats + warm refresh with "
                                           f"Bjorck of both factors + precondition; mean per-tile time extrapolated "
                                           f"to the whole workload (extrapolated)")}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
