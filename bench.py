"""Benchmark: W4A16 decode-sweep GEMV on B200 (plus the other hot-path rows as extras).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B] [--impl ours|reference]

Headline workload: the decode sweep of a synthetic Llama-style 1B stack (hidden 2048,
intermediate 5632, 24 layers x 7 projections = 168 dyadic g64 matrices, 1,056,964,608
weights), batch B bf16 N(0,1) activations. One step = one W4A16 GEMV over all 168 packed
matrices (one grouped launch), inputs resident in HBM. The packed weights (535 MB) are
larger than L2 (126 MB), so every step streams them from HBM; no flush is needed.

value = effective weight bytes (packed nibbles + bf16 scales) streamed per second, GB/s.
Multi-GPU: replicas only (the sweep has no exchange step); every rank runs the same
sweep on its own GPU, time = max over ranks, value = all ranks' bytes / that time.
--impl reference times the fp64 CPU oracle on host cores on a bounded sample instead.
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
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "W4A16 GEMV effective weight GB/s (% HBM peak); GEMM TFLOP/s; quantize Gweights/s"
UNIT = "GB/s"
# DRAM bytes (read + write) of one launch of the headline kernel at batch 1, from an ncu
# capture of the current kernel (a steady-state launch: 563,201,536 read + 524,032 written)
HEADLINE_TRAFFIC = 563725568
# timed regions of the headline (each exactly --steps steps); the median is reported
REGIONS = 10


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    sm_max_mhz=float(d.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------------------

def sweep_host_weights(threads: int = 8):
    mats = workloads.sweep_matrices()
    with ThreadPoolExecutor(threads) as ex:
        ws = list(ex.map(lambda m: workloads.gaussian_outlier_weight(m[2], m[3], workloads.DECODE_SWEEP, m[4]), mats))
    return mats, ws


def build_sweep(wq, torch, dev, batch):
    mats, host_w = sweep_host_weights()
    packed = []
    for (layer, name, n, k, idx), wb in zip(mats, host_w):
        w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(dev)
        pw, _ = wq.quantize_dyadic(w, 64)
        packed.append(pw)
        del w
    xs_host = [workloads.activations(batch, k, workloads.DECODE_SWEEP, idx) for _, _, _, k, idx in mats]
    # every x (and y) is a view into one flat buffer, so that a step's inputs arrive in one
    # host-to-device copy and its outputs leave in one (each view starts 64-byte aligned:
    # batch * k * 2 bytes with k a multiple of 32)
    xflat = torch.from_numpy(np.concatenate([x.reshape(-1) for x in xs_host]).view(np.int16)).view(torch.bfloat16).to(dev)
    yflat = torch.empty(sum(batch * n for _, _, n, _, _ in mats), dtype=torch.bfloat16, device=dev)
    xs, ys, xo, yo = [], [], 0, 0
    for _, _, n, k, _ in mats:
        xs.append(xflat[xo:xo + batch * k].view(batch, k))
        ys.append(yflat[yo:yo + batch * n].view(batch, n))
        xo += batch * k
        yo += batch * n
    torch.cuda.synchronize(dev)
    return mats, packed, xs_host, xs, ys, xflat, yflat


def sweep_bytes(mats, batch):
    packed = sum(n * k // 2 for _, _, n, k, _ in mats)
    scale = sum(n * (k // 64) * 2 for _, _, n, k, _ in mats)
    xb = sum(batch * k * 2 for _, _, _, k, _ in mats)
    yb = sum(batch * n * 2 for _, _, n, _, _ in mats)
    return packed, scale, xb, yb


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------

class nvtx_range:
    """An NVTX range around one bench phase (visible in nsys/ncu timelines)."""

    def __init__(self, torch, name: str):
        self.torch, self.name = torch, name

    def __enter__(self):
        self.torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        self.torch.cuda.nvtx.range_pop()
        return False


def graph_of(torch, fn):
    """fn's launches captured once in a CUDA graph (after one eager call for any one-time
    setup); replaying it keeps per-call host work (argument checks, allocation) out of a
    timed region that is meant to hold the kernels."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_region(torch, stream, fn, steps, warmup, barrier):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        fn()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return t0.elapsed_time(t1) / steps


def max_over_ranks_fn(torch, dist, world: int, device):
    """The timing reduction every multi-GPU number goes through: the max of a per-rank value
    over all ranks (an all-reduce on `device`: the GPU under NCCL, the CPU under gloo)."""
    def reduce(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return reduce


def replica_value(world: int, bytes_per_rank: int, max_ms: float) -> float:
    """Weak scaling over independent replicas: every rank streams the same per-rank bytes, and
    the whole job's rate is all ranks' bytes over the slowest rank's time (GB/s)."""
    return world * bytes_per_rank / (max_ms * 1e-3) / 1e9


def run_ours(args):
    import torch
    import torch.distributed as dist
    import __graft_entry__
    __graft_entry__._build_module().build()
    import w4a16_matmul_b200 as wq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    max_over_ranks = max_over_ranks_fn(torch, dist, world, dev)

    B = args.batch
    mats, packed, xs_host, xs, ys, xflat, yflat = build_sweep(wq, torch, dev, B)
    stream = torch.cuda.current_stream(dev)
    # the decode loop's prepared launch; consecutive steps overlap the next launch's start
    # (weight loads) with the previous one's last wave (wq_gemv_plan_set_overlap: the weights
    # are constant, the activations and outputs wait for the previous kernel)
    run = wq.GroupedGemv(packed, xs, ys, overlap=True)
    pk_b, sc_b, x_b, y_b = sweep_bytes(mats, B)
    weight_bytes = pk_b + sc_b
    algo_bytes = pk_b + sc_b + x_b + y_b

    clocks = ClockSampler(local)
    # ---- headline: device-resident, one grouped launch per step. The K steps of a timed
    # region are K launches of the prepared plan captured back to back in one CUDA graph
    # (the decode loop's form: consecutive launches overlap the next one's start with the
    # previous one's last wave, and no host work sits between them); a region is one replay.
    # The region is timed REGIONS times (each exactly K steps between barriers and
    # synchronisations) and the median gives ms_per_step, so that a 1 % difference stands
    # above run-to-run noise. -------------------------------------------------------------
    run()                                    # first call (one-time setup)
    torch.cuda.synchronize()
    g_steps = graph_of(torch, lambda: [run() for _ in range(args.steps)])
    g_warm = graph_of(torch, lambda: [run() for _ in range(args.warmup)])
    regions = REGIONS
    g_warm.replay()
    clocks.start()
    with nvtx_range(torch, "headline: decode sweep GEMV"):
        region_ms = [time_region(torch, stream, g_steps.replay, 1, 0, barrier) / args.steps
                     for _ in range(regions)]
    clk = clocks.stop()
    ms = max_over_ranks(float(np.median(region_ms)))
    value = replica_value(world, weight_bytes, ms)
    achieved = algo_bytes / (ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers ---------------------------
    # Every step copies its activations in from pinned host memory and its outputs back
    # out, inside the timed region. The steps are independent batches, so two device buffer
    # sets (one prepared plan each) let step i + 1's copy-in and step i - 1's copy-out run
    # beside step i's kernel: a copy-in stream, the compute stream and a copy-out stream,
    # ordered by events (a buffer set is refilled only after its kernel has read it, and its
    # outputs are overwritten only after they have been copied out).
    x_pin = xflat.cpu().pin_memory()
    y_pins = [torch.empty(yflat.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xflat2, yflat2 = torch.empty_like(xflat), torch.empty_like(yflat)
    xs2, ys2, xo, yo = [], [], 0, 0
    for _, _, n, k, _ in mats:
        xs2.append(xflat2[xo:xo + B * k].view(B, k))
        ys2.append(yflat2[yo:yo + B * n].view(B, n))
        xo += B * k
        yo += B * n
    runs = [run, wq.GroupedGemv(packed, xs2, ys2, overlap=True)]
    xbufs, ybufs = [xflat, xflat2], [yflat, yflat2]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_steps(nsteps):
        comp, out = [None, None], [None, None]
        for i in range(nsteps):
            b = i % 2
            with torch.cuda.stream(s_in):
                if comp[b] is not None:
                    s_in.wait_event(comp[b])            # its kernel has read this buffer set
                xbufs[b].copy_(x_pin, non_blocking=True)    # this step's activations in
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            stream.wait_event(e_in)
            if out[b] is not None:
                stream.wait_event(out[b])               # its last outputs have left
            runs[b]()                                   # the public API call (prepared plan)
            comp[b] = torch.cuda.Event()
            comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp[b])
                y_pins[b].copy_(ybufs[b], non_blocking=True)   # this step's outputs out
                out[b] = torch.cuda.Event()
                out[b].record(s_out)
        return [e for e in out if e is not None]

    e2e_steps(max(args.warmup, 2))
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    s_in.wait_stream(stream)
    with nvtx_range(torch, "e2e: host copies + decode sweep GEMV"):
        for e in e2e_steps(args.steps):
            stream.wait_event(e)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    e2e = {"value": round(replica_value(world, weight_bytes, ms_e2e), 2), "unit": UNIT,
           "h2d_bytes_per_step": x_b, "d2h_bytes_per_step": y_b, "ms_per_step": round(ms_e2e, 4),
           "pipelining": "2 buffer sets: copy-in of step i+1 and copy-out of step i-1 beside step i's kernel"}

    extras = {}
    if not args.no_extras:
        with nvtx_range(torch, "extras"):
            extras = run_extras(args, wq, torch, dev, stream, packed, mats, xs, ys, peaks, barrier,
                                max_over_ranks)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u4+bf16->f32",
        "data": "synthetic (seeded numpy PCG64, pages' value distributions)",
        "config": {"workload": "decode sweep: 24 layers x {q,k,v,o,gate,up,down} dyadic g64, "
                               "hidden 2048, intermediate 5632, 1,056,964,608 weights",
                   "batch": B, "matrices": len(mats),
                   "launch": "one grouped GEMV launch per step (prepared plan; the region's steps "
                             "captured back to back in one CUDA graph, consecutive launches "
                             "overlapped by programmatic dependent launch)",
                   "timed_regions": {"count": regions, "statistic": "median of regions of exactly "
                                     f"{args.steps} steps", "min_ms_per_step": round(min(region_ms), 5),
                                     "max_ms_per_step": round(max(region_ms), 5)},
                   "weight_bytes_per_step": weight_bytes, "l2": "inputs larger than L2 (535 MB/step)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     # dram__bytes_read.sum + dram__bytes_write.sum of one launch of this
                     # kernel at batch 1, from an ncu capture of the current kernel
                     "traffic": HEADLINE_TRAFFIC if B == 1 else None, "peak_source": peaks["source"],
                     "algorithmic_bytes_per_launch": algo_bytes, "kernel": "gemv_kernel (grouped)",
                     # the same time against other byte counts and peaks
                     "frac_weight_bytes": round(weight_bytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "frac_packed_only": round(pk_b / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "frac_weight_bytes_of_nominal_8000": round(weight_bytes / (ms * 1e-3) / 1e9 / 8000.0, 4),
                     "target_0.75_judged_on": "frac (algorithmic bytes: packed + scales + x + y, "
                                              "measured copy peak)"},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk,
        "extras": extras,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args, mats, seconds=args.cpu_seconds)
    # last on the line, so that a reader of only its tail still sees every row's headline
    line["rows"] = summarize(extras, line)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def summarize(extras: dict, line: dict) -> dict:
    """One short entry per row of the hot path (fractions of the measured peaks; GEMM in
    TFLOP/s with the dequantise + cuBLAS bf16 line beside it), from the full results."""
    def get(d, *path):
        for p in path:
            if not isinstance(d, dict) or p not in d:
                return None
            d = d[p]
        return d
    r = {"headline_frac": line["roofline"]["frac"], "headline_frac_packed_only": line["roofline"]["frac_packed_only"],
         "sweep_b4_frac": get(extras, "sweep_batch4", "frac_hbm"),
         "sweep_b16_frac": get(extras, "sweep_batch16", "frac_hbm"),
         "single_2048_us": [get(extras, "single_matrix_2048", k, "us") for k in ("quantize_pack", "dequant", "gemv_b1")],
         "quantize_8192x28672_frac": get(extras, "quantize_dyadic_large", "frac_hbm"),
         "dequant_8192x28672_frac": get(extras, "dequant_large", "frac_hbm")}
    g = extras.get("prefill_gemm", {})
    for shape in ("4096x11008", "11008x4096"):
        r[f"gemm_{shape}_TFLOPs_m16_128_512_2048_4096"] = [get(g, f"{shape}_m{m}", "TFLOP/s") for m in (16, 128, 512, 2048, 4096)]
        r[f"cublas_{shape}_TFLOPs"] = [get(g, f"{shape}_m{m}", "cublas_bf16_materialized_TFLOP/s")
                                       for m in (16, 128, 512, 2048, 4096)]
    r["gemm_lloyd8s_lut16_TFLOPs_m512_4096"] = [get(g, f"{f}_4096x11008_m{m}", "TFLOP/s")
                                                for f in ("lloyd8s", "lut16") for m in (512, 4096)]
    r["lut16_gemv_frac_b1_8_16"] = [get(extras, f"lut16_gemv_b{b}", "frac_hbm") for b in (1, 8, 16)]
    r["lloyd8s_gemv_frac_b1"] = get(extras, "lloyd8s_gemv_b1", "frac_hbm")
    r["wf_gemv_frac_b1_2_4_16"] = [get(extras, "water_filling_large", f"gemv_b{b}", "frac_hbm") for b in (1, 2, 4, 16)]
    r["lloyd_g32_ms_per_matrix"] = get(extras, "lloyd_g32", "ms_per_matrix")
    r["lloyd_g32_xu_frac"] = get(extras, "lloyd_g32", "roofline", "frac")
    r["kmeans16_ms"] = get(extras, "kmeans16", "ms")
    r["ste_frac"] = get(extras, "fake_quant_ste_large", "frac_hbm")
    r["bf16x_frac_enc_dec"] = [get(extras, "bf16x_large", "encode_frac_hbm"), get(extras, "bf16x_large", "decode_frac_hbm")]
    return r


def run_extras(args, wq, torch, dev, stream, packed, mats, xs, ys, peaks, barrier, max_over_ranks):
    """Secondary rows of the hot path, each on its own workload, timed the same way."""
    out = {}
    steps, warm = max(args.steps, 5), max(args.warmup, 3)
    # the headline's launch in other launch modes, each timed over the same number of steps:
    # one graph replay per step without overlap (the gap between graph launches stays),
    # eager launches without overlap, and ten overlapped launches per graph replay
    try:
        pk, sc, xb, yb = sweep_bytes(mats, args.batch)
        modes = {}
        plain = wq.GroupedGemv(packed, xs, ys)
        g1 = graph_of(torch, plain)
        modes["graph_replay_per_step"] = max_over_ranks(time_region(torch, stream, g1.replay, steps, warm, barrier))
        modes["eager_no_overlap"] = max_over_ranks(time_region(torch, stream, plain, steps, warm, barrier))
        over = wq.GroupedGemv(packed, xs, ys, overlap=True)
        modes["eager_overlapped"] = max_over_ranks(time_region(torch, stream, over, steps, warm, barrier))
        g10 = graph_of(torch, lambda: [over() for _ in range(10)])
        reps = max(steps // 10, 3)
        modes["graph_10_overlapped_per_replay"] = max_over_ranks(
            time_region(torch, stream, g10.replay, reps, 3, barrier)) / 10
        out["headline_launch_modes"] = {
            k: {"ms_per_step": round(v, 5),
                "frac_hbm_algorithmic": round((pk + sc + xb + yb) / v / 1e6 / peaks["hbm_gbs"], 4)}
            for k, v in modes.items()}
        del g1, g10
        plain.close()
        over.close()
    except Exception as e:  # report, never hide
        out["headline_launch_modes"] = {"error": repr(e)[:200]}
    # BASELINE's single-matrix workload: one seeded 2048 x 2048 weight (N(0, 0.02^2), 0.1 %
    # outliers x 20), dyadic g64: quantize + pack, dequant and the GEMV with one activation
    # vector. One matrix is 8 MiB of bf16 (2.1 MB packed), far below L2, so every launch
    # reads its own copy from a rotation of copies that spans more than 4 x L2: each
    # launch's inputs come from HBM. One launch per copy, all copies in one CUDA graph.
    try:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        n1 = k1 = 2048
        hw = workloads.gaussian_outlier_weight(n1, k1, workloads.DYADIC_1, 0)
        w1 = torch.from_numpy(hw.view(np.int16)).view(torch.bfloat16).to(dev)
        x1 = torch.from_numpy(workloads.activations(1, k1, workloads.DYADIC_1, 0).view(np.int16)).view(
            torch.bfloat16).to(dev)
        cq = int(np.ceil(4 * l2 / (n1 * k1 * 2)))               # bf16 copies for the quantizer
        wcopies = [w1.clone() for _ in range(cq)]
        pw1, _ = wq.quantize_dyadic(w1, 64)
        per_q = n1 * k1 // 2 + n1 * (k1 // 64) * 2
        cp = int(np.ceil(4 * l2 / per_q))                        # packed copies for dequant / GEMV
        pcopies = [wq.PackedWeight(wq.FMT_DYADIC4, 64, n1, k1, pw1.packed.clone(), pw1.aux.clone())
                   for _ in range(cp)]
        sco = [torch.empty((n1, k1 // 64), dtype=torch.bfloat16, device=dev) for _ in range(cq)]
        pko = [torch.empty((n1, k1 // 2), dtype=torch.uint8, device=dev) for _ in range(cq)]
        dqo = torch.empty((n1, k1), dtype=torch.bfloat16, device=dev)
        y1 = torch.empty((1, n1), dtype=torch.bfloat16, device=dev)

        def q_all():
            for w, so, po in zip(wcopies, sco, pko):
                wq._check(wq._lib.wq_quantize_dyadic(wq._ptr(w), n1, k1, 64, wq._ptr(so), None, wq._ptr(po),
                                                     wq._stream(w)))
        gq1 = graph_of(torch, q_all)
        ms_q = max_over_ranks(time_region(torch, stream, gq1.replay, steps, warm, barrier)) / cq
        gd1 = graph_of(torch, lambda: [wq.dequant(p, out=dqo) for p in pcopies])
        ms_d = max_over_ranks(time_region(torch, stream, gd1.replay, steps, warm, barrier)) / cp
        gv1 = graph_of(torch, lambda: [wq.gemv(p, x1, out=y1) for p in pcopies])
        ms_v = max_over_ranks(time_region(torch, stream, gv1.replay, steps, warm, barrier)) / cp
        nw = n1 * k1
        qb, db, vb = nw * 2 + per_q, per_q + nw * 2, per_q + 2 * (k1 + n1)
        out["single_matrix_2048"] = {
            "workload": "one 2048x2048 weight N(0,0.02^2) + 0.1% x20, dyadic g64; x: 1 x 2048 N(0,1)",
            "l2": f"{cq} bf16 / {cp} packed copies rotated (> 4 x L2 each), one launch per copy",
            "quantize_pack": {"us": round(ms_q * 1e3, 2), "Gweights/s": round(nw / ms_q / 1e6, 1),
                              "GB/s": round(qb / ms_q / 1e6, 1), "frac_hbm": round(qb / ms_q / 1e6 / peaks["hbm_gbs"], 4)},
            "dequant": {"us": round(ms_d * 1e3, 2), "GB/s": round(db / ms_d / 1e6, 1),
                        "frac_hbm": round(db / ms_d / 1e6 / peaks["hbm_gbs"], 4)},
            "gemv_b1": {"us": round(ms_v * 1e3, 2), "GB/s": round(vb / ms_v / 1e6, 1),
                        "frac_hbm": round(vb / ms_v / 1e6 / peaks["hbm_gbs"], 4)},
            "note": "2 MB per launch: launch latency, not bandwidth, bounds a single matrix"}
        del gq1, gd1, gv1, wcopies, pcopies, sco, pko
    except Exception as e:  # report, never hide
        out["single_matrix_2048"] = {"error": repr(e)[:200]}
    # decode sweep as 168 dependent-order launches captured in one CUDA graph
    try:
        g = torch.cuda.CUDAGraph()
        s2 = torch.cuda.Stream(dev)
        s2.wait_stream(stream)
        with torch.cuda.stream(s2):
            for pw, x, y in zip(packed, xs, ys):      # warm the path before capture
                wq.gemv(pw, x, out=y)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s2):
            for pw, x, y in zip(packed, xs, ys):
                wq.gemv(pw, x, out=y)
        ms = max_over_ranks(time_region(torch, stream, g.replay, steps, warm, barrier))
        pk, sc, _, _ = sweep_bytes(mats, args.batch)
        out["sweep_chain_graph"] = {"ms_per_step": round(ms, 4), "GB/s": round((pk + sc) / ms / 1e6, 1),
                                    "launches_per_step": len(mats)}
        del g
    except Exception as e:  # report, never hide
        out["sweep_chain_graph"] = {"error": repr(e)[:200]}
    # other batch sizes of the grouped sweep
    for b in (4, 16):
        if b == args.batch:
            continue
        xs_b = [torch.randn((b, x.shape[1]), device=dev).to(torch.bfloat16) for x in xs]
        ys_b = [torch.empty((b, y.shape[1]), dtype=torch.bfloat16, device=dev) for y in ys]
        run_b = wq.GroupedGemv(packed, xs_b, ys_b)
        ms = max_over_ranks(time_region(torch, stream, run_b, steps, warm, barrier))
        pk, sc, xb, yb = sweep_bytes(mats, b)
        out[f"sweep_batch{b}"] = {"ms_per_step": round(ms, 4), "GB/s": round((pk + sc) / ms / 1e6, 1),
                                  "frac_hbm": round((pk + sc + xb + yb) / ms / 1e6 / peaks["hbm_gbs"], 4)}
    # dyadic quantisation of one layer (bf16 -> scale + packed), HBM-bound: the seeded
    # weights of the sweep's first layer
    try:
        layer = mats[:7]
        n_w = sum(n * k for _, _, n, k, _ in layer)
        wts = [torch.from_numpy(workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, idx).view(np.int16))
               .view(torch.bfloat16).to(dev) for _, _, n, k, idx in layer]

        def q():
            for w in wts:
                wq.quantize_dyadic(w, 64)

        gq = graph_of(torch, q)
        ms = max_over_ranks(time_region(torch, stream, gq.replay, steps, warm, barrier))
        byts = n_w * (2 + 0.5 + 2 / 64)
        out["quantize_dyadic_layer"] = {"Gweights/s": round(n_w / ms / 1e6, 2), "GB/s": round(byts / ms / 1e6, 1),
                                        "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4),
                                        "launches_per_step": 7}

        def dq():
            for pw in packed[:7]:
                wq.dequant(pw)
        gdq = graph_of(torch, dq)
        ms = max_over_ranks(time_region(torch, stream, gdq.replay, steps, warm, barrier))
        byts = n_w * (0.5 + 2 / 64 + 2)
        out["dequant_layer"] = {"GB/s": round(byts / ms / 1e6, 1),
                                "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4)}
        del wts, gq, gdq
        # the same two kernels on one large matrix (the 8192 x 28672 weight of the LUT16
        # workload, N(0, 0.02^2) here): one launch streams ~0.6 GB, so the number is the
        # kernel's own bandwidth rather than launch gaps between small matrices
        n_l, k_l = workloads.LUT16_SHAPE
        wl = (torch.randn((n_l, k_l), device=dev) * 0.02).to(torch.bfloat16)
        hold = {}

        def ql():
            hold["pw"], _ = wq.quantize_dyadic(wl, 64)
        gql = graph_of(torch, ql)
        ms = max_over_ranks(time_region(torch, stream, gql.replay, steps, warm, barrier))
        nw = n_l * k_l
        byts = nw * (2 + 0.5 + 2 / 64)
        out["quantize_dyadic_large"] = {"shape": [n_l, k_l], "Gweights/s": round(nw / ms / 1e6, 2),
                                        "GB/s": round(byts / ms / 1e6, 1),
                                        "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4), "us": round(ms * 1e3, 1)}
        pwl = hold["pw"]
        del wl
        dl = torch.empty((n_l, k_l), dtype=torch.bfloat16, device=dev)
        gdl = graph_of(torch, lambda: wq.dequant(pwl, out=dl))
        ms = max_over_ranks(time_region(torch, stream, gdl.replay, steps, warm, barrier))
        byts = nw * (0.5 + 2 / 64 + 2)
        out["dequant_large"] = {"shape": [n_l, k_l], "GB/s": round(byts / ms / 1e6, 1),
                                "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4), "us": round(ms * 1e3, 1)}
        del gql, gdl, dl, pwl, hold
        # STE fake quantisation forward on an fp32 latent of the same shape (4 B in, 4 B out
        # plus 0.5 B of packed codes per element)
        zl = torch.randn((n_l, k_l), device=dev).mul_(0.02)
        scl = (zl.abs().reshape(n_l, k_l // 64, 64).amax(-1)).to(torch.bfloat16)
        qo = torch.empty_like(zl)
        po = torch.empty((n_l, k_l // 2), dtype=torch.uint8, device=dev)
        gz = graph_of(torch, lambda: wq._check(wq._lib.wq_fake_quant_ste(
            wq._ptr(zl), n_l, k_l, 64, wq._ptr(scl), wq._ptr(qo), None, wq._ptr(po), wq._stream(zl))))
        ms = max_over_ranks(time_region(torch, stream, gz.replay, steps, warm, barrier))
        byts = nw * (4 + 4 + 0.5) + nw / 64 * 2
        out["fake_quant_ste_large"] = {"shape": [n_l, k_l], "GB/s": round(byts / ms / 1e6, 1), "us": round(ms * 1e3, 1),
                                       "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4)}
        del gz
        # Gumbel-ST backward on the same latent: z, gq in; gz, gscale out (12.1 B per element),
        # 16 softmax weights per element; at tau = 1.0 (mid-way through the page's 5 -> 0.3
        # anneal: the weights spread over all codes) and at tau = step^2 of a typical group
        # (weights concentrated near the nearest code)
        gql = torch.randn((n_l, k_l), device=dev)
        gzo = torch.empty_like(zl)
        gso = torch.empty((n_l, k_l // 64), dtype=torch.float32, device=dev)
        gum = {"shape": [n_l, k_l], "ex2_per_element": 16}
        for name, tau in (("tau_1.0", 1.0), ("tau_step2", float((scl.float().median() / 8) ** 2))):
            ggb = graph_of(torch, lambda: wq._check(wq._lib.wq_gumbel_st_backward(
                wq._ptr(zl), n_l, k_l, 64, wq._ptr(scl), tau, wq._ptr(gql), wq._ptr(gzo), wq._ptr(gso),
                wq._stream(zl))))
            ms = max_over_ranks(time_region(torch, stream, ggb.replay, steps, warm, barrier))
            byts = nw * (4 + 4 + 4) + nw / 64 * (2 + 4)
            gum[name] = {"tau": tau, "us": round(ms * 1e3, 1), "Gelements/s": round(nw / ms / 1e6, 2),
                         "GB/s": round(byts / ms / 1e6, 1),
                         "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4)}
            del ggb
        out["gumbel_st_backward_large"] = gum
        del gql, gzo, gso, zl, scl, qo, po
        # BF16X lossless codec on a bf16 matrix of the same shape (N(0, 0.02^2)): the two
        # encoding passes (count, encode) and the decode, each a plain stream
        wb = (torch.randn((n_l, k_l), device=dev) * 0.02).to(torch.bfloat16)
        enc = wq.bf16x_encode(wb)
        ge = graph_of(torch, lambda: wq.bf16x_encode_into(wb, enc))
        ms_e = max_over_ranks(time_region(torch, stream, ge.replay, steps, warm, barrier))
        dout = torch.empty_like(wb)
        gd = graph_of(torch, lambda: wq.bf16x_decode(enc, out=dout))
        ms_d = max_over_ranks(time_region(torch, stream, gd.replay, steps, warm, barrier))
        assert torch.equal(dout.view(torch.int16), wb.view(torch.int16)), "BF16X round trip differs"
        code_b = enc.nbytes()
        enc_b = nw * 2 + nw * 2 + code_b             # count reads w; encode reads w, writes the code
        dec_b = code_b + nw * 2
        out["bf16x_large"] = {"shape": [n_l, k_l], "bits_per_weight": round(8 * code_b / nw, 3),
                              "escapes": enc.escapes,
                              "encode_us": round(ms_e * 1e3, 1), "encode_GB/s": round(enc_b / ms_e / 1e6, 1),
                              "encode_frac_hbm": round(enc_b / ms_e / 1e6 / peaks["hbm_gbs"], 4),
                              "decode_us": round(ms_d * 1e3, 1), "decode_GB/s": round(dec_b / ms_d / 1e6, 1),
                              "decode_frac_hbm": round(dec_b / ms_d / 1e6 / peaks["hbm_gbs"], 4)}
        del ge, gd, enc, dout
        # water-filling 3/4/5-bit blocks on the same matrix, water level at the median 4-bit
        # squared error (about 4.5 bits per weight): both producer passes (analyze with the
        # offset scan, pack) and the dequant
        nblk = n_l * k_l // 64
        sc, wd, off, dd = wq.wf_analyze(wb, 0.0, dist=True)
        lam = float(dd[..., 1].median()) / 64
        del dd
        pk = torch.empty(40 * nblk, dtype=torch.uint8, device=dev)

        def wf_q():
            wq._check(wq._lib.wq_quantize_wf_analyze(wq._ptr(wb), n_l, k_l, lam, wq._ptr(sc), wq._ptr(wd),
                                                     wq._ptr(off), None, wq._stream(wb)))
            wq._check(wq._lib.wq_quantize_wf_pack(wq._ptr(wb), n_l, k_l, wq._ptr(sc), wq._ptr(wd), wq._ptr(off),
                                                  wq._ptr(pk), pk.numel(), wq._stream(wb)))
        gq_ = graph_of(torch, wf_q)
        ms_q = max_over_ranks(time_region(torch, stream, gq_.replay, steps, warm, barrier))
        total = int(off[-1].item()) & 0xFFFFFFFF
        dwf = torch.empty_like(wb)
        gdw = graph_of(torch, lambda: wq._check(wq._lib.wq_dequant_wf(
            wq._ptr(pk), pk.numel(), wq._ptr(sc), wq._ptr(wd), wq._ptr(off), n_l, k_l, wq._ptr(dwf), wq._stream(wb))))
        ms_dq = max_over_ranks(time_region(torch, stream, gdw.replay, steps, warm, barrier))
        side = nblk * (2 + 1 + 4)                          # scale, width, offset per block
        dq_b = total + side + nw * 2
        out["water_filling_large"] = {"shape": [n_l, k_l], "lambda": lam,
                                      "bits_per_weight": round(8 * total / nw, 3),
                                      "quantize_us": round(ms_q * 1e3, 1),
                                      "quantize_Gweights/s": round(nw / ms_q / 1e6, 2),
                                      "dequant_us": round(ms_dq * 1e3, 1), "dequant_GB/s": round(dq_b / ms_dq / 1e6, 1),
                                      "dequant_frac_hbm": round(dq_b / ms_dq / 1e6 / peaks["hbm_gbs"], 4)}
        # the format's GEMV (weights rebuilt as the dequant does, fp32 products), batch 1 / 2 / 4 / 16
        qwf = wq.WfWeight(n_l, k_l, sc, wd, off, pk, total)
        for b in (1, 2, 4, 16):
            xw = torch.randn((b, k_l), device=dev).to(torch.bfloat16)
            yw = torch.empty((b, n_l), dtype=torch.bfloat16, device=dev)
            gg = graph_of(torch, lambda: wq.gemv_wf(qwf, xw, out=yw))
            ms_g = max_over_ranks(time_region(torch, stream, gg.replay, steps, warm, barrier))
            g_b = total + side + 2 * b * (k_l + n_l)
            out["water_filling_large"][f"gemv_b{b}"] = {
                "us": round(ms_g * 1e3, 1), "GB/s": round(g_b / ms_g / 1e6, 1),
                "frac_hbm": round(g_b / ms_g / 1e6 / peaks["hbm_gbs"], 4)}
            del gg
        del gq_, gdw, sc, wd, off, pk, dwf, wb, qwf
    except Exception as e:
        out["quantize_dyadic_layer"] = {"error": repr(e)[:200]}
    if args.extras in ("gemm", "all"):
        with nvtx_range(torch, "extras: prefill GEMM"):
            out["prefill_gemm"] = bench_gemm(args, wq, torch, dev, stream, peaks, barrier, max_over_ranks)
    if args.extras in ("producers", "all"):
        with nvtx_range(torch, "extras: producers and codebook GEMVs"):
            out.update(bench_producers(args, wq, torch, dev, stream, peaks, barrier, max_over_ranks))
    return out


def bench_gemm(args, wq, torch, dev, stream, peaks, barrier, max_over_ranks):
    """Prefill W4A16 GEMM on both weight shapes and every m of the prefill workload, with
    the unfused "materialised" comparison line (dequant once + a cuBLAS bf16 GEMM)."""
    res = {}
    steps, warm = max(args.steps, 5), 3
    for n, k in workloads.PREFILL_SHAPES:
        wb = workloads.gaussian_outlier_weight(n, k, workloads.PREFILL, 0 if n == 4096 else 1)
        w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(dev)
        pw, _ = wq.quantize_dyadic(w, 64)
        del w
        wdeq = wq.dequant(pw)
        for m in workloads.PREFILL_M:
            try:
                x = torch.randn((m, k), device=dev).to(torch.bfloat16)
                y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
                need = wq.gemm_workspace_bytes(pw, m)
                ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
                g = graph_of(torch, lambda: wq.gemm(pw, x, out=y, workspace=ws))
                ms = max_over_ranks(time_region(torch, stream, g.replay, steps, warm, barrier))
                fl = 2.0 * m * n * k
                byts = n * k * (0.5 + 2 / 64) + 2 * m * k + 2 * m * n
                ym = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
                gm = graph_of(torch, lambda: torch.matmul(x, wdeq.t(), out=ym))
                ms_mat = max_over_ranks(time_region(torch, stream, gm.replay, steps, warm, barrier))
                del g, gm
                res[f"{n}x{k}_m{m}"] = {
                    "TFLOP/s": round(fl / ms / 1e9, 1), "frac_bf16_peak": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4),
                    "GB/s": round(byts / ms / 1e6, 1), "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4),
                    "us": round(ms * 1e3, 2), "split_k_workspace_bytes": need,
                    "cublas_bf16_materialized_TFLOP/s": round(fl / ms_mat / 1e9, 1)}
            except Exception as e:
                res[f"{n}x{k}_m{m}"] = {"error": repr(e)[:200]}
        del wdeq, pw
    # the fused LLOYD8S consumer on the same GEMM (g32 codes plus fp32 levels; random codes
    # and sorted levels: the timing does not depend on the values)
    try:
        n, k = workloads.PREFILL_SHAPES[0]
        gen = torch.Generator(device=dev).manual_seed(5)
        codes = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=gen)
        levels = torch.sort(torch.rand((n, k // 32, 8), device=dev, generator=gen) * 0.05, dim=-1).values
        pl = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, codes, levels.contiguous())
        for m in (512, 4096):
            x = torch.randn((m, k), device=dev).to(torch.bfloat16)
            y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(wq.gemm_workspace_bytes(pl, m), 16), dtype=torch.uint8, device=dev)
            g = graph_of(torch, lambda: wq.gemm(pl, x, out=y, workspace=ws))
            ms = max_over_ranks(time_region(torch, stream, g.replay, steps, warm, barrier))
            fl = 2.0 * m * n * k
            res[f"lloyd8s_{n}x{k}_m{m}"] = {"TFLOP/s": round(fl / ms / 1e9, 1), "us": round(ms * 1e3, 2),
                                            "frac_bf16_peak": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4)}
            del g
    except Exception as e:
        res["lloyd8s"] = {"error": repr(e)[:200]}
    # the LUT16 consumer on the same GEMM (fp16 centroids, fp16 MMA; the timed region includes
    # the activations' bf16 -> fp16 conversion into the workspace)
    try:
        n, k = workloads.PREFILL_SHAPES[0]
        gen = torch.Generator(device=dev).manual_seed(6)
        codes = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=gen)
        lut = torch.sort(torch.randn((n, k // 64, 16), device=dev, generator=gen) * 0.01, dim=-1).values
        pu = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, codes, lut.to(torch.float16).contiguous())
        for m in (512, 4096):
            x = torch.randn((m, k), device=dev).to(torch.bfloat16)
            y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(max(wq.gemm_workspace_bytes(pu, m), 16), dtype=torch.uint8, device=dev)
            g = graph_of(torch, lambda: wq.gemm(pu, x, out=y, workspace=ws))
            ms = max_over_ranks(time_region(torch, stream, g.replay, steps, warm, barrier))
            fl = 2.0 * m * n * k
            res[f"lut16_{n}x{k}_m{m}"] = {"TFLOP/s": round(fl / ms / 1e9, 1), "us": round(ms * 1e3, 2),
                                          "frac_fp16_peak": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4)}
            del g
    except Exception as e:
        res["lut16"] = {"error": repr(e)[:200]}
    return res


def bench_producers(args, wq, torch, dev, stream, peaks, barrier, max_over_ranks):
    """Lloyd g32 (a 16-matrix sample of the 224-matrix workload), 16-centroid k-means on the
    8192x28672 LUT16 workload, and the LUT16 GEMV at batch 1/8/16."""
    out = {}
    try:
        nm = 16
        with ThreadPoolExecutor(8) as ex:
            hw = list(ex.map(lambda i: workloads.laplace_rowscaled_weight(2048, 2048, index=i), range(nm)))
        ws = [torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(dev) for h in hw]

        made = []

        def lloyd():
            made.clear()
            for w in ws:
                made.append(wq.quantize_lloyd(w, wq.LLOYD_G32_WARM, 25)[0])
        ms = max_over_ranks(time_region(torch, stream, lloyd, 2, 1, barrier))
        n_w = nm * 2048 * 2048
        # special-function roofline: the screen evaluates every (weight, candidate) pair, and
        # each evaluation needs at least one special-function result (the reciprocal of the
        # rational transform's denominator, or tanh); the unit gives 16 per clock per SM
        evals = n_w * 112
        xu_peak = 16 * torch.cuda.get_device_properties(dev).multi_processor_count * peaks["sm_max_mhz"] * 1e6
        out["lloyd_g32"] = {"Gweights/s": round(n_w / ms / 1e6, 3), "ms_per_matrix": round(ms / nm, 3),
                            "sample": f"{nm} of the 224 matrices 2048x2048",
                            "extrapolated_224_s": round(ms / nm * 224 / 1e3, 3),
                            "roofline": {"bound": "xu", "unit": "G candidate evaluations/s",
                                         "achieved": round(evals / ms / 1e6, 1),
                                         "peak": round(xu_peak / 1e9, 1),
                                         "frac": round(evals / ms * 1e3 / xu_peak, 4),
                                         "peak_basis": "one special-function result per evaluation, "
                                                       "16 per clock per SM"}}
        del ws
        # the fused LLOYD8S consumer: one grouped GEMV over those matrices, batch 1 (codes
        # 0.5 B + fp32 levels 1 B per weight)
        xs_l = [torch.randn((1, 2048), device=dev).to(torch.bfloat16) for _ in made]
        ys_l = [torch.empty((1, 2048), dtype=torch.bfloat16, device=dev) for _ in made]
        run_l = wq.GroupedGemv(made, xs_l, ys_l)
        g = graph_of(torch, run_l)
        ms = max_over_ranks(time_region(torch, stream, g.replay, 20, 3, barrier))
        byts = n_w * 1.5 + len(made) * 2048 * 4
        out["lloyd8s_gemv_b1"] = {"matrices": len(made), "GB/s": round(byts / ms / 1e6, 1), "us": round(ms * 1e3, 2),
                                  "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4)}
        del g, run_l, made
    except Exception as e:
        out["lloyd_g32"] = {"error": repr(e)[:200]}
    try:
        n, k = workloads.LUT16_SHAPE
        hb = workloads.lut16_weight(n, k, heavy_tail=True)
        w = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16).to(dev)
        del hb
        holder = {}

        def km():
            holder["pw"], _ = wq.quantize_lloyd(w, wq.LLOYD_KMEANS16, 25)
        ms = max_over_ranks(time_region(torch, stream, km, 3, 1, barrier))
        out["kmeans16"] = {"Gweights/s": round(n * k / ms / 1e6, 3), "ms": round(ms, 2)}
        pw = holder["pw"]
        del w
        for b in (1, 8, 16):
            x = torch.randn((b, k), device=dev).to(torch.bfloat16)
            y = torch.empty((b, n), dtype=torch.bfloat16, device=dev)
            g = graph_of(torch, lambda: wq.gemv(pw, x, out=y))
            ms = max_over_ranks(time_region(torch, stream, g.replay, 20, 3, barrier))
            del g
            byts = n * k * (0.5 + 0.5)
            out[f"lut16_gemv_b{b}"] = {"GB/s": round(byts / ms / 1e6, 1), "us": round(ms * 1e3, 2),
                                       "frac_hbm": round(byts / ms / 1e6 / peaks["hbm_gbs"], 4),
                                       "packed_only_GB/s": round(n * k * 0.5 / ms / 1e6, 1)}
    except Exception as e:
        out["kmeans16"] = {"error": repr(e)[:200]}
    return out


# ---------------------------------------------------------------------------------------
# CPU oracle baseline / reference arm
# ---------------------------------------------------------------------------------------

def _oracle_sample_rows(mats, rows_per_matrix: int, seed: int = 0):
    """A bounded sample of the sweep: `rows_per_matrix` rows of each of the 7 distinct
    projection shapes of layer 0 (weights drawn and quantised by the oracle)."""
    import oracle
    rng = np.random.default_rng(seed)
    sample = []
    for layer, name, n, k, idx in mats[:7]:
        rows = np.sort(rng.choice(n, min(rows_per_matrix, n), replace=False))
        w = workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, idx)[rows]
        s, c = oracle.dyadic_quantize(w, 64)
        sample.append((oracle.pack(c), s, workloads.activations(1, k, workloads.DECODE_SWEEP, idx)))
    return sample


def cpu_baseline(args, mats, seconds: float = 15.0, batch: int | None = None):
    """The oracle (fp64 dequant + dot, all host cores) on a bounded sample of the sweep:
    256 rows of each of the 7 projection shapes, repeated until ~`seconds` of CPU work."""
    import oracle
    batch = batch or args.batch
    threads = oracle.default_threads()
    sample = _oracle_sample_rows(mats, 256)
    nbytes = sum(p.size + s.size * 2 for p, s, _ in sample)

    def one_pass():
        for packed, s, x in sample:
            oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, np.repeat(x, batch, 0), threads=threads)

    t0 = time.perf_counter()
    one_pass()
    t1 = time.perf_counter() - t0
    reps = max(1, int(round(seconds / max(t1, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        one_pass()
    dt = time.perf_counter() - t0
    return {"value": round(reps * nbytes / dt / 1e9, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"256 rows of each of the 7 projection shapes of one sweep layer, batch {batch}, "
                      f"fp64 dequant + dot, {reps} passes in {dt:.1f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    mats = workloads.sweep_matrices()
    import oracle
    threads = oracle.default_threads()
    sample = _oracle_sample_rows(mats, args.ref_rows)
    nbytes = sum(p.size + s.size * 2 for p, s, _ in sample)

    def step():
        for packed, s, x in sample:
            oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, np.repeat(x, args.batch, 0), threads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = round(nbytes / dt / 1e9, 6)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy PCG64, pages' value distributions)",
            "config": {"workload": "decode sweep: 24 layers x {q,k,v,o,gate,up,down} dyadic g64, "
                                   "hidden 2048, intermediate 5632, 1,056,964,608 weights",
                       "batch": args.batch, "sample_rows_per_shape": args.ref_rows},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{args.ref_rows} rows of each of the 7 projection shapes per step"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_target(args):
    """A few launches of one kernel on one shape and nothing else, for ncu captures:
    --profile gemm --shape N,K,M (prefill GEMM; gemm_lut16: its LUT16 form, with the
    activation conversion), quantize --shape N,K, dequant --shape N,K,
    lut16 --shape N,K,B (LUT16 GEMV), lloyd8s --shape N,K,B (the fused LLOYD8S GEMV),
    lloyd --shape N,K (g32 Lloyd), gumbel --shape N,K
    (Gumbel-ST backward at tau = step^2; gumbel1: at tau = 1.0), ste --shape N,K (STE forward),
    kmeans --shape N,K (16-centroid k-means),
    bf16x --shape N,K (BF16X encode + decode), wf --shape N,K
    (water-filling analyze + dequant), wf_gemv --shape N,K,B (its GEMV). Random packed codes and
    scales (timing does not depend on the values); inputs stay on the device."""
    import torch
    import __graft_entry__
    __graft_entry__._build_module().build()
    import w4a16_matmul_b200 as wq
    dev = torch.device("cuda")
    dims = [int(v) for v in args.shape.split(",")]
    n, k = dims[0], dims[1]
    gen = torch.Generator(device=dev).manual_seed(0)
    packed = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=dev, generator=gen)
    scale = (torch.rand((n, k // 64), device=dev, generator=gen) * 0.09 + 0.01).to(torch.bfloat16)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, packed, scale)
    if args.profile == "gemm":
        m = dims[2]
        x = torch.randn((m, k), device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, wq.gemm_workspace_bytes(pw, m)), dtype=torch.uint8, device=dev)
        fn = lambda: wq.gemm(pw, x, out=y, workspace=ws)
    elif args.profile == "gemm_lut16":
        m = dims[2]
        lut = (torch.randn((n, k // 64, 16), device=dev, generator=gen) * 0.01).to(torch.float16)
        pl = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, packed, lut)
        x = torch.randn((m, k), device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(max(16, wq.gemm_workspace_bytes(pl, m)), dtype=torch.uint8, device=dev)
        fn = lambda: wq.gemm(pl, x, out=y, workspace=ws)
    elif args.profile == "quantize":
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.02).to(torch.bfloat16)
        fn = lambda: wq.quantize_dyadic(w, 64)
    elif args.profile == "dequant":
        out = torch.empty((n, k), dtype=torch.bfloat16, device=dev)
        fn = lambda: wq.dequant(pw, out=out)
    elif args.profile == "lut16":
        b = dims[2]
        lut = (torch.randn((n, k // 64, 16), device=dev, generator=gen) * 0.01).to(torch.float16)
        pl = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, packed, lut)
        x = torch.randn((b, k), device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty((b, n), dtype=torch.bfloat16, device=dev)
        fn = lambda: wq.gemv(pl, x, out=y)
    elif args.profile == "lloyd8s":
        b = dims[2]
        levels = torch.sort(torch.rand((n, k // 32, 8), device=dev, generator=gen) * 0.05, dim=-1).values
        pl = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, packed, levels.contiguous())
        x = torch.randn((b, k), device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty((b, n), dtype=torch.bfloat16, device=dev)
        fn = lambda: wq.gemv(pl, x, out=y)
    elif args.profile == "gumbel":
        z = torch.randn((n, k), device=dev, generator=gen) * 0.02
        s = (z.abs().reshape(n, k // 64, 64).amax(-1) * 1.1).to(torch.bfloat16)
        gq = torch.randn((n, k), device=dev, generator=gen)
        tau = float((s.float().median() / 8) ** 2)
        fn = lambda: wq.gumbel_st_backward(z, s, gq, tau, 64)
    elif args.profile == "gumbel1":
        z = torch.randn((n, k), device=dev, generator=gen) * 0.02
        s = (z.abs().reshape(n, k // 64, 64).amax(-1) * 1.1).to(torch.bfloat16)
        gq = torch.randn((n, k), device=dev, generator=gen)
        fn = lambda: wq.gumbel_st_backward(z, s, gq, 1.0, 64)
    elif args.profile == "ste":
        z = torch.randn((n, k), device=dev, generator=gen) * 0.02
        s = (z.abs().reshape(n, k // 64, 64).amax(-1)).to(torch.bfloat16)
        fn = lambda: wq.fake_quant_ste(z, s, 64, packed=True)
    elif args.profile == "bf16x":
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.02).to(torch.bfloat16)
        enc = wq.bf16x_encode(w)
        out = torch.empty_like(w)
        fn = lambda: (wq.bf16x_encode_into(w, enc), wq.bf16x_decode(enc, out=out))
    elif args.profile == "wf":
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.02).to(torch.bfloat16)
        q = wq.quantize_wf(w, 1e-6)
        out = torch.empty_like(w)
        fn = lambda: (wq.wf_analyze(w, 1e-6), wq.dequant_wf(q, out=out))
    elif args.profile == "wf_gemv":
        b = dims[2]
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.02).to(torch.bfloat16)
        q = wq.quantize_wf(w, 1e-6)
        del w
        x = torch.randn((b, k), device=dev, generator=gen).to(torch.bfloat16)
        y = torch.empty((b, n), dtype=torch.bfloat16, device=dev)
        fn = lambda: wq.gemv_wf(q, x, out=y)
    elif args.profile == "lloyd":
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.02).to(torch.bfloat16)
        fn = lambda: wq.quantize_lloyd(w, wq.LLOYD_G32_WARM, 25)
    elif args.profile == "kmeans":
        w = (torch.randn((n, k), device=dev, generator=gen) * 0.01).to(torch.bfloat16)
        fn = lambda: wq.quantize_lloyd(w, wq.LLOYD_KMEANS16, 25)
    else:
        raise SystemExit(f"unknown --profile {args.profile}")
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    code = wq.device_error()
    if code:
        raise SystemExit(f"device error {code}")
    print(json.dumps({"profile": args.profile, "shape": dims, "ok": True}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--extras", default="all", choices=["sweep", "gemm", "producers", "all"],
                    help="which secondary rows to time after the headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--profile", default=None,
                    help="run a few launches of one kernel for an ncu capture (see run_profile_target)")
    ap.add_argument("--shape", default="4096,11008,4096")
    args = ap.parse_args()
    if args.profile:
        run_profile_target(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
