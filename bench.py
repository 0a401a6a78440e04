#!/usr/bin/env python
"""Throughput of one-layer GPTQ (INT4, g128) on a Llama-70B-shaped down_proj,
plus the AWQ alpha search and a 7B-shaped q_proj layer.

One step = the whole quantization of one layer through the C ABI
(gptq_quantize_layer: H = X^T X, damping, the FP64-grade factor, the blocked
sweep with its block updates, packing, output error on the calibration X).
Default workload (the largest single-GPU one): W 8192x28672 fp32 ~N(0, 0.01^2),
X 32768x28672 bf16 ~N(0, 1) with 143 channels x40; bits 4, g 128, damp 0.01.
``--workload q_proj_7b`` times W 4096^2 with X 131072x4096 (lognormal channel
stds, 41 channels x30) plus the error on the shifted X' instead.  Inputs are
synthetic and seeded (workloads/); X is larger than L2, so no flush is needed
between steps.

The JSON line also carries, unless switched off: the AWQ 20-point alpha search
on the 8192^2 layer (ms per layer, phases, their rooflines), the q_proj_7b
layer as a second record, per-phase roofline fractions of the headline layer,
and the FP64 oracle timed on the host cores (exactly on the tiny 256x512
layer; on a bounded sample of the headline layer, every scaled term labelled).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torch.distributed.run: every rank quantizes its own layer
(independent problems, no collective on the data path; weak scaling); the
timed region is bracketed by barriers and the max over ranks is reported.
``--impl reference`` times the FP64 oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
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

METRIC = "GPTQ INT4 sec/layer & Mweights/s; XᵀX TFLOPS; AWQ α-search ms/layer"
UNIT = "Mweights/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.idx)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        if not rows:
            return None
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:  # region shorter than the sampling period: nearest samples
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
        sm = [float(p[1]) for _, p in inside if p[1].replace(".", "").isdigit()]
        mx = [float(p[2]) for _, p in inside if p[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, p in inside:
            for k, name in enumerate(names):
                if p[5 + k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(inside)}


# ------------------------------------------------------------ distributed
def dist_setup(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch N>1 with "
                         "torch.distributed.run")
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------- workload
WORKLOADS = ("down_proj_70b", "q_proj_7b")
# DRAM bytes (read + write) per launch of the INT8 digit GEMM, averaged over the
# 864 launches of one down_proj_70b step in an ncu launch-list capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of this bench's own command.  It
# describes the kernel as it was captured; a changed kernel needs a new capture
# (or --traffic).
GEMM_TRAFFIC_PER_LAUNCH = {"down_proj_70b": 1.929e8}


def spec_of(name):
    from workloads import C2, C4
    return {"down_proj_70b": C4, "q_proj_7b": C2}[name]


def to_gpu_w(W, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).to(dev)


def to_gpu_x(Xbits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(Xbits).view(np.int16)).to(dev).view(
        torch.bfloat16)


def make_inputs(rank: int, n=None, workload="down_proj_70b"):
    """(W, X, X') of one rank's layer; X' (the shifted inputs) only for q_proj_7b."""
    from workloads import make_weight, make_x_bits
    spec = spec_of(workload)
    seed = spec.seed + rank               # each rank quantizes its own layer
    W = make_weight(spec, seed=seed)
    X = make_x_bits(spec, n=n, seed=seed)
    X2 = None
    if workload == "q_proj_7b":
        X2 = make_x_bits(spec, n=n, seed=seed + 1, permute_seed=seed + 1)
    return W, X, X2


def workload_config(spec, n, workload="down_proj_70b"):
    shifted = " (+ error on shifted X')" if workload == "q_proj_7b" else ""
    gb = n * spec.inp * 2 / 1e9
    return {"workload": f"{workload} GPTQ: W {spec.out}x{spec.inp} fp32, X {n}x{spec.inp} bf16"
                        f"{shifted}, bits {spec.bits}, g {spec.g}, damp {spec.damp}",
            "out": spec.out, "in": spec.inp, "samples": n, "bits": spec.bits, "g": spec.g,
            "l2_flush": f"not needed: inputs larger than L2 (X {gb:.2f} GB per step)"}


# ------------------------------------------------------------ roofline arithmetic
# Digits per operand of the FP64-grade products (library constants: factor 5,
# block updates 5) and the nominal INT8 : BF16 dense tensor ratio.
FACTOR_PAIRS = 5 * 6 // 2
SWEEP_PAIRS = 5 * 6 // 2
INT8_PER_BF16 = 2.0


def phase_rooflines(ph, out, inp, n, bf16_peak, hbm_peak):
    """Per-phase achieved rate and fraction of its roofline, from the phase
    times (ms) of one gptq_quantize_layer call.  Algorithmic work:
    hessian n in (in+1) bf16 flop (upper triangle); factor in^3 / 3 FP64 flop
    (Cholesky of the damped H), bound by the INT8 tensor rate over the 15 digit
    products of each FP64-grade product; sweep out in^2 FP64 flop of block
    updates (15 digit products); pack out in (1 + 4 + 4 + 1/2) bytes (codes and
    W read, D written, nibbles written); error 3 out in (in + 256) bf16 flop."""
    res = {}
    int8_peak = INT8_PER_BF16 * bf16_peak

    def put(k, work, unit, peak, scale):
        ms = ph.get(k)
        if ms:
            a = work / (ms / 1e3) / scale
            res[k] = {"ms": ms, "achieved": a, "unit": unit, "peak": peak, "frac": a / peak}

    put("hessian", float(n) * inp * (inp + 1), "TFLOP/s", bf16_peak, 1e12)
    put("factor", inp ** 3 / 3.0, "TFLOP/s (FP64-grade)", int8_peak / FACTOR_PAIRS, 1e12)
    put("sweep", float(out) * inp * inp, "TFLOP/s (FP64-grade)", int8_peak / SWEEP_PAIRS, 1e12)
    put("pack", out * inp * 9.5, "GB/s", hbm_peak, 1e9)
    put("error", 3.0 * out * inp * (inp + 256), "TFLOP/s", bf16_peak, 1e12)
    return res


# ---------------------------------------------------------- oracle baseline
def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample(W, X, X2, n_full, n_rows=1024, w_rows=64, sub_in=4096):
    """The FP64 oracle on a bounded sample of one layer, scaled to the full
    layer.  Returns (seconds per full layer, description).  Every scaled term
    is named in the description:
      H on n_rows of n_full samples, scaled by samples;
      factor (damping, inv, cholesky) of the leading sub_in x sub_in block of
        that H, scaled by (in / sub_in)^3 when in > sub_in;
      blocked sweep of w_rows rows over the leading sub_in columns, scaled by
        rows and by (in / sub_in)^2;
      output errors on n_rows samples x w_rows rows, scaled by samples x rows."""
    import oracle as O
    from oracle.gptq import gptq_sweep_blocked_ref
    from oracle.pack import dequant_ref
    n, inp = n_full, X.shape[1]
    out = W.shape[0]
    si = min(sub_in, inp)
    t0 = time.perf_counter()
    H = O.hessian_ref(X[:n_rows])
    t_h = time.perf_counter() - t0
    t0 = time.perf_counter()
    perm, U, lam = O.gptq_prepare_ref(H[:si, :si], 0.01, False)
    t_f = time.perf_counter() - t0
    Ws = W[:w_rows, :si].astype(np.float64)
    t0 = time.perf_counter()
    codes, scales, _ = gptq_sweep_blocked_ref(Ws[:, perm], U, 4, 128)
    t_s = time.perf_counter() - t0
    What = dequant_ref(codes, scales, perm, 128)
    t0 = time.perf_counter()
    O.output_error_ref(W[:w_rows, :si], What, X[:n_rows, :si])
    t_e = (time.perf_counter() - t0) * (inp / si)
    n_err = 2 if X2 is not None else 1
    fs = (inp / si) ** 3
    total = (t_h * n / n_rows + t_f * fs + t_s * (out / w_rows) * (inp / si) ** 2
             + n_err * t_e * (n / n_rows) * (out / w_rows))
    desc = (f"measured: H on {n_rows}/{n} samples (scaled x{n / n_rows:g}); factor of the "
            f"{si}x{si} leading block (scaled x{fs:g}); blocked sweep of {w_rows}/{out} rows "
            f"over {si}/{inp} columns (scaled x{(out / w_rows) * (inp / si) ** 2:g}); "
            f"{n_err} output error(s) on {n_rows} samples x {w_rows} rows x {si} columns "
            f"(scaled x{(n / n_rows) * (out / w_rows) * (inp / si):g}); "
            f"float64 NumPy/OpenBLAS")
    return total, desc


def oracle_tiny_exact():
    """The oracle's literal loop on the whole tiny layer (W 256x512, X 2048x512,
    4-bit g128): seconds, measured, nothing scaled."""
    import oracle as O
    from workloads import C1, make_weight, make_x_bits
    W, X = make_weight(C1), make_x_bits(C1)
    t0 = time.perf_counter()
    r = O.gptq_ref(W, X, bits=4, g=128, log=False)
    from oracle.pack import dequant_ref
    O.output_error_ref(W, dequant_ref(r.codes, r.scales, r.perm, 128), X)
    return time.perf_counter() - t0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    spec = spec_of(args.workload)
    n_sample = 1024
    W, X, X2 = make_inputs(0, n=n_sample, workload=args.workload)
    # each step a bounded sample: about five seconds of host float64 work
    kw = dict(n_rows=n_sample, w_rows=32, sub_in=2048)
    for _ in range(args.warmup):
        oracle_sample(W, X, X2, spec.n, **kw)
    secs = []
    desc = ""
    for _ in range(args.steps):
        s, desc = oracle_sample(W, X, X2, spec.n, **kw)
        secs.append(s)
    layer_s = statistics.median(secs)
    value = spec.out * spec.inp / layer_s / 1e6
    cfg = workload_config(spec, spec.n, args.workload)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": layer_s * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours
def time_layer(piq, torch, Wg, Xg, X2g, spec, ws, ws_err, res, steps, warmup, world, local,
               sample_clocks=True):
    """Device-timed steps of one layer (inputs resident in HBM): (ms per step,
    mean phase times, launches per step, fallbacks, clocks, last output, last
    shifted error, mean digit-GEMM stats per step)."""
    stream = torch.cuda.current_stream()

    def step():
        o = piq.gptq_quantize_layer(Wg, Xg, bits=spec.bits, g=spec.g, damp=spec.damp,
                                    workspace=ws, out=res)
        e2 = None
        if X2g is not None:
            e2 = piq.layer_output_error(Wg, o.qweight, o.scales, X2g, spec.bits, spec.g,
                                        g_idx=o.g_idx, workspace=ws_err)
        return o, e2

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    sampler = None
    if sample_clocks:
        sampler = ClockSampler(local if world > 1 else torch.cuda.current_device())
        sampler.start()
        time.sleep(0.3)
    piq.set_timing(True)
    phases = {}
    gemm = []
    l0 = piq.kernel_launches()
    f0 = piq.simt_gemm_fallbacks()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(steps):
        o, e2 = step()
        for k, v in piq.last_phase_times().items():
            phases.setdefault(k, []).append(v)
        gemm.append(piq.last_gemm_stats())
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.time()
    launches = piq.kernel_launches() - l0
    fallbacks = piq.simt_gemm_fallbacks() - f0
    piq.set_timing(False)
    ms = ev0.elapsed_time(ev1)
    clocks = None
    if sampler is not None:
        time.sleep(0.2)
        sampler.stop()
        clocks = sampler.summary(t_wall0, t_wall1)
    ms = max_over_ranks(ms, world)
    ph = {k: statistics.mean(v) for k, v in phases.items()}
    gs = {k: statistics.mean(g[k] for g in gemm) for k in ("ms", "int8_ops", "launches")}
    return ms / steps, ph, launches, fallbacks, clocks, o, e2, gs


def alloc_layer(piq, torch, spec, n, dev, with_shift):
    out_rows, inp = spec.out, spec.inp
    ws = torch.empty(piq.gptq_workspace_bytes(out_rows, inp, n, g=spec.g), dtype=torch.uint8,
                     device=dev)
    ws_err = None
    if with_shift:
        ws_err = torch.empty(piq.output_error_workspace_bytes(out_rows, inp, n),
                             dtype=torch.uint8, device=dev)
    res = piq.GPTQOutput(torch.empty(out_rows, inp // 8, dtype=torch.int32, device=dev),
                         torch.empty(out_rows, -(-inp // spec.g), dtype=torch.float16,
                                     device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev), None)
    return ws, ws_err, res


def run_ours(args):
    import torch
    import post_int4_weight_gptq_b200 as piq

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    spec = spec_of(args.workload)

    W, X, X2 = make_inputs(rank, n=args.samples, workload=args.workload)
    out_rows, inp = W.shape
    n = X.shape[0]
    Wg, Xg = to_gpu_w(W, dev), to_gpu_x(X, dev)
    X2g = to_gpu_x(X2, dev) if X2 is not None else None
    ws, ws_err, res = alloc_layer(piq, torch, spec, n, dev, X2 is not None)

    ms_step, ph, launches, fallbacks, clocks, o, e2, gs = time_layer(
        piq, torch, Wg, Xg, X2g, spec, ws, ws_err, res, args.steps, args.warmup, world, local)
    value = world * out_rows * inp / (ms_step / 1e3) / 1e6

    # ---- end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        stream = torch.cuda.current_stream()
        Wh = torch.from_numpy(W).pin_memory()
        Xh = torch.from_numpy(X.view(np.int16)).pin_memory()
        X2h = torch.from_numpy(X2.view(np.int16)).pin_memory() if X2 is not None else None
        Wd, Xd = torch.empty_like(Wg), torch.empty_like(Xg)
        X2d = torch.empty_like(X2g) if X2g is not None else None
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in res[:4]]
        h2d = Wh.numel() * 4 + Xh.numel() * 2 + (X2h.numel() * 2 if X2h is not None else 0)
        d2h = sum(t.numel() * t.element_size() for t in host_out) + 8 * (2 if X2 is not None else 1)
        k_e2e = max(1, min(args.steps, 5))
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k_e2e):
            Wd.copy_(Wh, non_blocking=True)
            Xd.copy_(Xh.view(torch.bfloat16), non_blocking=True)
            if X2d is not None:
                X2d.copy_(X2h.view(torch.bfloat16), non_blocking=True)
            oo = piq.gptq_quantize_layer(Wd, Xd, bits=spec.bits, g=spec.g, damp=spec.damp,
                                         workspace=ws, out=res)
            if X2d is not None:
                piq.layer_output_error(Wd, oo.qweight, oo.scales, X2d, spec.bits, spec.g,
                                       g_idx=oo.g_idx, workspace=ws_err)
            for hbuf, d in zip(host_out, oo[:4]):
                hbuf.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world) / k_e2e
        e2e = {"value": world * out_rows * inp / (ms_e2e / 1e3) / 1e6, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ms_e2e, "steps": k_e2e}
        del Wd, Xd, X2d, Wh, Xh, X2h

    # ---- rooflines: burst peaks unless the timed region's clocks show the power cap
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    peak_key = "bf16_tflops_sustained" if capped else "bf16_tflops"
    bf16_peak = peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    phase_roof = phase_rooflines(ph, out_rows, inp, n, bf16_peak, hbm_peak)
    # the dominant kernel: the INT8 digit GEMM (FP64-grade products of the factor
    # and the sweep), timed per launch with CUDA events inside the timed steps;
    # its algorithmic work is 2 K per computed entry of C per digit pair
    int8_peak = INT8_PER_BF16 * bf16_peak
    g_tops = gs["int8_ops"] / (gs["ms"] / 1e3) / 1e12 if gs["ms"] > 0 else float("nan")
    roof = {"kernel": "ozaki_gemm_kernel<5> (INT8 digit products of the FP64-grade factor "
                      "and sweep; 48-wide tiles, stacked digits, tcgen05 kind::i8)",
            "bound": "tensor", "achieved": g_tops, "peak": int8_peak, "unit": "TOP/s (INT8)",
            "frac": g_tops / int8_peak,
            "traffic": (args.traffic if args.traffic is not None
                        else GEMM_TRAFFIC_PER_LAUNCH.get(args.workload)
                        if args.samples is None else None),
            "ms_per_step": gs["ms"], "share_of_step": gs["ms"] / ms_step,
            "launches_per_step": gs["launches"],
            "ms_per_launch": gs["ms"] / gs["launches"] if gs["launches"] else None,
            "int8_ops_per_launch": gs["int8_ops"] / gs["launches"] if gs["launches"] else None,
            "peak_source": f"{peak_src} {peak_key} x {INT8_PER_BF16:g} (nominal INT8 : BF16)"}
    ph_h = ph.get("hessian", float("nan"))
    xtx = float(n) * inp * (inp + 1) / (ph_h / 1e3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, desc = oracle_sample(W, X, X2, n)
        cpu = {"value": out_rows * inp / secs / 1e6, "unit": UNIT, "cores": cpu_cores(),
               "kind": "oracle", "sample": desc}
        t_tiny = oracle_tiny_exact()
        cpu["tiny_exact"] = {"workload": "tiny 256x512, X 2048x512, 4-bit g128 (whole layer, "
                                         "literal loop, nothing scaled)",
                             "seconds": t_tiny, "mweights_per_s": 256 * 512 / t_tiny / 1e6}
    del Wg, Xg, X2g, ws, ws_err
    torch.cuda.empty_cache()

    awq = None
    if not args.no_awq and rank == 0:
        awq = run_awq(dev, peaks)
    second = None
    if not args.no_second and rank == 0 and args.samples is None:
        other = "q_proj_7b" if args.workload == "down_proj_70b" else "down_proj_70b"
        second = run_second(piq, torch, dev, other)
    tiny = None
    if rank == 0 and cpu is not None:
        tiny = run_tiny(piq, torch, dev)
        tiny["oracle_seconds"] = cpu["tiny_exact"]["seconds"]
        tiny["speedup_vs_oracle"] = tiny["oracle_seconds"] / (tiny["ms_per_layer"] / 1e3)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "sec_per_layer": ms_step / 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 in, f64-grade factor/sweep", "data": "synthetic",
                "config": workload_config(spec, n, args.workload), "xtx_tflops": xtx,
                "awq_ms_per_layer": awq["ms_per_layer"] if awq else None,
                "phases_ms": ph, "phase_roofline": phase_roof, "roofline": roof,
                "cpu_baseline": cpu, "clocks": clocks, "e2e": e2e, "gpu_launches": launches,
                "simt_gemm_fallbacks": fallbacks, "awq": awq, "second_workload": second,
                "tiny_exact": tiny, "calib_error": o.err}
        if e2 is not None:
            line["shift_error"] = e2
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_second(piq, torch, dev, workload, steps=10, warmup=3):
    """A second GPTQ layer, device-timed like the headline one."""
    spec = spec_of(workload)
    W, X, X2 = make_inputs(0, workload=workload)
    Wg, Xg = to_gpu_w(W, dev), to_gpu_x(X, dev)
    X2g = to_gpu_x(X2, dev) if X2 is not None else None
    ws, ws_err, res = alloc_layer(piq, torch, spec, X.shape[0], dev, X2 is not None)
    ms, ph, _, _, _, o, e2, _ = time_layer(piq, torch, Wg, Xg, X2g, spec, ws, ws_err, res, steps,
                                        warmup, 1, 0, sample_clocks=False)
    r = {"workload": workload_config(spec, X.shape[0], workload)["workload"],
         "ms_per_layer": ms, "mweights_per_s": spec.out * spec.inp / (ms / 1e3) / 1e6,
         "xtx_tflops": float(X.shape[0]) * spec.inp * (spec.inp + 1) / (ph["hessian"] / 1e3) / 1e12,
         "phases_ms": ph, "calib_error": o.err}
    if e2 is not None:
        r["shift_error"] = e2
    del Wg, Xg, X2g, ws, ws_err
    torch.cuda.empty_cache()
    return r


def run_tiny(piq, torch, dev, steps=20, warmup=3):
    """The tiny layer on the GPU (device-timed), beside the oracle's exact time."""
    from workloads import C1, make_weight, make_x_bits
    Wg, Xg = to_gpu_w(make_weight(C1), dev), to_gpu_x(make_x_bits(C1), dev)
    for _ in range(warmup):
        piq.gptq_quantize_layer(Wg, Xg, bits=4, g=128)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        piq.gptq_quantize_layer(Wg, Xg, bits=4, g=128)
    e1.record()
    torch.cuda.synchronize()
    return {"workload": "tiny 256x512, X 2048x512, 4-bit g128",
            "ms_per_layer": e0.elapsed_time(e1) / steps}


def hbm_phase_rates(phases_ms, n, inp, out, n_alpha, hbm_peak_gbs):
    """Achieved HBM rate of AWQ's bandwidth-bound phases: algorithmic bytes
    (X read once for mean|x|: n*in*2; W read once and the n_alpha bf16 deltas
    written: out*in*4 + n_alpha*out*in*2) over the phase's measured time.  A
    phase time also holds its small launches (the grid copy, the finishing
    sums, the scale table), so these are lower bounds on the kernels' own."""
    algo = {"colstats": n * inp * 2, "quant_delta": out * inp * 4 + n_alpha * out * inp * 2}
    res = {}
    for k, b in algo.items():
        ms = phases_ms.get(k)
        if ms:
            gbs = b / (ms / 1e3) / 1e9
            res[k] = {"bytes": b, "gb_per_s": gbs, "frac": gbs / hbm_peak_gbs}
    return res


def run_awq(dev, peaks, steps=5, warmup=3):
    """AWQ alpha search (20-point grid) on the 8192x8192 layer: ms per layer."""
    import torch
    import post_int4_weight_gptq_b200 as piq
    from workloads import AWQ_GRID, C5, make_weight, make_x_bits
    W, X = make_weight(C5), make_x_bits(C5)
    Wg, Xg = to_gpu_w(W, dev), to_gpu_x(X, dev)
    ws = torch.empty(piq.awq_workspace_bytes(C5.out, C5.inp, C5.n, len(AWQ_GRID)),
                     dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        piq.awq_search_layer(Wg, Xg, C5.bits, C5.g, AWQ_GRID, workspace=ws)
    torch.cuda.synchronize()
    piq.set_timing(True)
    times, ph = [], {}
    for _ in range(steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        r = piq.awq_search_layer(Wg, Xg, C5.bits, C5.g, AWQ_GRID, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        for k, v in piq.last_phase_times().items():
            ph.setdefault(k, []).append(v)
    piq.set_timing(False)
    ph = {k: statistics.mean(v) for k, v in ph.items()}
    flops = 2.0 * C5.n * C5.inp * C5.out * len(AWQ_GRID)
    bf16 = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tf = flops / (ph["error_gemm"] / 1e3) / 1e12
    del Wg, Xg, ws
    torch.cuda.empty_cache()
    return {"workload": "AWQ 20-point alpha search: W 8192x8192, X 16384x8192, 4-bit g128",
            "ms_per_layer": statistics.median(times), "best_alpha": r.best_alpha,
            "phases_ms": ph, "error_gemm_tflops": tf, "error_gemm_frac": tf / bf16,
            "hbm": hbm_phase_rates(ph, C5.n, C5.inp, C5.out, len(AWQ_GRID),
                                   peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=WORKLOADS, default="down_proj_70b")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-awq", action="store_true", help="skip the AWQ search record")
    ap.add_argument("--no-second", action="store_true", help="skip the second GPTQ layer record")
    ap.add_argument("--samples", type=int, default=None,
                    help="calibration rows per layer (default: the workload's); a smaller "
                         "value is for profiler captures, not for reported numbers")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture of "
                         "the current kernel (reported as the roofline's traffic)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
