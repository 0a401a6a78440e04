#!/usr/bin/env python
"""Throughput of one-layer GPTQ (INT4, g128) on a Llama-7B-shaped q_proj.

One step = the whole quantization of one layer through the C ABI:
gptq_quantize_layer (H = X^T X, damping, upper factor, blocked sweep with
trailing GEMMs, packing, output error on the calibration X) plus the output
error on the shifted X' (piq_layer_output_error) that the workload asks for.
Workload: W 4096x4096 fp32 ~N(0, 0.02^2); X 131072x4096 bf16 with per-channel
std ~LogNormal(0, 1) and 41 channels x30; X' a fresh draw with the channel stds
reshuffled; bits 4, g 128, damp 0.01.  Inputs are synthetic and seeded
(workloads/), X is larger than L2 so no flush is needed between steps.

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
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one syrk_xtx launch on the
# 131072 x 4096 workload, from one ncu capture of the current kernel; to be retaken (or set to
# None) whenever that kernel changes.
SYRK_TRAFFIC_BYTES = 1.93e9 + 21.82e6


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
def to_gpu_w(W, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).to(dev)


def to_gpu_x(Xbits, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(Xbits).view(np.int16)).to(dev).view(
        torch.bfloat16)


def make_inputs(rank: int, n=None):
    from workloads import C2, make_weight, make_x_bits
    seed = C2.seed + rank               # each rank quantizes its own layer
    W = make_weight(C2, seed=seed)
    X = make_x_bits(C2, n=n, seed=seed)
    X2 = make_x_bits(C2, n=n, seed=seed + 1, permute_seed=seed + 1)
    return W, X, X2


def workload_config(spec, n):
    return {"workload": f"q_proj_7b GPTQ: W {spec.out}x{spec.inp} fp32, X {n}x{spec.inp} bf16 "
                        f"(+ error on shifted X'), bits {spec.bits}, g {spec.g}, damp {spec.damp}",
            "out": spec.out, "in": spec.inp, "samples": n, "bits": spec.bits, "g": spec.g,
            "l2_flush": "not needed: inputs larger than L2 (X 1.07 GB per step)"}


# ---------------------------------------------------------- oracle baseline
def oracle_sample(W, X, X2, n_full, n_rows=4096, w_rows=256):
    """Oracle on a bounded sample, scaled to one full layer of n_full samples.
    Returns (seconds per full layer, description)."""
    import oracle as O
    from workloads import C2
    n, inp = n_full, X.shape[1]
    out = W.shape[0]
    t0 = time.perf_counter()
    H = O.hessian_ref(X[:n_rows])
    t_h = time.perf_counter() - t0
    t0 = time.perf_counter()
    perm, U, lam = O.gptq_prepare_ref(H, C2.damp, False)
    t_f = time.perf_counter() - t0
    t0 = time.perf_counter()
    from oracle.gptq import gptq_sweep_blocked_ref
    codes, scales, _ = gptq_sweep_blocked_ref(W[:w_rows].astype(np.float64)[:, perm], U, C2.bits,
                                              C2.g)
    t_s = time.perf_counter() - t0
    from oracle.pack import dequant_ref
    What = dequant_ref(codes, scales, perm, C2.g)
    t0 = time.perf_counter()
    O.output_error_ref(W[:w_rows], What, X[:n_rows])
    t_e1 = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.output_error_ref(W[:w_rows], What, X2[:n_rows])
    t_e2 = time.perf_counter() - t0
    # H and error scale with samples; sweep and error with rows; factor is whole
    total = (t_h * n / n_rows + t_f + t_s * out / w_rows
             + (t_e1 + t_e2) * (n / n_rows) * (out / w_rows))
    desc = (f"H on {n_rows}/{n} samples (x{n // n_rows}); factor of the full {inp}x{inp} H; "
            f"sweep on {w_rows}/{out} rows (x{out // w_rows}); errors on {n_rows} samples x "
            f"{w_rows} rows (x{(n // n_rows) * (out // w_rows)}); float64 NumPy/OpenBLAS")
    return total, desc


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import C2
    n_sample = 4096
    W, X, X2 = make_inputs(0, n=n_sample)
    for _ in range(args.warmup):
        oracle_sample(W, X, X2, C2.n, n_rows=n_sample)
    secs = []
    desc = ""
    for _ in range(args.steps):
        s, desc = oracle_sample(W, X, X2, C2.n, n_rows=n_sample)
        secs.append(s)
    layer_s = statistics.median(secs)
    value = C2.out * C2.inp / layer_s / 1e6
    cfg = workload_config(C2, C2.n)
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
def run_ours(args):
    import torch
    import post_int4_weight_gptq_b200 as piq
    from workloads import C2

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()

    W, X, X2 = make_inputs(rank, n=args.samples)
    out_rows, inp = W.shape
    n = X.shape[0]
    Wg, Xg, X2g = to_gpu_w(W, dev), to_gpu_x(X, dev), to_gpu_x(X2, dev)
    ws = torch.empty(piq.gptq_workspace_bytes(out_rows, inp, n), dtype=torch.uint8, device=dev)
    ws_err = torch.empty(piq.output_error_workspace_bytes(out_rows, inp, n), dtype=torch.uint8,
                         device=dev)
    res = piq.GPTQOutput(torch.empty(out_rows, inp // 8, dtype=torch.int32, device=dev),
                         torch.empty(out_rows, inp // C2.g, dtype=torch.float16, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev), None)
    stream = torch.cuda.current_stream()

    def step(Wd, Xd, X2d):
        o = piq.gptq_quantize_layer(Wd, Xd, bits=C2.bits, g=C2.g, damp=C2.damp, workspace=ws,
                                    out=res)
        e2 = piq.layer_output_error(Wd, o.qweight, o.scales, X2d, C2.bits, C2.g, g_idx=o.g_idx,
                                    workspace=ws_err)
        return o, e2

    for _ in range(args.warmup):
        step(Wg, Xg, X2g)
    torch.cuda.synchronize()

    # ---- device-timed region (inputs resident in HBM)
    sampler = ClockSampler(local if world > 1 else torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    piq.set_timing(True)
    phases = {}
    l0 = piq.kernel_launches()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        o, e2 = step(Wg, Xg, X2g)
        for k, v in piq.last_phase_times().items():
            phases.setdefault(k, []).append(v)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.time()
    launches = piq.kernel_launches() - l0
    piq.set_timing(False)
    ms = ev0.elapsed_time(ev1)
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    ms = max_over_ranks(ms, world)
    ms_step = ms / args.steps
    value = world * out_rows * inp / (ms_step / 1e3) / 1e6

    # ---- end to end through the public API from pinned host buffers
    e2e = None
    if not args.no_e2e:
        Wh = torch.from_numpy(W).pin_memory()
        Xh = torch.from_numpy(X.view(np.int16)).pin_memory()
        X2h = torch.from_numpy(X2.view(np.int16)).pin_memory()
        Wd, Xd, X2d = torch.empty_like(Wg), torch.empty_like(Xg), torch.empty_like(X2g)
        host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in res[:4]]
        h2d = Wh.numel() * 4 + Xh.numel() * 2 + X2h.numel() * 2
        d2h = sum(t.numel() * t.element_size() for t in host_out) + 16
        k_e2e = max(1, min(args.steps, 5))
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k_e2e):
            Wd.copy_(Wh, non_blocking=True)
            Xd.copy_(Xh.view(torch.bfloat16), non_blocking=True)
            X2d.copy_(X2h.view(torch.bfloat16), non_blocking=True)
            o, e2 = step(Wd, Xd, X2d)
            for h, d in zip(host_out, o[:4]):
                h.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world) / k_e2e
        e2e = {"value": world * out_rows * inp / (ms_e2e / 1e3) / 1e6, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ms_e2e, "steps": k_e2e}

    # ---- roofline of the dominant kernel, the X^T X build (per-phase CUDA
    # events on the launching stream, averaged over the timed steps).  The
    # denominator is the measured burst bf16 peak unless the clock samples of
    # the timed region show the power cap, then the sustained one.
    ph = {k: statistics.mean(v) for k, v in phases.items()}
    t_h = ph.get("hessian", float("nan"))
    flops_h = float(n) * inp * (inp + 1)
    capped = "sw_power_cap" in (clocks or {}).get("reasons", [])
    peak_key = "bf16_tflops_sustained" if capped else "bf16_tflops"
    peak = peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    ach_h = flops_h / (t_h / 1e3) / 1e12
    roof = {"kernel": "syrk_xtx (tcgen05 H = X^T X, 1024-sample chunks summed in registers)",
            "bound": "tensor", "achieved": ach_h, "peak": peak, "unit": "TFLOP/s",
            "frac": ach_h / peak,
            "traffic": args.traffic if args.traffic is not None else (
                SYRK_TRAFFIC_BYTES if args.samples is None else None),
            "flops_per_launch": flops_h,
            "flops_formula": "n*in*(in+1) (upper triangle)", "ms_per_launch": t_h,
            "peak_source": f"{peak_src} {peak_key}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, desc = oracle_sample(W, X, X2, n)
        cpu = {"value": out_rows * inp / secs / 1e6, "unit": UNIT, "cores": cpu_cores(),
               "kind": "oracle", "sample": desc}

    awq = None
    if args.awq and rank == 0:
        awq = run_awq(dev)
    variants = None
    if args.variants and rank == 0:
        variants = run_variants(dev, Wg, Xg)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "sec_per_layer": ms_step / 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16/f32", "data": "synthetic",
                "config": workload_config(C2, n), "xtx_tflops": ach_h,
                "phases_ms": ph, "roofline": roof,
                "cpu_baseline": cpu, "clocks": clocks, "e2e": e2e, "gpu_launches": launches,
                "awq": awq, "variants": variants, "shift_error": e2, "calib_error": o.err}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


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


def run_awq(dev, steps=3, warmup=1):
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
    peaks, src = load_peaks()
    return {"workload": "AWQ 20-point alpha search: W 8192x8192, X 16384x8192",
            "ms_per_layer": statistics.median(times), "best_alpha": r.best_alpha,
            "phases_ms": ph, "error_gemm_tflops": flops / (ph["error_gemm"] / 1e3) / 1e12,
            "hbm": hbm_phase_rates(ph, C5.n, C5.inp, C5.out, len(AWQ_GRID), peaks["hbm_gbs"]),
            "hbm_peak_source": f"{src} hbm_gbs"}


def run_variants(dev, Wg, Xg, steps=5, warmup=3):
    """The q_proj layer through plain GPTQ, AWQ-scaled GPTQ (s from AWQ's
    20-point search, run once untimed) and GPTQ with asymmetric groups, timed
    interleaved step by step so that all three see the same clocks: ms per layer
    (median) and each one's output error."""
    import torch
    import post_int4_weight_gptq_b200 as piq
    from workloads import AWQ_GRID, C2
    out_rows, inp = Wg.shape
    n = Xg.shape[0]
    a = piq.awq_search_layer(Wg, Xg, C2.bits, C2.g, AWQ_GRID)
    ws = torch.empty(piq.gptq_workspace_bytes(out_rows, inp, n), dtype=torch.uint8, device=dev)
    calls = {
        "gptq": lambda: piq.gptq_quantize_layer(Wg, Xg, C2.bits, C2.g, C2.damp, workspace=ws),
        "awq_then_gptq": lambda: piq.awq_gptq_quantize_layer(Wg, Xg, a.s, C2.bits, C2.g,
                                                             C2.damp, workspace=ws),
        "gptq_asym": lambda: piq.gptq_quantize_layer(Wg, Xg, C2.bits, C2.g, C2.damp,
                                                     workspace=ws, sym=False),
    }
    for _ in range(warmup):
        for f in calls.values():
            f()
    times = {k: [] for k in calls}
    errs = {}
    for _ in range(steps):
        for k, f in calls.items():
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            r = f()
            e1.record()
            torch.cuda.synchronize()
            times[k].append(e0.elapsed_time(e1))
            errs[k] = r.err
    res = {"workload": "q_proj 4096x4096, X 131072x4096, 4-bit g128: three GPTQ variants "
                       "timed interleaved", "awq_alpha": a.best_alpha,
           "awq_error": a.err_per_alpha[int(np.argmin([abs(x - a.best_alpha) for x in AWQ_GRID]))]}
    for k in calls:
        ms = statistics.median(times[k])
        res[k] = {"ms_per_layer": ms, "mweights_per_s": out_rows * inp / (ms / 1e3) / 1e6,
                  "error": errs[k]}
    return res


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--awq", action="store_true", help="also time the AWQ search (8192^2 layer)")
    ap.add_argument("--variants", action="store_true",
                    help="also time plain, AWQ-scaled and asymmetric-group GPTQ on the same "
                         "layer, interleaved")
    ap.add_argument("--samples", type=int, default=None,
                    help="calibration rows per layer (default: the workload's 131072); a smaller "
                         "value is for profiler captures, not for reported numbers")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per syrk_xtx launch from an ncu capture of the current "
                         "kernel (overrides the recorded figure)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
