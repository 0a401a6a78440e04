"""Seeded synthetic layers: the only module both the CUDA path's tests and the
oracle's tests take inputs from.

It draws weights and calibration inputs and encodes them; it holds none of the
quantization arithmetic.  Every config below is a one-layer workload in the
shapes the GPTQ/AWQ pages talk about ("GPTQ versus AWQ objectives", the Hessian
size block: Llama q/k/v_proj input 8,192 and down_proj input 28,672), with
outlier input channels standing in for real calibration text.

Recipes (all float64 draws cast once; X is drawn in float32 and rounded to
bfloat16 with round-to-nearest-even, so both sides see the same bytes):

* W ~ N(0, w_std^2) drawn in float64, cast to float32.
* X[:, j] ~ N(0, 1) * sigma_j (or Student-t(4)/sqrt(2) * sigma_j), then a set
  of ``n_outlier`` distinct channels chosen without replacement is multiplied
  by ``outlier_gain``.  sigma_j is 1, or LogNormal(0, sigma_ln).
* Student-t(4)/sqrt(2) (variance 1) is drawn as Z / sqrt(G) with Z ~ N(0,1)
  and G ~ Gamma(2, 1): t_4 = Z / sqrt(chi2_4 / 4) and chi2_4 = 2 G.
* X is drawn in row chunks of ``CHUNK`` rows, each from its own spawned
  SeedSequence child, so the bytes do not depend on the thread count.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os

import numpy as np

CHUNK = 4096


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    out: int
    inp: int
    n: int
    w_std: float
    dist: str = "normal"          # "normal" | "t4"
    sigma_ln: float = 0.0         # 0 -> sigma_j = 1; else LogNormal(0, sigma_ln)
    n_outlier: int = 0
    outlier_gain: float = 1.0
    bits: int = 4
    g: int = 128
    damp: float = 0.01
    act_order: bool = False
    seed: int = 0


# The five workloads.  The outlier counts are round(frac * in) for the stated
# fractions (1%, 0.5%); C1 states its count directly.
C1 = LayerSpec("tiny", 256, 512, 2048, 0.02, n_outlier=5, outlier_gain=20.0)
C2 = LayerSpec("q_proj_7b", 4096, 4096, 131072, 0.02, sigma_ln=1.0,
               n_outlier=41, outlier_gain=30.0)
C3 = LayerSpec("down_proj_7b_actorder", 4096, 11008, 65536, 0.015, dist="t4",
               sigma_ln=1.2, act_order=True)
C4 = LayerSpec("down_proj_70b", 8192, 28672, 32768, 0.01, n_outlier=143,
               outlier_gain=40.0)
C5 = LayerSpec("awq_8192", 8192, 8192, 16384, 0.02, n_outlier=82, outlier_gain=50.0)
CONFIGS = {"C1": C1, "C2": C2, "C3": C3, "C4": C4, "C5": C5}

AWQ_GRID = tuple(k / 20.0 for k in range(20))


def make_weight(spec: LayerSpec, seed: int | None = None) -> np.ndarray:
    ss = np.random.SeedSequence([spec.seed if seed is None else seed, 1])
    rng = np.random.default_rng(ss)
    return (rng.standard_normal((spec.out, spec.inp)) * spec.w_std).astype(np.float32)


def make_channel_scales(inp: int, seed: int, sigma: float = 0.5) -> np.ndarray:
    """A positive per-input-channel vector s ~ LogNormal(0, sigma), float32 [in]
    (a stand-in for a searched channel scaling, so that a scaled layer can be
    tested without running the search)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 4]))
    return rng.lognormal(0.0, sigma, inp).astype(np.float32)


def channel_gains(spec: LayerSpec, seed: int | None = None,
                  permute_seed: int | None = None) -> np.ndarray:
    """Per-channel multiplier sigma_j * (outlier gain), float32 [in].

    ``permute_seed`` reshuffles the channel multipliers (the shifted X' of the
    q_proj workload: same stds, moved to other channels)."""
    ss = np.random.SeedSequence([spec.seed if seed is None else seed, 2])
    rng = np.random.default_rng(ss)
    if spec.sigma_ln > 0:
        sig = rng.lognormal(0.0, spec.sigma_ln, spec.inp)
    else:
        sig = np.ones(spec.inp)
    if spec.n_outlier:
        idx = rng.choice(spec.inp, spec.n_outlier, replace=False)
        sig[idx] *= spec.outlier_gain
    if permute_seed is not None:
        prng = np.random.default_rng(np.random.SeedSequence([permute_seed, 3]))
        sig = sig[prng.permutation(spec.inp)]
    return sig.astype(np.float32)


def _draw_chunk(args):
    child, rows, inp, dist, gains = args
    rng = np.random.default_rng(child)
    z = rng.standard_normal((rows, inp), dtype=np.float32)
    if dist == "t4":
        gam = rng.standard_gamma(2.0, (rows, inp), dtype=np.float32)
        z /= np.sqrt(gam)
    elif dist != "normal":
        raise ValueError(dist)
    z *= gains[None, :]
    return bf16_bits_from_f32(z)


def make_x_bits(spec: LayerSpec, n: int | None = None, seed: int | None = None,
                permute_seed: int | None = None, threads: int | None = None) -> np.ndarray:
    """Calibration inputs X [n, in] as bfloat16 bit patterns (uint16)."""
    n = spec.n if n is None else n
    s = spec.seed if seed is None else seed
    gains = channel_gains(spec, seed=s, permute_seed=permute_seed)
    nchunk = (n + CHUNK - 1) // CHUNK
    children = np.random.SeedSequence([s, 4]).spawn(nchunk)
    jobs = [(children[c], min(CHUNK, n - c * CHUNK), spec.inp, spec.dist, gains)
            for c in range(nchunk)]
    out = np.empty((n, spec.inp), dtype=np.uint16)
    threads = threads or min(32, os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for c, blk in enumerate(ex.map(_draw_chunk, jobs)):
            out[c * CHUNK: c * CHUNK + blk.shape[0]] = blk
    return out


def small_spec(out: int, inp: int, n: int, **kw) -> LayerSpec:
    """An ad-hoc layer for tests (ragged sizes, other bit widths and groups)."""
    base = dict(w_std=0.02, n_outlier=max(1, inp // 100), outlier_gain=20.0)
    base.update(kw)
    return LayerSpec("adhoc", out, inp, n, **base)
