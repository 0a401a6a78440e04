"""GPU-vs-oracle comparison helpers (used by the gpu tests and smoke()).

Contract (the benchmark spec's): at least 99.9% of the codes are
identical to the oracle's before anything is forced, and every code decided
differently lies where the oracle's w/scale is within 1e-4 of a rounding tie.
Because GPTQ feeds every rounding error forward, one tie flip changes the rest
of its row, so the comparison is teacher-forced: the oracle is re-run on the
affected rows with the GPU's code forced at the first mismatching site (which
must be a tie), until the rows agree; the forced sites are the codes decided
differently.  Scales and output errors then agree within 1e-3 relative.

Large layers (2048 columns and more) are re-run with the oracle's blocked
sweep, the same arithmetic as the literal loop (pinned by the oracle tests).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from oracle.gptq import NO_FORCE

TIE_TOL = 1e-4
MAX_MISMATCH_FRAC = 1e-3
REL_TOL = 1e-3
BLOCKED_FROM = 2048  # columns from which the forced re-runs use the blocked sweep


def to_gpu_w(W: np.ndarray, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).to(device)


def to_gpu_x(Xbits: np.ndarray, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(Xbits).view(np.int16)).to(device).view(
        torch.bfloat16)


def tie_distance(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    return np.abs(a - np.floor(a) - 0.5)


def fp32_drift(Wp: np.ndarray, U: np.ndarray, bits: int, g: int, ref) -> float:
    """Largest |w/scale| difference between the loop run in float32 and the
    float64 oracle ``ref`` on the same rows, up to each row's first differing
    code (after it the two runs follow different codes).  A diagnostic of what
    FP32 arithmetic alone does to the loop; the contract's tie window does not
    depend on it."""
    c32, _, v32, _ = O.gptq_sweep_ref(Wp, U, bits, g, dtype=np.float32)
    codes64, _, v64, _ = ref
    drift = 0.0
    for k in range(Wp.shape[0]):
        d = np.nonzero(c32[k] != codes64[k])[0]
        lim = d[0] if d.size else Wp.shape[1]
        if lim:
            drift = max(drift, float(np.abs(v32[k, :lim] - v64[k, :lim]).max()))
    return drift


def _sweep(Wr, U, bits, g, asym, force=None, force_zero=None):
    """(codes, scales, zeros, zv, v) of the oracle's loop (blocked for wide layers)."""
    if Wr.shape[1] >= BLOCKED_FROM:
        if asym:
            c, s, z, v, zv = O.gptq_sweep_blocked_asym_ref(Wr, U, bits, g, force=force,
                                                           force_zero=force_zero)
            return c, s, z, zv, v
        c, s, v = O.gptq_sweep_blocked_ref(Wr, U, bits, g, force=force)
        return c, s, None, None, v
    if asym:
        c, s, z, zv, v, _ = O.gptq_sweep_asym_ref(Wr, U, bits, g, force=force,
                                                  force_zero=force_zero)
        return c, s, z, zv, v
    c, s, v, _ = O.gptq_sweep_ref(Wr, U, bits, g, force=force)
    return c, s, None, None, v


def teacher_forced_compare(gpu_codes: np.ndarray, Wp: np.ndarray, U: np.ndarray, bits: int,
                           g: int, ref=None, max_iters: int = 64, tie_tol: float = TIE_TOL,
                           gpu_zeros: np.ndarray | None = None, bound: str = "raw"):
    """gpu_codes (signed), Wp in quantization order.  Returns (stats, codes,
    scales) of the forced oracle run on all rows, plus its zero-points when
    ``gpu_zeros`` ([out, ngroups], asymmetric groups) is given; raises
    AssertionError on a contract violation.  ``ref`` = (codes, scales, v) of
    the oracle's unforced run, when the caller has it.  A zero-point is a
    rounded value too (-lo / scale): where the GPU's differs, the oracle's
    unrounded value must be within the tie window of a half-integer, and it is
    forced like a code.

    bound="raw": mismatches before forcing (codes and zero-points) at most 0.1%
    of the codes; bound="forced": the forced sites at most 0.1% (for the FP32
    step entry, whose rows may diverge after a legitimate tie flip)."""
    asym = gpu_zeros is not None
    if asym and ref is not None:
        raise ValueError("a precomputed ref carries no zero-points; pass ref=None")
    gpu_codes = np.asarray(gpu_codes, dtype=np.int16)
    if ref is None:
        codes0, scales0, zeros0, _, _ = _sweep(Wp, U, bits, g, asym)
    else:
        codes0, scales0 = ref[0], ref[1]
        zeros0 = None
    mism0 = gpu_codes != codes0
    zmism0 = (gpu_zeros != zeros0) if asym else np.zeros((Wp.shape[0], 1), dtype=bool)
    n0 = int(mism0.sum())
    total = gpu_codes.size
    stats = {"mismatches": n0, "zero_mismatches": int(zmism0.sum()), "total": total,
             "frac": n0 / total, "forced": 0, "iters": 0, "forced_zeros": 0, "max_tie": 0.0}
    codes, scales = codes0.copy(), scales0.copy()
    zeros = zeros0.copy() if asym else None
    rows = np.unique(np.concatenate([np.nonzero(mism0)[0], np.nonzero(zmism0)[0]]))
    if rows.size:
        force = np.full((rows.size, gpu_codes.shape[1]), NO_FORCE, dtype=np.int16)
        fz = np.full((rows.size, scales0.shape[1]), NO_FORCE, dtype=np.int16) if asym else None
        Wr = Wp[rows]
        for it in range(max_iters):
            c, s, z, zv, v = _sweep(Wr, U, bits, g, asym, force, fz)
            d = c != gpu_codes[rows]
            dz = (z != gpu_zeros[rows]) if asym else np.zeros((rows.size, 1), dtype=bool)
            stats["iters"] = it + 1
            if not d.any() and not dz.any():
                codes[rows], scales[rows] = c, s
                if asym:
                    zeros[rows] = z
                break
            for k in np.nonzero(d.any(axis=1) | dz.any(axis=1))[0]:
                j = int(np.argmax(d[k])) if d[k].any() else gpu_codes.shape[1]
                jz = int(np.argmax(dz[k])) if dz[k].any() else None
                if jz is not None and jz * g <= j:   # the group's zero-point differs first
                    td = float(tie_distance(zv[k, jz]))
                    assert td < tie_tol, (
                        f"row {rows[k]} group {jz}: GPU zero-point {gpu_zeros[rows[k], jz]} vs "
                        f"oracle {z[k, jz]} at -lo/scale = {zv[k, jz]!r} (tie distance {td:.3g})")
                    fz[k, jz] = gpu_zeros[rows[k], jz]
                    stats["forced_zeros"] += 1
                    stats["max_tie"] = max(stats["max_tie"], td)
                    continue
                td = float(tie_distance(v[k, j]))
                assert td < tie_tol, (
                    f"row {rows[k]} col {j}: GPU code {gpu_codes[rows[k], j]} vs oracle "
                    f"{c[k, j]} at w/scale = {v[k, j]!r} (tie distance {td:.3g})")
                force[k, j] = gpu_codes[rows[k], j]
                stats["forced"] += 1
                stats["max_tie"] = max(stats["max_tie"], td)
        else:
            raise AssertionError("teacher forcing did not converge")
    if bound == "raw":
        assert n0 + stats["zero_mismatches"] <= MAX_MISMATCH_FRAC * total, (
            f"{n0} of {total} codes (and {stats['zero_mismatches']} zero-points) differ before "
            f"forcing ({stats['forced']} forced tie sites)")
    else:
        assert stats["forced"] + stats["forced_zeros"] <= MAX_MISMATCH_FRAC * total, (
            f"{stats['forced']} of {total} codes decided differently")
    if asym:
        return stats, codes, scales, zeros
    return stats, codes, scales


def rel(a, b):
    return abs(a - b) / max(abs(b), 1e-300)


def unpack_gpu(qweight: torch.Tensor, bits: int) -> np.ndarray:
    return O.unpack_ref(qweight.cpu().numpy().view(np.uint32), bits)


def fp16_scales(scales: torch.Tensor) -> np.ndarray:
    return scales.cpu().numpy().astype(np.float64)
