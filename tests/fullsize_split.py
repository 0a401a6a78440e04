"""Full-size parity of the 70B-shaped layer, split across two hosts.

The oracle's float64 H (32768 x 28672^2) and U (28672^3) take several minutes
of host time, which a GPU host would spend idle.  So the comparison splits:

  python tests/fullsize_split.py --dump gpurun_out/c4_rows.npz   # GPU host
  python tests/fullsize_split.py --check gpurun_out/c4_rows.npz  # any host

--dump runs the layer at full size for 4 and 3 bits and saves, for 256 rows
drawn with a fixed seed, the GPU's codes (memory order) and fp16 scales, with
the perm, g_idx and the reported output error.  --check rebuilds the same
seeded inputs, builds H and U in float64, sweeps the sampled rows with the
oracle's blocked loop and compares them teacher-forced under the contract of
tests/parity.py (raw mismatches at most 0.1% of the codes, every differing
decision within 1e-4 of a rounding tie), and the scales within 1e-3.  The
oracle here is test infrastructure, as everywhere under tests/.
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from workloads import C4, make_weight, make_x_bits  # noqa: E402

N_ROWS = 256
BITS = (4, 3)


def _rows(out: int) -> np.ndarray:
    return np.sort(np.random.default_rng(77).choice(out, N_ROWS, replace=False))


def dump(path: str) -> None:
    import torch

    import post_int4_weight_gptq_b200 as piq
    from tests.parity import to_gpu_w, to_gpu_x, unpack_gpu
    spec = C4
    W, X = make_weight(spec), make_x_bits(spec)
    Wg, Xg = to_gpu_w(W), to_gpu_x(X)
    rows = _rows(W.shape[0])
    res = {"rows": rows}
    for bits in BITS:
        out = piq.gptq_quantize_layer(Wg, Xg, bits=bits, g=spec.g, damp=spec.damp,
                                      act_order=spec.act_order)
        torch.cuda.synchronize()
        res[f"codes{bits}"] = unpack_gpu(out.qweight, bits)[rows].astype(np.int8)
        res[f"scales{bits}"] = out.scales.cpu().numpy()[rows]
        res[f"perm{bits}"] = out.perm.cpu().numpy()
        res[f"g_idx{bits}"] = out.g_idx.cpu().numpy()
        res[f"err{bits}"] = np.float64(out.err)
    np.savez_compressed(path, **res)
    print(f"dumped {N_ROWS} rows x {W.shape[1]} columns for bits {BITS} to {path}")


def check(path: str) -> int:
    import oracle as O
    from oracle.gptq import gptq_sweep_blocked_ref
    from tests.parity import REL_TOL, teacher_forced_compare
    spec = C4
    d = np.load(path)
    rows = d["rows"]
    t0 = time.time()
    W, X = make_weight(spec), make_x_bits(spec)
    H = O.hessian_ref(X)
    del X
    perm, U, _ = O.gptq_prepare_ref(H, spec.damp, spec.act_order)
    del H
    print(f"oracle H and U: {time.time() - t0:.0f} s", flush=True)
    Wp = W.astype(np.float64)[:, perm][rows]
    fails = 0
    for bits in BITS:
        assert np.array_equal(d[f"perm{bits}"], perm)
        assert np.array_equal(d[f"g_idx{bits}"], O.g_idx_ref(perm, spec.g))
        codes = d[f"codes{bits}"].astype(np.int64)[:, perm]
        ref = gptq_sweep_blocked_ref(Wp, U, bits, spec.g)
        try:
            stats, _, s_ref = teacher_forced_compare(codes, Wp, U, bits, spec.g, ref=ref)
            s16 = s_ref.astype(np.float16).astype(np.float64)
            sc = d[f"scales{bits}"].astype(np.float64)
            live = s16 > 0
            srel = float((np.abs(sc[live] - s16[live]) / s16[live]).max())
            assert srel < REL_TOL, srel
            print(f"{bits}-bit, {N_ROWS} sampled rows: {stats}; scales max rel {srel:.2e}; "
                  f"GPU error {float(d[f'err{bits}']):.6g}", flush=True)
        except AssertionError as exc:
            fails += 1
            print(f"{bits}-bit FAILED: {exc}", flush=True)
    return 1 if fails else 0


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    g = ap.add_mutually_exclusive_group(required=True)
    g.add_argument("--dump", metavar="NPZ")
    g.add_argument("--check", metavar="NPZ")
    a = ap.parse_args()
    if a.dump:
        dump(a.dump)
        return 0
    return check(a.check)


if __name__ == "__main__":
    sys.exit(main())
