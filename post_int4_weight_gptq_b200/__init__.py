"""B200 (sm_100a) layer-wise INT4/INT3 weight quantization: GPTQ and AWQ.

A thin binding over the C ABI of ``lib/libpiq.so`` (declared in
``include/piq.h``).  The functions here only marshal arguments: PyTorch
supplies device memory and the current CUDA stream, and every step of the
quantization runs in the library's own CUDA kernels.  There is no CPU path:
if the library is missing or the device is not a B200, calls raise.

Methods (web pages on the subject, cited by title and section):
* GPTQ - "GPTQ versus AWQ objectives", "A strong answer" (the column loop with
  error feedback through the upper Cholesky factor of the inverse proxy
  Hessian, group scales, block-batched updates) and "What interviewers probe
  next" (act-order, damping).
* AWQ  - same page, AWQ paragraph: per-channel scales mean|x_j|^alpha, one
  alpha per layer by grid search on the calibration output error.
* AWQ then GPTQ - same page, the serving decision list: the two compose, AWQ's
  scaling first and GPTQ's rounding after (GPTQ on W diag(s), X diag(1/s)).
"""
from __future__ import annotations

import collections
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libpiq.so")

PIQ_OK = 0
PIQ_ERR_INVALID_ARG = -1
PIQ_ERR_WORKSPACE_TOO_SMALL = -2
PIQ_ERR_NOT_PD = -3
PIQ_ERR_CUDA = -4
PIQ_ERR_TIMEOUT = -5
PIQ_ERR_UNSUPPORTED_DEVICE = -6

AWQ_DEFAULT_GRID = tuple(k / 20.0 for k in range(20))

_c_i64 = ctypes.c_int64
_c_int = ctypes.c_int
_c_float = ctypes.c_float
_c_size_p = ctypes.POINTER(ctypes.c_size_t)
_vp = ctypes.c_void_p

# name -> (restype, argtypes); kept in the order of include/piq.h
SIGNATURES = {
    "piq_status_string": (ctypes.c_char_p, [_c_int]),
    "piq_hessian_bytes": (_c_int, [_c_i64, _c_size_p]),
    "piq_hessian": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_int, _vp]),
    "piq_upper_factor_workspace_bytes": (_c_int, [_c_i64, _c_size_p]),
    "piq_upper_factor": (_c_int, [_vp, _c_i64, _c_float, _vp, _vp,
                                  ctypes.POINTER(ctypes.c_double), _vp, ctypes.c_size_t, _vp]),
    "piq_gptq_sweep_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_size_p]),
    "piq_gptq_sweep": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_int, _c_int, _vp, _vp, _vp,
                                ctypes.c_size_t, _vp]),
    "piq_gptq_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_i64, _c_int, _c_int, _c_size_p]),
    "gptq_quantize_layer": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_i64, _c_int, _c_int, _c_float,
                                     _c_int, _vp, _vp, _vp, _vp,
                                     ctypes.POINTER(ctypes.c_double), _vp, ctypes.c_size_t,
                                     _vp]),
    "piq_layer_statistics_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_size_p]),
    "piq_layer_statistics": (_c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "piq_gptq_from_h_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_int, _c_size_p]),
    "gptq_quantize_rows_from_h": (_c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _c_int, _c_int,
                                           _c_float, _c_int, _vp, _vp, _vp, _vp, _vp,
                                           ctypes.POINTER(ctypes.c_double), _vp,
                                           ctypes.c_size_t, _vp]),
    "gptq_quantize_layer_asym": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_i64, _c_int, _c_int,
                                          _c_float, _c_int, _vp, _vp, _vp, _vp, _vp,
                                          ctypes.POINTER(ctypes.c_double), _vp, ctypes.c_size_t,
                                          _vp]),
    "piq_awq_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_i64, _c_int, _c_size_p]),
    "awq_search_layer": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_i64, _c_int, _c_int,
                                  ctypes.POINTER(ctypes.c_float), _c_int,
                                  ctypes.POINTER(ctypes.c_float), _vp, _vp, _vp,
                                  ctypes.POINTER(ctypes.c_double), _vp, ctypes.c_size_t, _vp]),
    "awq_gptq_quantize_layer": (_c_int, [_vp, _c_i64, _c_i64, _vp, _c_i64, _vp, _c_int, _c_int,
                                         _c_float, _c_int, _vp, _vp, _vp, _vp,
                                         ctypes.POINTER(ctypes.c_double), _vp, ctypes.c_size_t,
                                         _vp]),
    "piq_rtn_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_size_p]),
    "piq_rtn_quantize_layer": (_c_int, [_vp, _c_i64, _c_i64, _c_int, _c_int, _vp, _vp, _vp,
                                        ctypes.c_size_t, _vp]),
    "piq_output_error_workspace_bytes": (_c_int, [_c_i64, _c_i64, _c_i64, _c_size_p]),
    "piq_layer_output_error": (_c_int, [_vp, _c_i64, _c_i64, _vp, _vp, _vp, _vp, _vp, _c_int,
                                        _c_int, _vp, _c_i64, ctypes.POINTER(ctypes.c_double), _vp,
                                        ctypes.c_size_t, _vp]),
    "piq_set_timing": (_c_int, [_c_int]),
    "piq_last_phase_times": (_c_int, [ctypes.POINTER(ctypes.c_double), _c_int,
                                      ctypes.POINTER(_c_int)]),
    "piq_phase_name": (ctypes.c_char_p, [_c_int]),
    "piq_last_gemm_stats": (_c_int, [ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_c_int)]),
    "piq_gemm_tile_order": (_c_i64, [_c_int, _c_int, _c_int, _c_i64, _vp, _vp]),
    "piq_kernel_launches": (ctypes.c_uint64, []),
    "piq_simt_gemm_fallbacks": (ctypes.c_uint64, []),
    "piq_last_cuda_error": (ctypes.c_char_p, []),
    "piq_wait_selftest": (_c_int, [ctypes.c_uint64, ctypes.POINTER(_c_int), _vp, ctypes.c_size_t,
                                   _vp]),
    "piq_upper_factor_noalloc": (_c_int, [_vp, _c_i64, _c_float, _vp, _vp,
                                          ctypes.POINTER(ctypes.c_double), _vp]),
}

_lib = None


class PiqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def load_library(path: str = LIB_PATH):
    """Load libpiq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m post_int4_weight_gptq_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().piq_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc != PIQ_OK:
        if rc == PIQ_ERR_CUDA:
            where = f"{where} [{load_library().piq_last_cuda_error().decode()}]"
        raise PiqError(rc, where)


def last_cuda_error() -> str:
    """The last CUDA runtime error the library saw ('' if none)."""
    return load_library().piq_last_cuda_error().decode()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes: int, device, workspace=None):
    if workspace is not None and workspace.numel() >= nbytes:
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _query(fn, *args) -> int:
    out = ctypes.c_size_t(0)
    _check(fn(*args, ctypes.byref(out)), fn.__name__)
    return int(out.value)


# ------------------------------------------------------------------ entry points
def hessian_bytes(inp: int) -> int:
    return _query(load_library().piq_hessian_bytes, inp)


def hessian(X, H=None, accumulate=False, stream=None):
    """H = X^T X (upper triangle valid), fp32 [in, in]."""
    lib = load_library()
    _need(X, torch.bfloat16, "X")
    n, inp = X.shape
    if H is None:
        H = torch.empty(inp, inp, dtype=torch.float32, device=X.device)
    _need(H, torch.float32, "H")
    _check(lib.piq_hessian(_ptr(X), n, inp, _ptr(H), int(bool(accumulate)), _stream(stream)),
           "piq_hessian")
    return H


def upper_factor(H, damp=0.01, perm=None, stream=None, workspace=None):
    """(U, lambda): U upper with inv(H[perm][:, perm] + lambda I) = U^T U."""
    lib = load_library()
    _need(H, torch.float32, "H")
    inp = H.shape[0]
    if perm is not None:
        _need(perm, torch.int32, "perm")
    U = torch.empty_like(H)
    ws = _workspace(_query(lib.piq_upper_factor_workspace_bytes, inp), H.device, workspace)
    lam = ctypes.c_double(0.0)
    _check(lib.piq_upper_factor(_ptr(H), inp, float(damp), _ptr(perm), _ptr(U), ctypes.byref(lam),
                                _ptr(ws), ws.numel(), _stream(stream)), "piq_upper_factor")
    return U, lam.value


def gptq_sweep(Wp, U, bits=4, g=128, stream=None, workspace=None):
    """(codes int8 [out, in], qscale fp32 [out, ceil(in/g)]) in quantization order."""
    lib = load_library()
    _need(Wp, torch.float32, "Wp")
    _need(U, torch.float32, "U")
    out, inp = Wp.shape
    codes = torch.empty(out, inp, dtype=torch.int8, device=Wp.device)
    qscale = torch.empty(out, -(-inp // g), dtype=torch.float32, device=Wp.device)
    ws = _workspace(_query(lib.piq_gptq_sweep_workspace_bytes, out, inp), Wp.device, workspace)
    _check(lib.piq_gptq_sweep(_ptr(Wp), out, inp, _ptr(U), bits, g, _ptr(codes), _ptr(qscale),
                              _ptr(ws), ws.numel(), _stream(stream)), "piq_gptq_sweep")
    return codes, qscale


GPTQOutput = collections.namedtuple("GPTQOutput", "qweight scales perm g_idx err zeros",
                                    defaults=(None,))
AWQOutput = collections.namedtuple("AWQOutput", "best_alpha s qweight scales err_per_alpha")


def gptq_workspace_bytes(out, inp, n, act_order=False, g=128) -> int:
    return _query(load_library().piq_gptq_workspace_bytes, out, inp, n, int(g),
                  int(bool(act_order)))


def gptq_quantize_layer(W, X, bits=4, g=128, damp=0.01, act_order=False, with_error=True,
                        stream=None, workspace=None, out=None, sym=True):
    """GPTQ of one layer W [out, in] (fp32) on calibration X [n, in] (bf16).
    sym=False: a scale and a zero-point per group (gptq_quantize_layer_asym);
    the zero-points come back in ``zeros`` (uint8 [out, ceil(in/g)])."""
    lib = load_library()
    _need(W, torch.float32, "W")
    _need(X, torch.bfloat16, "X")
    rows, inp = W.shape
    n = X.shape[0]
    if X.shape[1] != inp:
        raise ValueError("W and X disagree on the input dimension")
    dev = W.device
    ng = -(-inp // g)
    if out is None:
        out = GPTQOutput(torch.empty(rows, inp // 8, dtype=torch.int32, device=dev),
                         torch.empty(rows, ng, dtype=torch.float16, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev), None,
                         None if sym else torch.empty(rows, ng, dtype=torch.uint8, device=dev))
    ws = _workspace(gptq_workspace_bytes(rows, inp, n, act_order, g), dev, workspace)
    err = ctypes.c_double(0.0)
    eptr = ctypes.byref(err) if with_error else None
    if sym:
        rc = lib.gptq_quantize_layer(_ptr(W), rows, inp, _ptr(X), n, bits, g, float(damp),
                                     int(bool(act_order)), _ptr(out.qweight), _ptr(out.scales),
                                     _ptr(out.perm), _ptr(out.g_idx), eptr, _ptr(ws),
                                     ws.numel(), _stream(stream))
        _check(rc, "gptq_quantize_layer")
    else:
        _need(out.zeros, torch.uint8, "zeros")
        rc = lib.gptq_quantize_layer_asym(_ptr(W), rows, inp, _ptr(X), n, bits, g, float(damp),
                                          int(bool(act_order)), _ptr(out.qweight),
                                          _ptr(out.scales), _ptr(out.zeros), _ptr(out.perm),
                                          _ptr(out.g_idx), eptr, _ptr(ws), ws.numel(),
                                          _stream(stream))
        _check(rc, "gptq_quantize_layer_asym")
    return out._replace(err=err.value if with_error else None)


def layer_statistics(X, want_sumsq=True, stream=None, workspace=None):
    """(H, sumsq) of one shard of calibration samples X [n, in] (bf16): H fp64
    [in, in] (upper triangle = X^T X), sumsq fp64 [in] (the act-order key) or
    None.  Shards add up: the layer's statistics are their sums."""
    lib = load_library()
    _need(X, torch.bfloat16, "X")
    n, inp = X.shape
    H = torch.empty(inp, inp, dtype=torch.float64, device=X.device)
    sq = torch.empty(inp, dtype=torch.float64, device=X.device) if want_sumsq else None
    ws = _workspace(_query(lib.piq_layer_statistics_workspace_bytes, n, inp), X.device, workspace)
    _check(lib.piq_layer_statistics(_ptr(X), n, inp, _ptr(H), _ptr(sq), _ptr(ws), ws.numel(),
                                    _stream(stream)), "piq_layer_statistics")
    return H, sq


def gptq_rows_from_h(W, H, sumsq=None, bits=4, g=128, damp=0.01, act_order=False, sym=True,
                     with_error=True, stream=None, workspace=None):
    """GPTQ of the rows W [rows, in] (fp32) of a layer whose statistics H (fp64,
    upper triangle of X^T X) and sumsq (fp64 act-order key) are given.  Returns
    a GPTQOutput; err is these rows' share of the layer's output error."""
    lib = load_library()
    _need(W, torch.float32, "W")
    _need(H, torch.float64, "H")
    if sumsq is not None:
        _need(sumsq, torch.float64, "sumsq")
    rows, inp = W.shape
    dev = W.device
    ng = -(-inp // g)
    out = GPTQOutput(torch.empty(rows, inp // 8, dtype=torch.int32, device=dev),
                     torch.empty(rows, ng, dtype=torch.float16, device=dev),
                     torch.empty(inp, dtype=torch.int32, device=dev),
                     torch.empty(inp, dtype=torch.int32, device=dev), None,
                     None if sym else torch.empty(rows, ng, dtype=torch.uint8, device=dev))
    ws = _workspace(_query(lib.piq_gptq_from_h_workspace_bytes, rows, inp, int(g)), dev,
                    workspace)
    err = ctypes.c_double(0.0)
    eptr = ctypes.byref(err) if with_error else None
    rc = lib.gptq_quantize_rows_from_h(_ptr(W), rows, inp, _ptr(H), _ptr(sumsq), bits, g,
                                       float(damp), int(bool(act_order)), _ptr(out.qweight),
                                       _ptr(out.scales), _ptr(out.zeros), _ptr(out.perm),
                                       _ptr(out.g_idx), eptr, _ptr(ws), ws.numel(),
                                       _stream(stream))
    _check(rc, "gptq_quantize_rows_from_h")
    return out._replace(err=err.value if with_error else None)


def awq_workspace_bytes(out, inp, n, n_alpha) -> int:
    return _query(load_library().piq_awq_workspace_bytes, out, inp, n, n_alpha)


def awq_search_layer(W, X, bits=4, g=128, alpha_grid=AWQ_DEFAULT_GRID, stream=None,
                     workspace=None):
    """AWQ scale search of one layer; returns the chosen alpha, s, packed codes, scales, errors."""
    lib = load_library()
    _need(W, torch.float32, "W")
    _need(X, torch.bfloat16, "X")
    rows, inp = W.shape
    n = X.shape[0]
    na = len(alpha_grid)
    dev = W.device
    grid = (ctypes.c_float * na)(*[float(a) for a in alpha_grid])
    errs = (ctypes.c_double * na)()
    best = ctypes.c_float(0.0)
    s = torch.empty(inp, dtype=torch.float32, device=dev)
    qweight = torch.empty(rows, inp // 8, dtype=torch.int32, device=dev)
    scales = torch.empty(rows, -(-inp // g), dtype=torch.float16, device=dev)
    ws = _workspace(awq_workspace_bytes(rows, inp, n, na), dev, workspace)
    _check(lib.awq_search_layer(_ptr(W), rows, inp, _ptr(X), n, bits, g, grid, na,
                                ctypes.byref(best), _ptr(s), _ptr(qweight), _ptr(scales), errs,
                                _ptr(ws), ws.numel(), _stream(stream)), "awq_search_layer")
    return AWQOutput(best.value, s, qweight, scales, list(errs))


def awq_gptq_quantize_layer(W, X, s, bits=4, g=128, damp=0.01, act_order=False,
                            with_error=True, stream=None, workspace=None, out=None):
    """GPTQ of the AWQ-scaled layer W diag(s) on inputs X diag(1/s).  The
    scales quantize W diag(s): the layer's weight is code * scale / s_j."""
    lib = load_library()
    _need(W, torch.float32, "W")
    _need(X, torch.bfloat16, "X")
    _need(s, torch.float32, "s")
    rows, inp = W.shape
    n = X.shape[0]
    if X.shape[1] != inp or s.numel() != inp:
        raise ValueError("W, X and s disagree on the input dimension")
    dev = W.device
    if out is None:
        out = GPTQOutput(torch.empty(rows, inp // 8, dtype=torch.int32, device=dev),
                         torch.empty(rows, -(-inp // g), dtype=torch.float16, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev),
                         torch.empty(inp, dtype=torch.int32, device=dev), None)
    ws = _workspace(gptq_workspace_bytes(rows, inp, n, act_order, g), dev, workspace)
    err = ctypes.c_double(0.0)
    _check(lib.awq_gptq_quantize_layer(_ptr(W), rows, inp, _ptr(X), n, _ptr(s), bits, g,
                                       float(damp), int(bool(act_order)), _ptr(out.qweight),
                                       _ptr(out.scales), _ptr(out.perm), _ptr(out.g_idx),
                                       ctypes.byref(err) if with_error else None, _ptr(ws),
                                       ws.numel(), _stream(stream)), "awq_gptq_quantize_layer")
    return out._replace(err=err.value if with_error else None)


def awq_then_gptq_layer(W, X, bits=4, g=128, damp=0.01, act_order=False,
                        alpha_grid=AWQ_DEFAULT_GRID, stream=None):
    """AWQ's search picks alpha* and s, then GPTQ rounds W diag(s):
    (AWQOutput, GPTQOutput); two library calls on the same stream."""
    a = awq_search_layer(W, X, bits, g, alpha_grid, stream=stream)
    return a, awq_gptq_quantize_layer(W, X, a.s, bits, g, damp, act_order, stream=stream)


def rtn_quantize_layer(W, bits=4, g=128, stream=None, workspace=None):
    """Plain group round-to-nearest: (qweight, scales)."""
    lib = load_library()
    _need(W, torch.float32, "W")
    rows, inp = W.shape
    dev = W.device
    qweight = torch.empty(rows, inp // 8, dtype=torch.int32, device=dev)
    scales = torch.empty(rows, -(-inp // g), dtype=torch.float16, device=dev)
    ws = _workspace(_query(lib.piq_rtn_workspace_bytes, rows, inp), dev, workspace)
    _check(lib.piq_rtn_quantize_layer(_ptr(W), rows, inp, bits, g, _ptr(qweight), _ptr(scales),
                                      _ptr(ws), ws.numel(), _stream(stream)),
           "piq_rtn_quantize_layer")
    return qweight, scales


def output_error_workspace_bytes(out, inp, n) -> int:
    return _query(load_library().piq_output_error_workspace_bytes, out, inp, n)


def layer_output_error(W, qweight, scales, X, bits=4, g=128, g_idx=None, s=None, stream=None,
                       workspace=None, zeros=None) -> float:
    """||X W^T - X What^T||^2 of a packed layer on inputs X."""
    lib = load_library()
    _need(W, torch.float32, "W")
    _need(X, torch.bfloat16, "X")
    rows, inp = W.shape
    n = X.shape[0]
    ws = _workspace(_query(lib.piq_output_error_workspace_bytes, rows, inp, n), W.device,
                    workspace)
    e = ctypes.c_double(0.0)
    _check(lib.piq_layer_output_error(_ptr(W), rows, inp, _ptr(qweight), _ptr(scales),
                                      _ptr(zeros), _ptr(g_idx), _ptr(s), bits, g, _ptr(X), n,
                                      ctypes.byref(e), _ptr(ws), ws.numel(), _stream(stream)),
           "piq_layer_output_error")
    return e.value


def set_timing(enable: bool):
    load_library().piq_set_timing(int(bool(enable)))


def last_phase_times() -> dict:
    lib = load_library()
    buf = (ctypes.c_double * 8)()
    n = ctypes.c_int(0)
    lib.piq_last_phase_times(buf, 8, ctypes.byref(n))
    return {lib.piq_phase_name(i).decode(): buf[i] for i in range(min(n.value, 8))}


def last_gemm_stats() -> dict:
    """With timing on: the INT8 digit GEMM launches of the last timed call,
    {"ms": summed device time, "int8_ops": algorithmic operations, "launches": n}."""
    lib = load_library()
    ms, ops, n = ctypes.c_double(0.0), ctypes.c_double(0.0), ctypes.c_int(0)
    lib.piq_last_gemm_stats(ctypes.byref(ms), ctypes.byref(ops), ctypes.byref(n))
    return {"ms": ms.value, "int8_ops": ops.value, "launches": n.value}


def gemm_tile_order(m_tiles: int, n_tiles: int, lower: bool = False):
    """(mt, nt): int32 arrays, the row and column tile of each tile of an INT8
    digit GEMM launch in the order its CTAs take them (host only)."""
    import numpy as np
    lib = load_library()
    total = int(lib.piq_gemm_tile_order(m_tiles, n_tiles, int(bool(lower)), 0, None, None))
    if total < 0:
        _check(total, "piq_gemm_tile_order")
    mt = np.empty(total, dtype=np.int32)
    nt = np.empty(total, dtype=np.int32)
    rc = int(lib.piq_gemm_tile_order(m_tiles, n_tiles, int(bool(lower)), total,
                                     mt.ctypes.data, nt.ctypes.data))
    if rc < 0:
        _check(rc, "piq_gemm_tile_order")
    return mt, nt


def kernel_launches() -> int:
    """Kernels launched by libpiq in this process so far."""
    return int(load_library().piq_kernel_launches())


def simt_gemm_fallbacks() -> int:
    """FP32-accurate GEMMs that ran on the SIMT kernel instead of the tensor
    cores (an operand not 16-byte aligned), in this process so far."""
    return int(load_library().piq_simt_gemm_fallbacks())


def wait_selftest(wait_ns=1_000_000, stream=None, workspace=None):
    """Run out one bounded device wait (a barrier nothing completes) with the
    given limit.  Returns (status, where): PIQ_ERR_TIMEOUT is the expected
    status.  Does not raise for it."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(256, dev, workspace)
    where = ctypes.c_int(0)
    rc = lib.piq_wait_selftest(int(wait_ns), ctypes.byref(where), _ptr(ws), ws.numel(),
                               _stream(stream))
    return rc, where.value


NOALLOC_MAX_IN = 512


def upper_factor_noalloc(H, damp=0.01, perm=None, stream=None):
    """upper_factor for callers that must not allocate device memory: the
    scratch is a fixed region inside the library (in <= NOALLOC_MAX_IN).  Only
    the output U is created here (pass-through of the C entry point)."""
    lib = load_library()
    _need(H, torch.float32, "H")
    if perm is not None:
        _need(perm, torch.int32, "perm")
    U = torch.empty_like(H)
    lam = ctypes.c_double(0.0)
    _check(lib.piq_upper_factor_noalloc(_ptr(H), H.shape[0], float(damp), _ptr(perm), _ptr(U),
                                        ctypes.byref(lam), _stream(stream)),
           "piq_upper_factor_noalloc")
    return U, lam.value
