"""Failure detection on the GPU without a GPU fault.

* A bounded device wait that runs out: piq_wait_selftest makes one block wait,
  through the library's own bounded-wait code, on a barrier nothing completes;
  the status word must come back PIQ_ERR_TIMEOUT after about the limit, and the
  same context must then run a normal GPTQ call correctly.
* Host-side injection (PIQ_FAULT): the binding raises PiqError with the
  injected status and the context stays usable.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
import post_int4_weight_gptq_b200 as piq
from tests.parity import teacher_forced_compare, to_gpu_w, to_gpu_x, unpack_gpu
from workloads import make_weight, make_x_bits, small_spec

pytestmark = pytest.mark.gpu


def _small_gptq_ok():
    spec = small_spec(64, 256, 1024, seed=5, sigma_ln=0.8)
    W, X = make_weight(spec), make_x_bits(spec)
    out = piq.gptq_quantize_layer(to_gpu_w(W), to_gpu_x(X), bits=4, g=128)
    H = O.hessian_ref(X)
    perm, U, _ = O.gptq_prepare_ref(H, 0.01, False)
    teacher_forced_compare(unpack_gpu(out.qweight, 4), W.astype(np.float64), U, 4, 128)


@pytest.mark.parametrize("wait_ns", [1_000_000, 20_000_000])
def test_bounded_wait_runs_out(wait_ns):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    rc, where = piq.wait_selftest(wait_ns)
    dt = time.perf_counter() - t0
    assert rc == piq.PIQ_ERR_TIMEOUT, piq.status_string(rc)
    assert where == 901
    assert dt >= wait_ns * 1e-9
    assert dt < 5.0
    _small_gptq_ok()


@pytest.mark.parametrize("value,status", [("notpd", piq.PIQ_ERR_NOT_PD),
                                          ("timeout", piq.PIQ_ERR_TIMEOUT),
                                          ("oom", piq.PIQ_ERR_CUDA)])
def test_injected_fault_then_normal_call(monkeypatch, value, status):
    spec = small_spec(32, 128, 256, seed=6)
    Wg, Xg = to_gpu_w(make_weight(spec)), to_gpu_x(make_x_bits(spec))
    monkeypatch.setenv("PIQ_FAULT", value)
    with pytest.raises(piq.PiqError) as e:
        piq.gptq_quantize_layer(Wg, Xg, bits=4, g=128)
    assert e.value.status == status
    monkeypatch.delenv("PIQ_FAULT")
    _small_gptq_ok()
