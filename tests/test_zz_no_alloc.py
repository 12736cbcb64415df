"""wq_gemm_w4a16_static: the GEMM for callers that cannot allocate device memory (its
split-K scratch lives in a static device array of the library). Called through the C ABI,
on two calls in a row, and compared within the tolerance of the other GEMM tests both with
the oracle's fp64 product and with wq_gemm_w4a16 given a caller workspace. This file is
collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import f32, matmul_tolerance, to_dev, to_dev_bits

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["dyadic", "lut16", "lut16_small_x"])
def test_static_scratch_gemm_matches_workspace_gemm(wq, fmt):
    """LUT16 also keeps its scaled fp16 copy of the activations and their row factors in the
    scratch; lut16_small_x feeds it activations around 1e-8, mixed with 1e2 in odd rows."""
    n, k, m = 1024, 8192, 48                  # small m: K is split, so the scratch is used
    if fmt == "dyadic":
        w_bits = workloads.gaussian_outlier_weight(n, k, workloads.PREFILL, 21)
        s, c = oracle.dyadic_quantize(w_bits, 64)
        code, aux = oracle.DYADIC4, s
    else:
        g = np.random.default_rng(21)
        c = g.integers(0, 16, (n, k), dtype=np.uint8)
        code, aux = oracle.LUT16, oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    packed = oracle.pack(c)
    if fmt == "dyadic":
        pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(aux))
    else:
        pw = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(aux, torch.float16))
    d = pw.desc()
    need = wq.gemm_workspace_bytes(pw, m)
    assert 0 < need <= (16 << 20)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rows = np.arange(0, n, 5)
    for call in range(2):
        x_bits = workloads.activations(m, k, workloads.PREFILL, 100 + call)
        if fmt == "lut16_small_x":
            xv = oracle.bf16_to_f64(x_bits) * 1e-8
            xv[1::2, ::3] *= 1e10
            x_bits = workloads.f64_to_bf16_bits(xv)
        x = to_dev_bits(x_bits)
        y_static = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        st = wq._lib.wq_gemm_w4a16_static(ctypes.byref(d), ctypes.c_void_p(x.data_ptr()), m,
                                          ctypes.c_void_p(y_static.data_ptr()), stream)
        assert st == wq.WQ_OK, wq.last_error()
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        y_ws = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        st = wq._lib.wq_gemm_w4a16(ctypes.byref(d), ctypes.c_void_p(x.data_ptr()), m,
                                   ctypes.c_void_p(y_ws.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                   need, stream)
        assert st == wq.WQ_OK, wq.last_error()
        torch.cuda.synchronize()
        y_ref, bound = oracle.matmul_rows(code, packed, aux, 64, x_bits, rows=rows)
        a, b = f32(y_static)[:, rows], f32(y_ws)[:, rows]
        assert np.all(np.abs(a - y_ref) <= matmul_tolerance(y_ref, bound))
        assert np.all(np.abs(b - y_ref) <= matmul_tolerance(y_ref, bound))
        assert np.all(np.abs(a - b) <= matmul_tolerance(b, bound))
        assert wq.device_error() == 0


def test_static_scratch_gemm_rejects_oversized_problems(wq):
    tiny = torch.zeros(16, dtype=torch.uint8, device="cuda")
    shape = None
    for n, k, m in [(4224, 8192, 256), (2176, 16384, 256), (4224, 16384, 256)]:
        probe = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, tiny, tiny)
        if wq.gemm_workspace_bytes(probe, m) > (16 << 20):
            shape = (n, k, m)
            break
    assert shape is not None
    n, k, m = shape
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k,
                         torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda"),
                         torch.zeros((n, k // 64), dtype=torch.bfloat16, device="cuda"))
    d = pw.desc()
    x = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    st = wq._lib.wq_gemm_w4a16_static(ctypes.byref(d), ctypes.c_void_p(x.data_ptr()), m,
                                      ctypes.c_void_p(y.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == wq.WQ_EINVAL and "static scratch" in wq.last_error()
