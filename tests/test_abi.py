"""CPU-side checks of the C ABI: the library loads, exports every function include/wq.h
declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes

import numpy as np
import pytest
import torch


def test_library_exports_every_header_function(wq):
    names = wq.header_functions()
    expected = {"wq_status_string", "wq_last_error", "wq_version", "wq_quantize_dyadic",
                "wq_quantize_lloyd", "wq_pack", "wq_unpack", "wq_dequant", "wq_gemv_w4a16",
                "wq_gemv_w4a16_grouped", "wq_gemm_workspace_bytes", "wq_gemm_w4a16",
                "wq_debug_fail_next_launches", "wq_device_error", "wq_gemm_w4a16_static",
                "wq_gemv_plan_create", "wq_gemv_plan_launch", "wq_gemv_plan_destroy", "wq_gemv_plan_set_overlap",
                "wq_fake_quant_ste", "wq_bf16x_superblocks", "wq_bf16x_count", "wq_bf16x_encode",
                "wq_bf16x_decode", "wq_gumbel_st_backward", "wq_quantize_wf_analyze",
                "wq_quantize_wf_pack", "wq_dequant_wf", "wq_gemv_wf"}
    assert expected <= set(names), set(names) ^ expected
    for n in names:
        assert hasattr(wq._lib, n), n


def test_status_strings_and_version(wq):
    for s in range(7):
        assert wq._lib.wq_status_string(s).decode().startswith("WQ_")
    assert wq._lib.wq_status_string(99).decode() == "unknown wq_status"
    assert wq.version() >= 100


def test_shape_and_group_checks_fail_before_any_cuda_call(wq):
    lib = wq._lib
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    # unsupported group
    assert lib.wq_quantize_dyadic(p, 4, 64, 16, p, p, p, None) == wq.WQ_EUNSUPPORTED
    assert "group" in wq.last_error()
    # k not a multiple of 32 / of the group, non-positive sizes
    assert lib.wq_quantize_dyadic(p, 4, 48, 32, p, p, p, None) == wq.WQ_EINVAL
    assert lib.wq_quantize_dyadic(p, 4, 96, 64, p, p, p, None) == wq.WQ_EINVAL
    assert lib.wq_quantize_dyadic(p, 0, 64, 64, p, p, p, None) == wq.WQ_EINVAL
    assert lib.wq_pack(p, 4, 30, p, None) == wq.WQ_EINVAL
    # NULL weight descriptor, bad batch, bad lloyd params
    assert lib.wq_gemv_w4a16(None, p, 1, p, None) == wq.WQ_EINVAL
    d = wq.WqWeight(wq.FMT_DYADIC4, 64, 4, 64, p.value, p.value)
    assert lib.wq_gemv_w4a16(ctypes.byref(d), p, 17, p, None) == wq.WQ_EINVAL
    d.fmt = 7
    assert lib.wq_dequant(ctypes.byref(d), p, None) == wq.WQ_EINVAL
    prm = wq.WqLloydParams(5, 25)
    assert lib.wq_quantize_lloyd(p, 4, 64, ctypes.byref(prm), p, p, p, None, None, None) == wq.WQ_EINVAL
    prm = wq.WqLloydParams(0, 100)
    assert lib.wq_quantize_lloyd(p, 4, 64, ctypes.byref(prm), p, p, p, None, None, None) == wq.WQ_EINVAL
    assert lib.wq_gemv_w4a16_grouped(None, None, None, 1, 1, None) == wq.WQ_EINVAL
    assert lib.wq_fake_quant_ste(p, 4, 64, 16, p, p, None, None, None) == wq.WQ_EUNSUPPORTED
    assert lib.wq_fake_quant_ste(p, 4, 96, 64, p, p, None, None, None) == wq.WQ_EINVAL
    # BF16X: k % 32, n*k below 2^32, ovf_bytes >= 0
    assert lib.wq_bf16x_superblocks(3, 96) == 2 and lib.wq_bf16x_superblocks(16, 4096) == 256
    assert lib.wq_bf16x_superblocks(4, 40) == -1
    assert lib.wq_bf16x_count(p, 4, 48, p, None) == wq.WQ_EINVAL
    assert lib.wq_bf16x_count(p, 1 << 20, 1 << 12, p, None) == wq.WQ_EINVAL
    assert "2^32" in wq.last_error()
    assert lib.wq_bf16x_encode(p, 4, 64, p, p, p, p, -1, None) == wq.WQ_EINVAL
    assert lib.wq_bf16x_decode(p, p, p, p, 16, 4, 80, p, None) == wq.WQ_EINVAL
    # Gumbel-ST: group, temperature (positive normal finite), shapes
    assert lib.wq_gumbel_st_backward(p, 4, 64, 16, p, 1.0, p, p, None, None) == wq.WQ_EUNSUPPORTED
    for tau in (0.0, -1.0, float("nan"), float("inf"), 1e-39):
        assert lib.wq_gumbel_st_backward(p, 4, 64, 64, p, tau, p, p, None, None) == wq.WQ_EINVAL
    assert "tau" in wq.last_error()
    assert lib.wq_gumbel_st_backward(p, 4, 96, 64, p, 1.0, p, p, None, None) == wq.WQ_EINVAL
    assert lib.wq_gumbel_st_backward(p, 0, 64, 64, p, 1.0, p, p, None, None) == wq.WQ_EINVAL
    # water-filling: k % 64, block offsets below 2^32, lambda >= 0, buffer sizes >= 0
    assert lib.wq_quantize_wf_analyze(p, 4, 96, 0.0, p, p, p, None, None) == wq.WQ_EINVAL
    assert lib.wq_quantize_wf_analyze(p, 1 << 20, 1 << 14, 0.0, p, p, p, None, None) == wq.WQ_EINVAL
    assert "2^32" in wq.last_error()
    assert lib.wq_quantize_wf_analyze(p, 4, 64, -1.0, p, p, p, None, None) == wq.WQ_EINVAL
    assert lib.wq_quantize_wf_analyze(p, 4, 64, float("nan"), p, p, p, None, None) == wq.WQ_EINVAL
    assert lib.wq_quantize_wf_pack(p, 4, 64, p, p, p, p, -1, None) == wq.WQ_EINVAL
    assert lib.wq_dequant_wf(p, -1, p, p, p, 4, 64, p, None) == wq.WQ_EINVAL
    assert lib.wq_dequant_wf(p, 16, p, p, p, 0, 64, p, None) == wq.WQ_EINVAL
    # the water-filled GEMV: the same shape rules, batch 1..16
    assert lib.wq_gemv_wf(p, 16, p, p, p, 4, 96, p, 1, p, None) == wq.WQ_EINVAL
    assert lib.wq_gemv_wf(p, -1, p, p, p, 4, 64, p, 1, p, None) == wq.WQ_EINVAL
    for batch in (0, 17):
        assert lib.wq_gemv_wf(p, 16, p, p, p, 4, 64, p, batch, p, None) == wq.WQ_EINVAL
        assert "batch" in wq.last_error()


def test_gemv_plan_rejects_bad_arguments_and_keeps_nothing(wq):
    lib = wq._lib
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    plan = ctypes.c_void_p(1234)
    d = wq.WqWeight(wq.FMT_DYADIC4, 64, 4, 64, p.value, p.value)
    arr = (ctypes.c_void_p * 1)(p.value)
    assert lib.wq_gemv_plan_create(None, None, None, 1, 1, ctypes.byref(plan)) == wq.WQ_EINVAL
    assert plan.value is None                            # NULL on failure
    assert lib.wq_gemv_plan_create(ctypes.byref(d), arr, arr, 1, 0, ctypes.byref(plan)) == wq.WQ_EINVAL
    assert lib.wq_gemv_plan_create(ctypes.byref(d), arr, arr, 1, 1, None) == wq.WQ_EINVAL
    # host memory is not accepted as a device buffer
    assert lib.wq_gemv_plan_create(ctypes.byref(d), arr, arr, 1, 1, ctypes.byref(plan)) == wq.WQ_EINVAL
    assert plan.value is None
    assert lib.wq_gemv_plan_launch(None, None) == wq.WQ_EINVAL
    assert lib.wq_gemv_plan_set_overlap(None, 1) == wq.WQ_EINVAL
    lib.wq_gemv_plan_destroy(None)                       # a no-op


def test_misaligned_and_host_pointers_are_rejected(wq):
    lib = wq._lib
    buf = (ctypes.c_uint8 * 256)()
    base = ctypes.addressof(buf)
    aligned = (base + 15) // 16 * 16
    st = lib.wq_pack(ctypes.c_void_p(aligned + 1), 2, 64, ctypes.c_void_p(aligned), None)
    assert st == wq.WQ_EALIGN
    # a host pointer is never accepted (no GPU here: the attribute query fails; on a GPU
    # box it reports unregistered host memory) -- either way WQ_EINVAL, nothing launched
    st = lib.wq_pack(ctypes.c_void_p(aligned), 2, 64, ctypes.c_void_p(aligned + 128), None)
    assert st == wq.WQ_EINVAL
    assert "device memory" in wq.last_error() or "cudaPointerGetAttributes" in wq.last_error()


def test_binding_refuses_cpu_tensors(wq):
    with pytest.raises(ValueError):
        wq.quantize_dyadic(torch.zeros(4, 64, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        wq.pack(torch.zeros(4, 64, dtype=torch.uint8))


def test_gemm_workspace_sizes(wq):
    """Host-side GEMM planning (no GPU: the SM count falls back to the B200's 148). Up to 16
    activation rows run on the GEMV and need nothing; on 4096 x 11008, m = 512 splits K two
    ways (64 tiles of 128 x 256) and m = 4096 runs 3 whole waves and splits its last 68
    tiles two ways. LUT16 plans the same launches as DYADIC4 and adds, in front, its scaled
    fp16 activations (2 m k bytes) and the rows' fp32 factors (4 m bytes), each rounded up
    to 1 KB."""
    def ws(fmt, group, n, k, m):
        d = wq.WqWeight(fmt, group, n, k, None, None)
        return int(wq._lib.wq_gemm_workspace_bytes(ctypes.byref(d), m))

    n, k = 4096, 11008
    for fmt, group in [(wq.FMT_DYADIC4, 64), (wq.FMT_LUT16, 64), (wq.FMT_LLOYD8S, 32)]:
        assert ws(fmt, group, n, k, 12) == 0 and ws(fmt, group, n, k, 16) == 0
    assert ws(wq.FMT_DYADIC4, 64, n, k, 4096) == 2 * 68 * 128 * 256 * 4
    # 11008 x 4096 at m = 4096 takes 384-row tiles (6 whole waves + 58 tiles: more than
    # three whole waves) and at m = 2048 has 4 waves + 96 tiles (more than half a wave
    # left): neither splits its last wave
    assert ws(wq.FMT_DYADIC4, 64, 11008, 4096, 4096) == 0
    assert ws(wq.FMT_DYADIC4, 64, 11008, 4096, 2048) == 0
    assert ws(wq.FMT_DYADIC4, 64, n, k, 512) == 16 << 20
    for m in (17, 48, 100, 128, 200, 512, 4096):
        for nn, kk in [(n, k), (11008, 4096), (200, 320)]:
            x_bytes = -(-2 * m * kk // 1024) * 1024 + -(-4 * m // 1024) * 1024
            assert ws(wq.FMT_LUT16, 64, nn, kk, m) == ws(wq.FMT_DYADIC4, 64, nn, kk, m) + x_bytes
    assert ws(wq.FMT_LUT16, 64, n, k, 0) == 0


def test_debug_library_builds_and_exports_every_header_function(wq):
    """The WQ_DEBUG build (device-side index and finite-input checks) is the same ABI."""
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_wq_build", os.path.join(root, "w4a16_matmul_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.build(debug=True)
    lib = ctypes.CDLL(path)
    for n in wq.header_functions():
        assert hasattr(lib, n), n
    lib.wq_status_string.restype = ctypes.c_char_p
    assert lib.wq_status_string(0).decode() == "WQ_OK"
