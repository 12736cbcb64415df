"""The WQ_DEBUG build (libwq_debug.so): kernels check derived indices and the finite-input
precondition on the device and report the first failed check through wq_device_error
(WQ_EDATA) instead of trapping. Run in a child process with WQ_DEBUG=1 (the binding picks
the library at import): each planted NaN / Inf input must be reported with its kernel's
code and leave the context usable, and clean inputs must give the same bits as the normal
build."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, ROOT); sys.path.insert(0, ROOT + "/tests")
import w4a16_matmul_b200 as wq, workloads
from _util import to_dev_bits
assert wq.DEBUG and wq.LIB_PATH.endswith("libwq_debug.so")
dev = "cuda"
def code():
    torch.cuda.synchronize()
    st = wq._lib.wq_device_error(wq.ctypes.byref(c := wq.ctypes.c_int32(0)))
    return st, c.value
out = {}
n, k = 256, 1024
w = workloads.gaussian_outlier_weight(n, k, workloads.DYADIC_1, 3)
wd = to_dev_bits(w)
pw, codes = wq.quantize_dyadic(wd, 64, codes=True)
x = to_dev_bits(workloads.activations(4, k, workloads.DYADIC_1, 3))
y = wq.gemv(pw, x)
out["clean"] = code()
np.save(OUT + "/packed.npy", pw.packed.cpu().numpy())
np.save(OUT + "/y.npy", y.view(torch.int16).cpu().numpy())
wbad = w.copy(); wbad[7, 100] = 0x7FC0                       # NaN weight
wq.quantize_dyadic(to_dev_bits(wbad), 64); out["quantize_nan"] = code()
wq.quantize_lloyd(to_dev_bits(wbad), wq.LLOYD_G32_WARM, 3); out["lloyd_nan"] = code()
wq.quantize_lloyd(to_dev_bits(wbad), wq.LLOYD_KMEANS16, 3); out["kmeans_nan"] = code()
xb = workloads.activations(4, k, workloads.DYADIC_1, 3).copy(); xb[2, 513] = 0x7F80   # +inf
wq.gemv(pw, to_dev_bits(xb)); out["gemv_inf"] = code()
xm = np.tile(workloads.activations(1, k, workloads.DYADIC_1, 4), (48, 1)); xm[40, 9] = 0xFF80
wq.gemm(pw, to_dev_bits(xm)); out["gemm_inf"] = code()
import oracle
g = np.random.default_rng(1)
lut = to_dev_bits(oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01), torch.float16)
pl = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, pw.packed, lut)
wq.gemm(pl, to_dev_bits(xm)); out["gemm_lut16_inf"] = code()
z = torch.randn((n, k), device=dev) * 0.02; z[5, 6] = float("nan")
s = (torch.nan_to_num(z).abs().reshape(n, k // 64, 64).amax(-1)).to(torch.bfloat16)
wq.fake_quant_ste(z, s, 64); out["ste_nan"] = code()
out["after"] = code()
print(repr(out))
'''


def test_debug_build_reports_bad_inputs_and_matches_normal_build(tmp_path):
    env = dict(os.environ, WQ_DEBUG="1")
    src = CHILD.replace("ROOT", repr(ROOT)).replace("OUT", repr(str(tmp_path)))
    r = subprocess.run([sys.executable, "-c", src], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    out = eval(r.stdout.strip().splitlines()[-1])
    EDATA = 6
    assert out["clean"] == (0, 0)
    assert out["quantize_nan"] == (EDATA, 3101)
    assert out["lloyd_nan"] == (EDATA, 3102)
    assert out["kmeans_nan"] == (EDATA, 3103)
    assert out["gemv_inf"] == (EDATA, 3201)
    assert out["gemm_inf"] == (EDATA, 3203)
    assert out["gemm_lut16_inf"] == (EDATA, 3202)
    assert out["ste_nan"] == (EDATA, 3301)
    assert out["after"] == (0, 0)                       # read and cleared; the context lives on
    # the clean results equal the normal build's
    import numpy as np
    import torch
    import w4a16_matmul_b200 as wq
    import workloads
    from _util import to_dev_bits
    assert not wq.DEBUG
    w = workloads.gaussian_outlier_weight(256, 1024, workloads.DYADIC_1, 3)
    pw, _ = wq.quantize_dyadic(to_dev_bits(w), 64, codes=True)
    y = wq.gemv(pw, to_dev_bits(workloads.activations(4, 1024, workloads.DYADIC_1, 3)))
    assert np.array_equal(pw.packed.cpu().numpy(), np.load(tmp_path / "packed.npy"))
    assert np.array_equal(y.view(torch.int16).cpu().numpy(), np.load(tmp_path / "y.npy"))
