"""GPU parity of dyadic quantisation, packing and reconstruction against the oracle:
bit-exact codes, scales, packed bytes and dequantised bf16 on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, to_dev, to_dev_bits

pytestmark = pytest.mark.gpu


def _quant_both(wq, w_bits, group):
    w = to_dev_bits(w_bits)
    pw, codes = wq.quantize_dyadic(w, group, codes=True)
    torch.cuda.synchronize()
    s_ref, c_ref = oracle.dyadic_quantize(w_bits, group)
    return pw, codes, s_ref, c_ref


@pytest.mark.parametrize("n,k,group", [(1, 64, 64), (3, 320, 64), (37, 96, 32), (5, 32, 32),
                                       (129, 2048, 64), (64, 5632, 64), (17, 4160, 32)])
def test_quantize_pack_dequant_bit_exact(wq, n, k, group):
    w_bits = workloads.gaussian_outlier_weight(n, k, workloads.DYADIC_1, n * 1000 + k)
    pw, codes, s_ref, c_ref = _quant_both(wq, w_bits, group)
    assert np.array_equal(bits(pw.aux), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(pw.packed.cpu().numpy(), oracle.pack(c_ref))
    d = wq.dequant(pw)
    assert np.array_equal(bits(d), oracle.dequant(oracle.DYADIC4, oracle.pack(c_ref), s_ref, group))


def test_full_size_single_matrix_2048(wq):
    """The 2048x2048 single-matrix workload, whole matrix compared bit for bit."""
    w_bits = workloads.gaussian_outlier_weight(2048, 2048, workloads.DYADIC_1, 0)
    pw, codes, s_ref, c_ref = _quant_both(wq, w_bits, 64)
    assert np.array_equal(bits(pw.aux), s_ref)
    assert np.array_equal(pw.packed.cpu().numpy(), oracle.pack(c_ref))
    assert np.array_equal(bits(wq.dequant(pw)), oracle.dequant(oracle.DYADIC4, oracle.pack(c_ref), s_ref, 64))


def test_every_bf16_value_against_several_scales(wq):
    """Exhaustive: every finite bf16 w in groups whose absmax is one of several scales
    (normal, subnormal, extreme), including exact midpoints (ties)."""
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    allb = allb[((allb >> 7) & 0xFF) != 0xFF]
    vals = oracle.bf16_to_f64(allb)
    rows = []
    for sb in [0x3F80, 0x3FFF, 0x0080, 0x0001, 0x00FF, 0x7F7F, 0x2F5A, 0x4049]:
        s = oracle.bf16_to_f64(np.array([sb], np.uint16))[0]
        sel = allb[np.abs(vals) <= s]
        per = 63
        sel = np.concatenate([sel, np.zeros((-len(sel)) % per, np.uint16)]).reshape(-1, per)
        rows.append(np.concatenate([np.full((sel.shape[0], 1), sb, np.uint16), sel], 1))
    w_bits = np.concatenate(rows, 0)
    pw, codes, s_ref, c_ref = _quant_both(wq, w_bits, 64)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(bits(pw.aux), s_ref)
    assert np.array_equal(bits(wq.dequant(pw)), oracle.dequant(oracle.DYADIC4, oracle.pack(c_ref), s_ref, 64))


def test_edge_groups(wq):
    w = np.zeros((4, 128), np.uint16)
    w[0, 3] = 0x8000                       # -0.0 in an all-zero group
    w[1, :64] = 0x3F80                     # all equal -> idx 15
    w[1, 64:] = 0xBF80                     # all equal negative -> idx 0
    w[2, 0], w[2, 1] = 0x7F7F, 0xFF7F      # largest finite magnitudes
    w[3, 0], w[3, 1], w[3, 2] = 0x3F80, 0x3D80, 0xBD80   # ties at +-scale/16
    pw, codes, s_ref, c_ref = _quant_both(wq, w, 64)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(bits(pw.aux), s_ref)
    assert np.array_equal(bits(wq.dequant(pw)), oracle.dequant(oracle.DYADIC4, oracle.pack(c_ref), s_ref, 64))


def test_pack_unpack_bit_exact(wq):
    g = np.random.default_rng(7)
    codes = g.integers(0, 16, (77, 160), dtype=np.uint8)
    p = wq.pack(to_dev(codes))
    assert np.array_equal(p.cpu().numpy(), oracle.pack(codes))
    assert np.array_equal(wq.unpack(p).cpu().numpy(), codes)
    hi = to_dev(codes | 0xA0)              # bits above the nibble are dropped
    assert np.array_equal(wq.pack(hi).cpu().numpy(), oracle.pack(codes))


def test_dequant_lloyd_and_lut16_formats_bit_exact(wq):
    g = np.random.default_rng(8)
    n, k = 9, 192
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    packed = oracle.pack(codes)
    levels = np.sort(np.abs(g.standard_normal((n, k // 32, 8))), -1).astype(np.float32) * 0.05
    pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, to_dev(packed), to_dev(levels))
    assert np.array_equal(bits(wq.dequant(pw)), oracle.dequant(oracle.LLOYD8S, packed, levels, 32))
    lut = oracle.f64_to_fp16(g.standard_normal((n, k // 64, 16)) * 0.01)
    pl = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(lut, torch.float16))
    assert np.array_equal(bits(wq.dequant(pl)), oracle.dequant(oracle.LUT16, packed, lut, 64))


def test_injected_launch_failure_and_device_checks(wq):
    w = to_dev_bits(workloads.gaussian_outlier_weight(4, 64, workloads.DYADIC_1, 1))
    wq.debug_fail_next_launches(1)
    with pytest.raises(wq.WqError) as e:
        wq.quantize_dyadic(w, 64)
    assert e.value.status == wq.WQ_ECUDA and "injected" in str(e.value)
    wq.quantize_dyadic(w, 64)              # the next call runs normally
    torch.cuda.synchronize()
    host = torch.zeros(4, 32, dtype=torch.uint8).pin_memory()
    import ctypes
    st = wq._lib.wq_unpack(ctypes.c_void_p(host.data_ptr()), 4, 64, ctypes.c_void_p(host.data_ptr()), None)
    assert st == wq.WQ_EINVAL and "device memory" in wq.last_error()


def test_dequant_every_code_at_every_scale(wq):
    """Dequant over all 16 codes at every finite non-negative bf16 scale (32,640 patterns,
    one per group of 64), bit-exact against the oracle: covers the fast bf16x2 path and the
    fp32 path for scales below 2^-120, subnormal and zero scales included."""
    scales = np.arange(0x7F80, dtype=np.uint16)                # +0 .. max finite
    groups = scales.size
    k = 64 * 64
    n = (groups + 63) // 64
    sc = np.zeros(n * 64, np.uint16)
    sc[:groups] = scales
    sc = sc.reshape(n, 64)
    codes = np.tile(np.arange(16, dtype=np.uint8), (n, k // 16))
    codes = np.roll(codes, 3, axis=1)                         # codes 0..15 in every word position
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, torch.from_numpy(packed).cuda(), to_dev_bits(sc))
    got = bits(wq.dequant(pw))
    torch.cuda.synchronize()
    assert np.array_equal(got, oracle.dequant(oracle.DYADIC4, packed, sc, 64))
