"""Pins for the oracle's number formats, dyadic code, packing, reconstruction and storage
accounting. Every expected value here comes from the pages' formulas worked by hand
(tests/golden), from a library routine (torch / numpy conversions and products), or
from an independent closed form; none comes from the CUDA path."""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden", "dyadic_worked_example.txt")


def _golden(section):
    rows = []
    for line in open(GOLD):
        line = line.split("#")[0].split()
        if line and line[0] == section:
            rows.append(line[1:])
    return rows


def _all_finite_bf16():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    e = (b >> 7) & 0xFF
    return b[e != 0xFF]


# --- number formats ----------------------------------------------------------------------

def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = oracle.bf16_to_f64(bits)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(ref[fin]))


def test_bf16_rounding_matches_torch_rne():
    # values exactly representable in fp32, so torch's fp32 -> bf16 RNE is an exact reference
    g = np.random.default_rng(0)
    f32 = np.concatenate([
        g.standard_normal(200000).astype(np.float32),
        (g.standard_normal(20000) * 1e-38).astype(np.float32),       # subnormal range
        (g.standard_normal(20000) * 3e38).astype(np.float32),        # overflow range
        # exact ties: bf16 value + half ulp
        (oracle.bf16_to_f64(_all_finite_bf16()[:20000]) * (1 + 2.0 ** -8)).astype(np.float32),
    ])
    f32 = f32[np.isfinite(f32)]
    ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(f32.astype(np.float64))
    assert np.array_equal(got, ref)


def test_fp16_rounding_matches_numpy():
    g = np.random.default_rng(1)
    v = np.concatenate([g.standard_normal(200000), g.standard_normal(20000) * 1e-6,
                        g.standard_normal(20000) * 7e4,
                        np.arange(-2048, 2048) + 0.5])                 # ties at fp16 integers
    ref = v.astype(np.float16).view(np.uint16)
    got = oracle.f64_to_fp16(v)
    assert np.array_equal(got, ref)
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    d = oracle.fp16_to_f64(allbits)
    r = allbits.view(np.float16).astype(np.float64)
    fin = np.isfinite(r)
    assert np.array_equal(d[fin], r[fin])


# --- dyadic code ----------------------------------------------------------------------------

def test_dyadic_worked_example_quantize():
    for scale_h, w_h, idx, wdeq_h in _golden("A"):
        scale = int(scale_h, 16)
        grp = np.zeros((1, 64), np.uint16)
        grp[0, 0] = scale
        grp[0, 1] = int(w_h, 16)
        s, c = oracle.dyadic_quantize(grp, 64, threads=1)
        assert s[0, 0] == scale
        assert c[0, 1] == int(idx), (scale_h, w_h)
        d = oracle.dyadic_dequant(c, s, 64, threads=1)
        assert d[0, 1] == int(wdeq_h, 16), (scale_h, w_h, hex(d[0, 1]))


def test_dyadic_worked_example_reconstruction():
    for scale_h, idx, wdeq_h in _golden("B"):
        c = np.full((1, 64), int(idx), np.uint8)
        s = np.array([[int(scale_h, 16)]], np.uint16)
        d = oracle.dyadic_dequant(c, s, 64, threads=1)
        assert d[0, 0] == int(wdeq_h, 16), (scale_h, idx, hex(d[0, 0]))


def test_pack_worked_example_and_roundtrip():
    for lo, hi, byte in _golden("C"):
        c = np.array([[int(lo), int(hi)]], np.uint8)
        assert oracle.pack(c, threads=1)[0, 0] == int(byte, 16)
    g = np.random.default_rng(2)
    codes = g.integers(0, 16, size=(37, 130), dtype=np.uint8)
    p = oracle.pack(codes)
    assert np.array_equal(p, (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8))
    assert np.array_equal(oracle.unpack(p), codes)


SCALES = [0x3F80, 0x3FFF, 0x0080, 0x3E4D, 0x4049, 0x7EFF, 0x3C00, 0x00FF, 0x2F5A]


@pytest.mark.parametrize("scale_bits", SCALES)
def test_dyadic_argmin_exhaustive_vs_midpoint_closed_form(scale_bits):
    """Every finite bf16 w with |w| <= scale: the oracle's brute-force argmin equals the
    closed form idx = #{j in 1..15 : w > (2j-17) * scale / 16} (round half down), whose
    midpoints are exact in double."""
    scale = oracle.bf16_to_f64(np.array([scale_bits], np.uint16))[0]
    allw = _all_finite_bf16()
    wv = oracle.bf16_to_f64(allw)
    wsel = allw[np.abs(wv) <= scale]
    group = 64
    per = group - 1
    npad = (-len(wsel)) % per
    wsel = np.concatenate([wsel, np.zeros(npad, np.uint16)])
    body = wsel.reshape(-1, per)
    grp = np.concatenate([np.full((body.shape[0], 1), scale_bits, np.uint16), body], axis=1)
    s, c = oracle.dyadic_quantize(grp, group)
    assert np.all(s == scale_bits)
    w = oracle.bf16_to_f64(grp)
    mids = (2.0 * np.arange(1, 16) - 17.0) * scale / 16.0
    closed = (w[..., None] > mids).sum(-1)
    assert np.array_equal(c, closed.astype(np.uint8))


def test_dyadic_edge_groups():
    g = np.zeros((1, 64), np.uint16)                  # all-zero group: scale 0, idx 0
    g[0, 5] = 0x8000                                  # a -0.0 too
    s, c = oracle.dyadic_quantize(g, 64, threads=1)
    assert s[0, 0] == 0 and np.all(c == 0)
    d = oracle.dyadic_dequant(c, s, 64, threads=1)
    assert np.all(d == 0x8000)                        # bf16(0 * (0 - 8)) = -0.0 (reading)
    g = np.full((1, 64), 0x0080, np.uint16)           # smallest normal everywhere
    s, c = oracle.dyadic_quantize(g, 64, threads=1)
    assert s[0, 0] == 0x0080 and np.all(c == 15)
    # +scale -> 15, -scale -> 0
    g = np.zeros((1, 32), np.uint16)
    g[0, 0], g[0, 1] = 0x4049, 0xC049
    s, c = oracle.dyadic_quantize(g, 32, threads=1)
    assert c[0, 0] == 15 and c[0, 1] == 0
    with pytest.raises(ValueError):                   # non-finite input is rejected
        bad = np.zeros((1, 64), np.uint16)
        bad[0, 3] = 0x7F80
        oracle.dyadic_quantize(bad, 64, threads=1)


def test_dyadic_dequant_all_codes_all_scales_vs_torch():
    """bf16(step * (idx - 8)) for 16 codes x every finite non-negative bf16 scale, against
    torch: the product is exact in fp32 (8-bit significand x integer <= 8), then torch's
    fp32 -> bf16 conversion rounds it once."""
    scales = _all_finite_bf16()
    scales = scales[scales < 0x8000]
    n = scales.size
    codes = np.tile(np.arange(16, dtype=np.uint8), (n, 4))               # [n, 64]
    d = oracle.dyadic_dequant(codes, scales.reshape(n, 1), 64)
    sf = torch.from_numpy(scales.view(np.int16)).view(torch.bfloat16).float() / 8.0
    ref = (sf[:, None] * (torch.from_numpy(codes.astype(np.float32)) - 8.0)).to(torch.bfloat16)
    assert np.array_equal(d, ref.view(torch.int16).numpy().view(np.uint16))


def test_dyadic_quantize_then_dequant_error_bound_on_workload():
    """Reconstruction error <= step/2 for every weight of a DYADIC_1-style matrix, except
    above the top code 7*step, where the error is w - 7*step (at most one step)."""
    w = workloads.gaussian_outlier_weight(64, 2048, workloads.DYADIC_1, 0)
    s, c = oracle.dyadic_quantize(w, 64)
    wd = oracle.bf16_to_f64(oracle.dyadic_dequant(c, s, 64))
    wv = oracle.bf16_to_f64(w)
    step = np.repeat(oracle.bf16_to_f64(s) / 8.0, 64, axis=1)
    exact = step * (c.astype(np.float64) - 8.0)
    bound = np.maximum(step / 2, wv - 7 * step)
    assert np.all(np.abs(wv - exact) <= bound)
    assert np.all(bound <= step)
    assert np.all(np.abs(wd - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-300)


# --- storage accounting -----------------------------------------------------------------------

def test_storage_accounting_dyadic_679M():
    """[DG] §2.5: 679M x 4 bit / 8 = 340 MB packed + 21 MB scale = 361 MB (g64, bf16)."""
    n = 679e6
    total = oracle.storage_bytes(oracle.DYADIC4, n, 64)
    packed = n * 4 / 8
    assert round(packed / 1e6) == 340 or round(packed / 1e6) == 339      # 339.5 MB
    assert round((total - packed) / 1e6) == 21
    assert round(total / 1e6) == 361


def test_storage_accounting_g32_lloyd():
    """[G32] §2: 4 bit per weight + 8 bit per group of 32 = 4.25 bit; 16 / 4.25 = 3.76x."""
    n = 2048 * 2048
    bits = oracle.storage_bytes(oracle.LLOYD8S, n, 32) * 8 / n
    assert bits == pytest.approx(4.25)
    assert round(16 / bits, 2) == 3.76
    # the codebook actually kept for decoding is counted apart: 8 fp32 per group
    assert oracle.storage_lloyd_codebook_bytes(n, 32) * 8 / n == pytest.approx(8.0)
