"""Pins of the oracle's STE fake quantisation ("MiniCPM5-1B 验证…" §2.3: hard argmin over the
dyadic codes on the fp32 latent z in the forward pass, identity backward), against
hand-worked values, closed forms, invariants, and the bf16 hard-argmin oracle where both
apply."""
import numpy as np

import oracle
import workloads

ONE = np.uint16(0x3F80)          # bf16 1.0: step 0.125, codes -1.0 .. 0.875


def _one(z, scale_bits=ONE, group=32):
    zz = np.zeros((1, group), np.float32)
    zz[0, 0] = z
    q, c = oracle.fake_quant_ste(zz, np.array([[scale_bits]], np.uint16), group)
    return float(q[0, 0]), int(c[0, 0])


def test_hand_worked_values_scale_one():
    # midpoint between code 8 (0.0) and code 9 (0.125): the lower index wins
    assert _one(0.0625) == (0.0, 8)
    assert _one(np.nextafter(np.float32(0.0625), np.float32(1))) == (0.125, 9)
    # midpoint between code 7 (-0.125) and code 8 (0.0): again the lower index, 7
    assert _one(-0.0625) == (-0.125, 7)
    assert _one(np.nextafter(np.float32(-0.0625), np.float32(1))) == (0.0, 8)
    # beyond the range the end codes: 0.875 (15) and -1.0 (0)
    assert _one(5.0) == (0.875, 15)
    assert _one(0.9375) == (0.875, 15)
    assert _one(-5.0) == (-1.0, 0)
    assert _one(-1.0) == (-1.0, 0)


def test_zero_scale_ties_every_code():
    q, c = _one(0.3, scale_bits=np.uint16(0))
    assert c == 0 and q == 0.0 and np.signbit(np.float32(q))     # (0 - 8) * 0 = -0.0


def test_each_code_value_maps_to_itself():
    g = np.random.default_rng(1)
    scales = workloads.f64_to_bf16_bits(np.abs(g.standard_normal(64)) + 0.01)
    z = np.zeros((64, 16), np.float32)
    step = oracle.bf16_to_f64(scales) / 8
    for j in range(16):
        z[:, j] = (step * (j - 8)).astype(np.float32)
    q, c = oracle.fake_quant_ste(z, scales[:, None], 16)
    assert np.array_equal(c, np.tile(np.arange(16, dtype=np.uint8), (64, 1)))
    assert np.array_equal(q, z)


def test_error_bound_and_monotone_codes():
    g = np.random.default_rng(2)
    z = np.sort(g.standard_normal((8, 256)).astype(np.float32) * 0.03, axis=1)
    scale = workloads.f64_to_bf16_bits(np.full((8, 4), 0.05))
    q, c = oracle.fake_quant_ste(z, scale, 64)
    step = 0.05 / 8
    inside = np.abs(z) <= 0.05 - step / 2
    assert np.all(np.abs(z - q)[inside] <= step / 2 + 1e-12)
    assert np.all(np.diff(c.astype(int), axis=1) >= 0)          # z sorted -> codes sorted


def test_agrees_with_the_bf16_hard_argmin_on_bf16_inputs():
    w_bits = workloads.gaussian_outlier_weight(32, 512, workloads.DYADIC_1, 5)
    scale, codes = oracle.dyadic_quantize(w_bits, 64)
    z = oracle.bf16_to_f64(w_bits).astype(np.float32)
    q, c = oracle.fake_quant_ste(z, scale, 64)
    assert np.array_equal(c, codes)
    # q is the exact code value (fp32 holds it); the bf16 reconstruction is its rounding
    step = oracle.bf16_to_f64(np.repeat(scale, 64, axis=1)) / 8
    assert np.array_equal(q.astype(np.float64), step * (codes.astype(np.float64) - 8))
    assert np.array_equal(oracle.f64_to_bf16(q.astype(np.float64)),
                          oracle.dyadic_dequant(codes, scale, 64))
