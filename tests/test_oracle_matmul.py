"""Pins for the oracle's W4A16 product reference y = Wdeq x (fp64) and its error scale."""
import numpy as np

import oracle
import workloads


def _dyadic(n, k, seed, group=64):
    w = workloads.gaussian_outlier_weight(n, k, workloads.DYADIC_1, seed)
    s, c = oracle.dyadic_quantize(w, group)
    return oracle.pack(c), s, c


def test_one_hot_activation_returns_the_dequantised_column():
    packed, s, c = _dyadic(40, 256, 11)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.DYADIC4, packed, s, 64))
    for col in (0, 1, 63, 64, 255):
        x = np.zeros((1, 256))
        x[0, col] = 1.0
        y, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, workloads.f64_to_bf16_bits(x))
        assert np.array_equal(y[0], wd[:, col])
        assert np.array_equal(bound[0], np.abs(wd[:, col]))


def test_all_codes_eight_give_exact_zero():
    n, k = 8, 128
    packed = np.full((n, k // 2), 0x88, np.uint8)
    s = workloads.f64_to_bf16_bits(np.random.default_rng(3).uniform(0.1, 2.0, (n, k // 64)))
    x = workloads.activations(3, k, workloads.DYADIC_1)
    y, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x)
    assert np.all(y == 0.0) and np.all(bound == 0.0)


def test_unit_activation_over_one_group_gives_integer_sum_times_step():
    """x = 1 on group g, 0 elsewhere: y = step * sum(idx - 8), exact (small integers)."""
    n, k = 16, 192
    g = np.random.default_rng(4)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    scale = np.full((n, k // 64), 0x3E00, np.uint16)          # 0.125 -> step 1/64
    packed = oracle.pack(codes)
    for grp in range(3):
        x = np.zeros((1, k))
        x[0, grp * 64:(grp + 1) * 64] = 1.0
        y, _ = oracle.matmul_rows(oracle.DYADIC4, packed, scale, 64, workloads.f64_to_bf16_bits(x))
        expect = (codes[:, grp * 64:(grp + 1) * 64].astype(np.int64) - 8).sum(1) / 64.0
        assert np.array_equal(y[0], expect)


def test_matches_numpy_matmul_on_dequantised_weights():
    packed, s, c = _dyadic(96, 320, 12)
    x = workloads.activations(5, 320, workloads.DYADIC_1, 1)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.DYADIC4, packed, s, 64))
    xd = oracle.bf16_to_f64(x)
    y, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x)
    ref = xd @ wd.T
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.abs(xd).sum() * np.abs(wd).max())
    assert np.allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-13)
    assert np.all(np.abs(y) <= bound * (1 + 1e-12))
    rows = np.array([95, 0, 17, 17], np.int64)                  # sampled rows, any order
    ys, _ = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x, rows=rows)
    assert np.array_equal(ys, y[:, rows])


def test_lut16_rows_use_the_fp16_centroid_exactly():
    n, k = 4, 128
    g = np.random.default_rng(5)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    lut = oracle.f64_to_fp16(g.standard_normal((n, k // 64, 16)) * 0.01)
    packed = oracle.pack(codes)
    wd = oracle.fp16_to_f64(oracle.dequant(oracle.LUT16, packed, lut, 64))
    expect = np.take_along_axis(lut.astype(np.float64) * 0 + oracle.fp16_to_f64(lut),
                                codes.reshape(n, 2, 64).astype(np.int64), axis=2).reshape(n, k)
    assert np.array_equal(wd, expect)


def test_lloyd_rows_apply_the_sign_bit():
    n, k = 2, 64
    levels = np.tile(np.array([0, 0.1, 0.2, 0.3, 0.4, 0.5, 0.6, 0.7], np.float32), (n, 2, 1))
    codes = np.tile(np.arange(16, dtype=np.uint8), (n, 4))
    packed = oracle.pack(codes)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.LLOYD8S, packed, levels, 32))
    lv = levels[0, 0].astype(np.float64)
    expect = np.concatenate([lv, -lv])
    expect = oracle.bf16_to_f64(workloads.f64_to_bf16_bits(expect))   # fp32 -> bf16 RNE
    assert np.array_equal(wd[0, :16], expect)
    assert np.signbit(wd[0, 8])                                       # -0.0 for level 0, sign 1


def test_codebook_formats_match_numpy_matmul_on_their_dequant():
    # LUT16 (fp16 centroids, blocks of 64) and LLOYD8S (signed fp32 levels, groups of 32):
    # the product equals x Wdeq^T with Wdeq from the separately pinned dequant
    g = np.random.default_rng(21)
    n, k = 40, 256
    x = workloads.activations(3, k, workloads.LUT16, 2)
    xd = oracle.bf16_to_f64(x)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    packed = oracle.pack(codes)
    lut = oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    levels = np.sort(np.abs(g.standard_normal((n, k // 32, 8))) * 0.02, -1).astype(np.float32)
    for fmt, aux, grp, decode in [(oracle.LUT16, lut, 64, oracle.fp16_to_f64),
                                  (oracle.LLOYD8S, levels, 32, oracle.bf16_to_f64)]:
        wd = decode(oracle.dequant(fmt, packed, aux, grp))
        y, bound = oracle.matmul_rows(fmt, packed, aux, grp, x)
        assert np.allclose(y, xd @ wd.T, rtol=0, atol=1e-13 * np.abs(xd).sum() * np.abs(wd).max())
        assert np.allclose(bound, np.abs(xd) @ np.abs(wd).T, rtol=1e-13)
        rows = np.array([n - 1, 3, 3], np.int64)
        ys, _ = oracle.matmul_rows(fmt, packed, aux, grp, x, rows=rows)
        assert np.array_equal(ys, y[:, rows])
