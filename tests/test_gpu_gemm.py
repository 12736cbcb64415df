"""GPU parity of the tcgen05 W4A16 GEMM against the oracle's fp64 product of its own
reconstruction: |y - y_ref| <= 2e-3 * sum_k |Wdeq[n, k]| |x[m, k]| per element, plus exact
special cases (one-hot activations reproduce a dequantised column; all-eight codes give
zero) and the split-K workspace path used for small m."""
import functools

import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import f32, matmul_tolerance, to_dev, to_dev_bits

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _weight(wq, n, k, group, seed, workload=workloads.PREFILL):
    w_bits = workloads.gaussian_outlier_weight(n, k, workload, seed)
    s, c = oracle.dyadic_quantize(w_bits, group)
    packed = oracle.pack(c)
    return wq.PackedWeight(wq.FMT_DYADIC4, group, n, k, to_dev(packed), to_dev_bits(s)), packed, s


def _check(y, y_ref, bound):
    err = np.abs(f32(y) - y_ref)
    ratio = err / np.maximum(bound, 1e-300)
    assert np.all(err <= matmul_tolerance(y_ref, bound, TOL)), f"max err/bound {ratio.max():.3g}"


@pytest.mark.parametrize("m", [1, 8, 9, 12, 13, 16, 17, 33, 64, 100, 128, 129, 256, 300])
@pytest.mark.parametrize("n,k,group", [(128, 256, 64), (200, 320, 64), (13, 64, 64), (256, 1024, 32)])
def test_gemm_matches_oracle(wq, m, n, k, group):
    pw, packed, s = _weight(wq, n, k, group, m * 7 + n + k)
    x_bits = workloads.activations(m, k, workloads.PREFILL, n + m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, group, x_bits)
    _check(y, y_ref, bound)
    assert wq.device_error() == 0


def test_gemm_one_hot_and_zero_codes_exact(wq):
    n, k = 256, 512
    pw, packed, s = _weight(wq, n, k, 64, 3)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.DYADIC4, packed, s, 64))
    cols = np.arange(0, 512, 3)
    x = np.zeros((len(cols), k))
    x[np.arange(len(cols)), cols] = 1.0
    y = f32(wq.gemm(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
    assert np.array_equal(y, wd[:, cols].T)
    zero = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(np.full((n, k // 2), 0x88, np.uint8)), pw.aux)
    xr = to_dev_bits(workloads.activations(64, k, workloads.PREFILL, 9))
    assert torch.count_nonzero(wq.gemm(zero, xr).float()).item() == 0


def test_gemm_split_k_uses_workspace(wq):
    pw, packed, s = _weight(wq, 1024, 8192, 64, 5)
    assert wq.gemm_workspace_bytes(pw, 16) == 0           # m <= 16 runs on the GEMV kernel
    assert wq.gemm_workspace_bytes(pw, 48) > 0            # small m splits K
    x_bits = workloads.activations(48, 8192, workloads.PREFILL, 5)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    rows = np.arange(0, 1024, 7)
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x_bits, rows=rows)
    err = np.abs(f32(y)[:, rows] - y_ref)
    assert np.all(err <= matmul_tolerance(y_ref, bound, TOL))


@functools.lru_cache(maxsize=2)
def _prefill_quantised(n, k):
    """A prefill weight quantised by the oracle on the host (packed codes, bf16 scales)."""
    w_bits = workloads.gaussian_outlier_weight(n, k, workloads.PREFILL, 0 if n == 4096 else 1)
    s, c = oracle.dyadic_quantize(w_bits, 64)
    return oracle.pack(c), s


@pytest.mark.parametrize("shape", workloads.PREFILL_SHAPES)
@pytest.mark.parametrize("m", workloads.PREFILL_M)
def test_gemm_full_size_sampled(wq, shape, m):
    """The prefill workload at full size: (n, k) = (4096, 11008) / (11008, 4096), every m;
    96 sampled weight rows x up to 128 sampled activation rows against the oracle."""
    n, k = shape
    packed, s = _prefill_quantised(n, k)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(s))
    x_bits = workloads.activations(m, k, workloads.PREFILL, m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rng = np.random.default_rng(m + n)
    rows = np.sort(rng.choice(n, 96, replace=False))
    ms = np.sort(rng.choice(m, min(m, 128), replace=False))
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x_bits[ms], rows=rows)
    got = f32(y)[np.ix_(ms, rows)]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound, TOL))


def test_gemm_one_hot_every_scale_regime(wq):
    """The GEMM's in-smem reconstruction across every scale regime (see the GEMV test of the
    same name): one-hot activations reproduce the dequantised column exactly."""
    regimes = [0x0001, 0x0031, 0x007F, 0x0080, 0x00FF, 0x3D4C, 0x3F80, 0x3FFF, 0x7C00, 0x7D80,
               0x7E55, 0x7F7F, 0x0000]
    n, k = 16 * len(regimes), 256
    g = np.random.default_rng(14)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    scale = np.repeat(np.array(regimes, np.uint16), 16)[:, None].repeat(k // 64, 1)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(scale))
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.DYADIC4, packed, scale, 64))
    x = np.zeros((k, k))
    x[np.arange(k), np.arange(k)] = 1.0
    y = f32(wq.gemm(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
    assert np.array_equal(y, wd.T)


def _lloyd(wq, n, k, seed, signed_levels=False):
    g = np.random.default_rng(seed)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    levels = np.sort(np.abs(g.standard_normal((n, k // 32, 8))) * 0.02, -1).astype(np.float32)
    if signed_levels:
        levels *= np.where(g.random(levels.shape) < 0.5, -1.0, 1.0).astype(np.float32)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, to_dev(packed), torch.from_numpy(levels).cuda())
    return pw, packed, levels


@pytest.mark.parametrize("m", [1, 8, 12, 13, 48, 128, 200, 256, 300])
@pytest.mark.parametrize("n,k", [(128, 256), (200, 320), (256, 1024)])
def test_gemm_lloyd8s_matches_oracle(wq, m, n, k):
    """The fused LLOYD8S consumer on the tensor-memory GEMM ("int4-g32+warm" §5.2): the
    group's 8 levels arrive by TMA with each stage and are rebuilt into a bf16 codebook."""
    if k % 64:
        pytest.skip("the GEMM needs k % 64 == 0")
    pw, packed, levels = _lloyd(wq, n, k, m * 3 + n + k)
    x_bits = workloads.activations(m, k, workloads.PREFILL, n + m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_rows(oracle.LLOYD8S, packed, levels, 32, x_bits)
    _check(y, y_ref, bound)
    assert wq.device_error() == 0


def test_gemm_lloyd8s_one_hot_exact(wq):
    n, k = 256, 512
    pw, packed, levels = _lloyd(wq, n, k, 17, signed_levels=True)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.LLOYD8S, packed, levels, 32))
    cols = np.arange(0, k, 3)
    x = np.zeros((len(cols), k))
    x[np.arange(len(cols)), cols] = 1.0
    y = f32(wq.gemm(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
    assert np.array_equal(y, wd[:, cols].T)


def test_gemm_last_wave_split(wq):
    """Wide tiles in whole waves plus a short tail: the tail tiles run as a second launch with
    K split across CTAs (partial sums in the workspace). 158 weight-row tiles of 128 on a
    148-SM B200 leave a tail of 10; rows of the tail tiles and of the first wave are
    sampled."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles = sms + 10
    n, k, m = 128 * tiles, 4096, 256
    pw, packed, s = _weight(wq, n, k, 64, 31)
    assert wq.gemm_workspace_bytes(pw, m) > 0               # the tail split is planned
    x_bits = workloads.activations(m, k, workloads.PREFILL, 31)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rows = np.concatenate([np.arange(0, 128 * sms, 397), np.arange(128 * sms, n, 5), [n - 1]])
    ms = np.arange(0, m, 3)
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x_bits[ms], rows=rows)
    got = f32(y)[np.ix_(ms, rows)]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound, TOL))
    # the same through the static-scratch entry point (the tail's scratch stays within it)
    assert wq.gemm_workspace_bytes(pw, m) <= (16 << 20)
    ys = wq.gemm_static(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    got = f32(ys)[np.ix_(ms, rows)]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound, TOL))


@pytest.mark.parametrize("fmt", ["dyadic", "lloyd8s", "lut16"])
@pytest.mark.parametrize("m", [48, 128, 300])
def test_gemm_split_k_across_many_ctas(wq, fmt, m):
    """8 weight-row tiles and K = 8192: the plans split K across many CTAs (narrow 128 x 64
    tiles at m = 48, 128 x 128 tiles with 128-column stages at m = 128, 128 x 256 at
    m = 300), so each tile's sum is assembled from many fp32 partials in the workspace.
    Every weight row of sampled activation rows against the oracle, for each weight format,
    and the static-scratch entry point the same where its scratch holds the partials."""
    n, k = 1024, 8192
    if fmt == "dyadic":
        pw, packed, aux = _weight(wq, n, k, 64, 50 + m)
        code, group = oracle.DYADIC4, 64
    elif fmt == "lloyd8s":
        g = np.random.default_rng(m)
        codes = g.integers(0, 16, (n, k), dtype=np.uint8)
        aux = np.sort(np.abs(g.standard_normal((n, k // 32, 8))) * 0.02, -1).astype(np.float32)
        packed = oracle.pack(codes)
        pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, to_dev(packed), torch.from_numpy(aux).cuda())
        code, group = oracle.LLOYD8S, 32
    else:
        pw, packed, aux = _lut16(wq, n, k, m)
        code, group = oracle.LUT16, 64
    assert wq.gemm_workspace_bytes(pw, m) > 0
    x_bits = workloads.activations(m, k, workloads.PREFILL, 70 + m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    try:
        ys = wq.gemm_static(pw, to_dev_bits(x_bits))
    except wq.WqError as e:          # LUT16 at m = 300: activations + partials pass 16 MiB
        assert e.status == wq.WQ_EINVAL and "static scratch" in str(e)
        ys = None
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    ms = np.arange(0, m, 7)
    y_ref, bound = oracle.matmul_rows(code, packed, aux, group, x_bits[ms])
    tol = matmul_tolerance(y_ref, bound, TOL)
    assert np.all(np.abs(f32(y)[ms] - y_ref) <= tol)
    if ys is not None:
        assert np.all(np.abs(f32(ys)[ms] - y_ref) <= tol)


@pytest.mark.parametrize("fmt", ["dyadic", "lloyd8s", "lut16"])
@pytest.mark.parametrize("m", [768, 700])
def test_gemm_384_row_activation_tiles(wq, fmt, m):
    """74 weight-row tiles: 384-row activation tiles need one wave where 256-row ones need
    two (at most 0.7 times the waves), so the plan takes them (two N = 192 MMAs per reconstructed weight slot, the
    activation tile loaded as two 192-row boxes; at m = 700 the second box of the last tile
    runs past the last row). Sampled activation rows, every weight row, against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n, k = 128 * (sms // 2), 1024
    if fmt == "dyadic":
        pw, packed, aux = _weight(wq, n, k, 64, 90 + m)
        code, group = oracle.DYADIC4, 64
    elif fmt == "lloyd8s":
        g = np.random.default_rng(m + 1)
        codes = g.integers(0, 16, (n, k), dtype=np.uint8)
        aux = np.sort(np.abs(g.standard_normal((n, k // 32, 8))) * 0.02, -1).astype(np.float32)
        packed = oracle.pack(codes)
        pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, to_dev(packed), torch.from_numpy(aux).cuda())
        code, group = oracle.LLOYD8S, 32
    else:
        pw, packed, aux = _lut16(wq, n, k, m + 2)
        code, group = oracle.LUT16, 64
    x_bits = workloads.activations(m, k, workloads.PREFILL, 95 + m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    ms = np.concatenate([np.arange(0, m, 37), [191, 192, 383, 384, 575, 576, m - 1]])
    y_ref, bound = oracle.matmul_rows(code, packed, aux, group, x_bits[ms])
    assert np.all(np.abs(f32(y)[ms] - y_ref) <= matmul_tolerance(y_ref, bound, TOL))


def _lut16(wq, n, k, seed):
    g = np.random.default_rng(seed)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    lut = oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(lut, torch.float16))
    return pw, packed, lut


@pytest.mark.parametrize("m", [1, 12, 13, 16, 48, 128, 200, 256, 300])
@pytest.mark.parametrize("n,k", [(128, 256), (200, 320), (256, 1024)])
def test_gemm_lut16_matches_oracle(wq, m, n, k):
    """The LUT16 consumer on the tensor-memory GEMM ("K-Means量化技术…" §2.2, the large-batch
    branch of §4.1): each stage's 16-entry fp16 tables arrive by TMA and the codes are looked
    up in them; the MMA runs in fp16 on activations converted from bf16."""
    pw, packed, lut = _lut16(wq, n, k, m * 5 + n + k)
    x_bits = workloads.activations(m, k, workloads.PREFILL, n + 2 * m)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, x_bits)
    _check(y, y_ref, bound)
    assert wq.device_error() == 0


def test_gemm_lut16_one_hot_exact(wq):
    """x = e_c gives bf16 of the fp16 centroid each row's code at column c selects."""
    n, k = 256, 512
    pw, packed, lut = _lut16(wq, n, k, 23)
    wd = oracle.fp16_to_f64(oracle.dequant(oracle.LUT16, packed, lut, 64))
    cols = np.arange(1, k, 3)
    x = np.zeros((len(cols), k))
    x[np.arange(len(cols)), cols] = 1.0
    y = wq.gemm(pw, to_dev_bits(workloads.f64_to_bf16_bits(x)))
    want = workloads.f64_to_bf16_bits(wd[:, cols].T)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("m,n,k", [(48, 1024, 8192), (256, None, 4096)])
def test_gemm_lut16_workspace_paths(wq, m, n, k):
    """Split-K (small m) and the last-wave split (whole waves plus a short tail): the fp32
    partial sums sit in the workspace after the fp16 activations; sampled rows against the
    oracle."""
    if n is None:
        n = 128 * (torch.cuda.get_device_properties(0).multi_processor_count + 10)
    pw, packed, lut = _lut16(wq, n, k, m + 41)
    need = wq.gemm_workspace_bytes(pw, m)
    assert need > 2 * m * k                                 # activations + partial sums
    x_bits = workloads.activations(m, k, workloads.PREFILL, m + 41)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rows = np.concatenate([np.arange(0, n, 97), [n - 1]])
    ms = np.arange(0, m, 5)
    y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, x_bits[ms], rows=rows)
    got = f32(y)[np.ix_(ms, rows)]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound, TOL))


@pytest.mark.parametrize("m", [512, 4096])
def test_gemm_lut16_bench_launch_sampled(wq, m):
    """The LUT16 GEMM in the launches bench.py times (4096 x 11008; m = 512 splits K in two,
    m = 4096 runs whole waves of 256-row activation tiles), random codes and sorted fp16
    centroids; 64 sampled weight rows x 64 sampled activation rows against the oracle."""
    n, k = workloads.PREFILL_SHAPES[0]
    pw, packed, lut = _lut16(wq, n, k, 6)
    x_bits = workloads.activations(m, k, workloads.PREFILL, m + 7)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rng = np.random.default_rng(m)
    rows = np.sort(rng.choice(n, 64, replace=False))
    ms = np.sort(rng.choice(m, 64, replace=False))
    y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, x_bits[ms], rows=rows)
    got = f32(y)[np.ix_(ms, rows)]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound, TOL))
