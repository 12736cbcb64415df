"""The LUT16 consumers over the whole range of bf16 activations ("K-Means量化技术…" §2.2: the
fp16 centroids are multiplied by the activations; the fp16 MMA needs fp16 activations).

Each activation row (GEMM) or each row's chunk of K staged by a CTA (GEMV) is converted to
fp16 times a power of two that puts its largest magnitude in [2^15, 2^16), and the fp32 sums
are multiplied back. Checked here against the oracle's fp64 product at the usual tolerance
(2e-3 * sum |W||x| plus half a bf16 ulp):
  * activations around 1e-8 (below fp16's normal range), around 1e30 (above its maximum),
    and rows mixing 1e-8 with 1e2;
  * batch rows of very different magnitudes in one call;
  * a "compensated" row whose magnitude steps by 2^5 every 512 columns while the centroids
    of those columns step the other way, so that every chunk of K contributes alike to
    each output and a wrong scale on any one chunk would show;
for the GEMV (batch 1 to 16, single and multi-chunk K, the cluster split of a large
matrix) and the tcgen05 GEMM (plain, split-K, last-wave split)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import f32, matmul_tolerance, to_dev, to_dev_bits

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _weight(wq, n, k, seed, compensated=False):
    g = np.random.default_rng(seed)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    lut = np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01
    if compensated:
        lut = lut * np.exp2(-_block_exponent(np.arange(k // 64) * 64))[None, :, None]
    lut = oracle.f64_to_fp16(lut)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(lut, torch.float16))
    return pw, packed, lut


def _block_exponent(cols):
    # -10, -5, 0, 5, 10, -10, ... per 512 columns
    return 5.0 * ((cols // 512) % 5) - 10.0


def _acts(kind, b, k, seed):
    g = np.random.default_rng(seed)
    z = g.standard_normal((b, k))
    if kind == "tiny":
        v = z * 1e-8
    elif kind == "huge":
        v = z * 1e30
    elif kind == "mixed":
        v = z * np.where(g.random((b, k)) < 0.5, 1e-8, 1e2)
    elif kind == "rows":                         # each batch row its own magnitude
        mags = np.array([1e-8, 1e2, 1e30, 1e-30, 1.0, 3e-5, 7e4, 1e-20])
        v = z * mags[np.arange(b) % len(mags)][:, None]
    elif kind == "compensated":
        v = z * np.exp2(_block_exponent(np.arange(k)))[None, :]
    else:
        raise ValueError(kind)
    return workloads.f64_to_bf16_bits(v)


def _check(y, x_bits, packed, lut, rows=None, ms=None):
    xs = x_bits if ms is None else x_bits[ms]
    y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, xs, rows=rows)
    got = f32(y)
    if ms is not None:
        got = got[ms]
    if rows is not None:
        got = got[:, rows]
    err = np.abs(got - y_ref)
    tol = matmul_tolerance(y_ref, bound, TOL)
    assert np.all(err <= tol), f"max err/bound {np.max(err / np.maximum(bound, 1e-300)):.3g}"
    assert np.any(y_ref != 0)


KINDS = ["tiny", "huge", "mixed", "rows"]


@pytest.mark.parametrize("kind", KINDS)
@pytest.mark.parametrize("batch", [1, 5, 16])
def test_lut16_gemv_activation_range(wq, kind, batch):
    n, k = 96, 2048
    pw, packed, lut = _weight(wq, n, k, 3 + batch)
    x_bits = _acts(kind, batch, k, 10 * batch + KINDS.index(kind))
    y = wq.gemv(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    _check(y, x_bits, packed, lut)


@pytest.mark.parametrize("batch,k", [(16, 4096), (1, 28672), (3, 16384)])
def test_lut16_gemv_compensated_chunks(wq, batch, k):
    """K walked in several staged chunks per CTA, each with its own scale."""
    n = 64
    pw, packed, lut = _weight(wq, n, k, batch + k, compensated=True)
    x_bits = _acts("compensated", batch, k, batch)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    _check(y, x_bits, packed, lut)


@pytest.mark.parametrize("batch", [1, 16])
def test_lut16_gemv_cluster_split_compensated(wq, batch):
    """A matrix large enough for the cluster split of K (each CTA of a cluster stages its own
    slice with its own scale; the partial sums meet unscaled); sampled rows."""
    n, k = 4096, 8192
    pw, packed, lut = _weight(wq, n, k, 77 + batch, compensated=True)
    x_bits = _acts("compensated", batch, k, 5 + batch)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, n, 61), [n - 1]])
    _check(y, x_bits, packed, lut, rows=rows)


@pytest.mark.parametrize("kind", KINDS + ["compensated"])
@pytest.mark.parametrize("m", [13, 48, 128, 300])
def test_lut16_gemm_activation_range(wq, kind, m):
    """m = 48 splits K across CTAs (partial sums in the workspace); the others run whole."""
    n, k = 256, 4096
    pw, packed, lut = _weight(wq, n, k, m, compensated=(kind == "compensated"))
    x_bits = _acts(kind, m, k, m + 1)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    _check(y, x_bits, packed, lut, ms=np.arange(0, m, 3))


def test_lut16_gemm_last_wave_split_mixed(wq):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n, k, m = 128 * (sms + 10), 4096, 256
    pw, packed, lut = _weight(wq, n, k, 8)
    assert wq.gemm_workspace_bytes(pw, m) > 2 * m * k      # the tail split is planned
    x_bits = _acts("rows", m, k, 9)
    y = wq.gemm(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rows = np.concatenate([np.arange(0, 128 * sms, 397), np.arange(128 * sms, n, 7), [n - 1]])
    _check(y, x_bits, packed, lut, rows=rows, ms=np.arange(0, m, 5))
