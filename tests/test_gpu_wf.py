"""GPU parity of water-filling ("MiniCPM5-1B 验证…" §2.1: 3/4/5-bit dyadic codebooks sharing one
level index space; §6: water-filling) with the oracle, through the C ABI: scales, widths,
the three fp64 distortions, block offsets, packed bit streams and the reconstruction are all
bit-exact, over water levels from zero to infinity, ragged shapes, zero blocks, scales far
outside the fast range, and sampled rows of a full-size launch; a too-small packed buffer is
flagged without any access past it. The format's GEMV is checked against the oracle's
product on the oracle's own encodings."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, f32, matmul_tolerance, to_dev_bits

pytestmark = pytest.mark.gpu


def _check(wq, w_bits, lam):
    n, k = w_bits.shape
    w = to_dev_bits(w_bits)
    scale, width, off, dist = wq.wf_analyze(w, lam, dist=True)
    q = wq.quantize_wf(w, lam)
    rec = wq.dequant_wf(q)
    torch.cuda.synchronize()
    s_ref, wd_ref, d_ref = oracle.wf_analyze(w_bits, lam)
    off_ref = oracle.wf_offsets(wd_ref)
    p_ref = oracle.wf_pack(w_bits, s_ref, wd_ref, off_ref)
    assert np.array_equal(bits(scale), s_ref)
    assert np.array_equal(width.cpu().numpy(), wd_ref)
    assert np.array_equal(dist.cpu().numpy().view(np.uint64), d_ref.view(np.uint64))   # bit-exact fp64
    assert np.array_equal(off.cpu().numpy().view(np.uint32), off_ref)
    assert q.total == int(off_ref[-1])
    assert np.array_equal(q.packed.cpu().numpy()[:q.total], p_ref)
    assert np.array_equal(bits(rec), oracle.wf_dequant(p_ref, s_ref, wd_ref, off_ref, n, k))
    assert wq.device_error() == 0
    return wd_ref


def _weights(seed, n, k, spread=3.0):
    g = np.random.default_rng(seed)
    w = g.standard_normal((n, k)) * 0.02 * g.uniform(1 / spread, spread, (n, 1))
    w[g.random((n, k)) < 0.002] *= 20
    return workloads.f64_to_bf16_bits(w)


@pytest.mark.parametrize("n,k", [(1, 64), (3, 192), (5, 2112), (64, 4096), (33, 1024)])
def test_matches_oracle_across_water_levels(wq, n, k):
    w = _weights(n * 7 + k, n, k)
    _, _, d = oracle.wf_analyze(w, 0.0)
    seen = set()
    for lam in [0.0, float(np.quantile(d[..., 1], 0.3) / 64), float(np.quantile(d[..., 0], 0.7) / 64),
                float("inf")]:
        seen |= set(np.unique(_check(wq, w, lam)).tolist())
    assert seen == {3, 4, 5} or n * k < 256


def test_zero_blocks_subnormals_and_extreme_scales(wq):
    w = _weights(11, 8, 512).astype(np.uint16)
    w[0, :64] = 0                                            # all-zero block: width 3, D = 0
    w[0, 64:128] = 0x8000                                   # negative zeros
    w[1, :] = np.arange(512) % 128                           # bf16 subnormals (scale < 2^-100)
    v = oracle.bf16_to_f64(w[2:4])                           # huge scales (> 2^100)
    w[2:4] = workloads.f64_to_bf16_bits(v * 2.0 ** 110)
    v = oracle.bf16_to_f64(w[4:6])                           # tiny normal scales (< 2^-100)
    w[4:6] = workloads.f64_to_bf16_bits(v * 2.0 ** -110)
    _, _, d = oracle.wf_analyze(w, 0.0)
    for lam in (0.0, float(np.median(d[6:, :, 1]) / 64), float("inf")):
        _check(wq, w, lam)


def test_full_size_launch_sampled_rows(wq):
    # the 8192 x 28672 matrix of the LUT16 workload (N(0, 0.01^2) variant), rows by sample;
    # the offsets are checked in full for consistency with the widths
    n, k = workloads.LUT16_SHAPE
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev).manual_seed(7)
    w = (torch.randn((n, k), device=dev, generator=gen) * 0.01).to(torch.bfloat16)
    lam = 8e-7                                  # about the median 4-bit squared error
    q = wq.quantize_wf(w, lam)
    rec = wq.dequant_wf(q)
    torch.cuda.synchronize()
    sizes = (q.blk_off[1:].to(torch.int64) & 0xFFFFFFFF) - (q.blk_off[:-1].to(torch.int64) & 0xFFFFFFFF)
    assert torch.equal(sizes, 8 * q.width.reshape(-1).to(torch.int64))
    assert int(q.blk_off[0]) == 0 and q.total == int((8 * q.width.to(torch.int64)).sum())
    rows = [0, 1, 4097, n - 1]
    nb = k // 64
    off_all = q.blk_off.cpu().numpy().view(np.uint32)
    packed = q.packed.cpu().numpy()
    for r in rows:
        wr = bits(w[r:r + 1])
        s_ref, wd_ref, _ = oracle.wf_analyze(wr, lam)
        assert np.array_equal(bits(q.scale[r:r + 1]), s_ref)
        assert np.array_equal(q.width[r:r + 1].cpu().numpy(), wd_ref)
        local_off = oracle.wf_offsets(wd_ref)
        p_ref = oracle.wf_pack(wr, s_ref, wd_ref, local_off)
        a, b = int(off_all[r * nb]), int(off_all[(r + 1) * nb])
        assert np.array_equal(packed[a:b], p_ref)
        assert np.array_equal(bits(rec[r:r + 1]), oracle.wf_dequant(p_ref, s_ref, wd_ref, local_off, 1, k))
    assert 3.0 < q.total * 8 / (n * k) < 5.0
    assert wq.device_error() == 0


def test_short_packed_buffer_is_flagged_not_overrun(wq):
    w_bits = _weights(13, 4, 256)
    w = to_dev_bits(w_bits)
    scale, width, off, _ = wq.wf_analyze(w, 0.0)              # every block 5 bits: 40 bytes
    total = int(off[-1].item())
    guard = torch.full((total + 64,), 0xAB, dtype=torch.uint8, device="cuda")
    short = total - 40                                        # the last block does not fit
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = wq._lib.wq_quantize_wf_pack(wq._ptr(w), 4, 256, wq._ptr(scale), wq._ptr(width), wq._ptr(off),
                                     wq._ptr(guard), short, stream)
    assert st == wq.WQ_OK
    torch.cuda.synchronize()
    assert np.all(guard.cpu().numpy()[short:] == 0xAB)       # nothing written past the limit
    code = ctypes.c_int32(0)
    assert wq._lib.wq_device_error(ctypes.byref(code)) == wq.WQ_EDATA and code.value == 2001
    assert wq.device_error() == 0                            # the flag was cleared by the read


def _oracle_encoding(wq, w_bits, lam):
    """The oracle's water-filled encoding of w, and the same bytes on the device."""
    n, k = w_bits.shape
    s, wd, _ = oracle.wf_analyze(w_bits, lam)
    off = oracle.wf_offsets(wd)
    p = oracle.wf_pack(w_bits, s, wd, off)
    dev = torch.device("cuda")
    packed = torch.zeros(max(p.size, 16), dtype=torch.uint8, device=dev)
    packed[:p.size] = torch.from_numpy(p).to(dev)
    q = wq.WfWeight(n, k, to_dev_bits(s), torch.from_numpy(wd).to(dev),
                    torch.from_numpy(off.view(np.int32)).to(dev), packed, int(p.size))
    return q, (p, s, wd, off)


def _gemv_check(wq, q, enc, x_bits, rows=None):
    y = wq.gemv_wf(q, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    y_ref, bound = oracle.wf_matmul_rows(*enc, q.n, q.k, x_bits, rows=rows)
    got = f32(y) if rows is None else f32(y)[:, rows]
    assert np.all(np.abs(got - y_ref) <= matmul_tolerance(y_ref, bound)), \
        f"max err/bound {np.max(np.abs(got - y_ref) / np.maximum(bound, 1e-300)):.3g}"
    assert wq.device_error() == 0


@pytest.mark.parametrize("n,k", [(1, 64), (5, 2112), (33, 1024), (64, 4096), (19, 28672)])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 8, 9, 16])
def test_gemv_matches_oracle(wq, n, k, batch):
    """The format's GEMV ("MiniCPM5-1B 验证…" §2.1, §6 blocks; the dyadic GEMV's contract) on
    mixed 3/4/5-bit rows: ragged row counts, a row tail of fewer than 32 blocks, batches
    that are not a multiple of the kernel's 8 activation rows per launch."""
    w = _weights(n * 3 + k, n, k)
    _, _, d = oracle.wf_analyze(w, 0.0)
    q, enc = _oracle_encoding(wq, w, float(np.median(d[..., 1]) / 64))
    _gemv_check(wq, q, enc, workloads.activations(batch, k, workloads.LUT16, n + batch))


def test_gemv_zero_blocks_subnormals_and_extreme_scales(wq):
    w = _weights(11, 8, 512).astype(np.uint16)
    w[0, :64] = 0
    w[1, :] = np.arange(512) % 128                           # subnormal weights and scales
    w[2:4] = workloads.f64_to_bf16_bits(oracle.bf16_to_f64(w[2:4]) * 2.0 ** 100)
    w[4:6] = workloads.f64_to_bf16_bits(oracle.bf16_to_f64(w[4:6]) * 2.0 ** -110)
    x = workloads.activations(4, 512, workloads.LUT16, 5)
    for lam in (0.0, float("inf")):
        q, enc = _oracle_encoding(wq, w, lam)
        _gemv_check(wq, q, enc, x)


def test_gemv_one_hot_exact(wq):
    """x = e_c gives column c of the reconstruction, bit for bit."""
    n, k = 40, 1024
    w = _weights(17, n, k)
    _, _, d = oracle.wf_analyze(w, 0.0)
    q, enc = _oracle_encoding(wq, w, float(np.median(d[..., 1]) / 64))
    wd = oracle.wf_dequant(*enc, n, k)
    cols = np.array([0, 5, 63, 64, 500, 1023, 777, 128, 129, 300, 640, 1000, 2, 3, 4, 6])
    x = np.zeros((16, k))
    x[np.arange(16), cols] = 1.0
    y = wq.gemv_wf(q, to_dev_bits(workloads.f64_to_bf16_bits(x)))
    assert np.array_equal(bits(y), wd[:, cols].T)


def test_gemv_full_size_sampled_rows(wq):
    """The 8192 x 28672 launch bench.py times (batch 1 and 16), the encoding made by the
    oracle, rows by sample."""
    n, k = workloads.LUT16_SHAPE
    g = np.random.default_rng(7)
    w = workloads.f64_to_bf16_bits(g.standard_normal((n, k)) * 0.01)
    q, enc = _oracle_encoding(wq, w, 8e-7)
    rows = np.array([0, 1, 777, 4097, n - 2, n - 1])
    for batch in (1, 4, 16):
        _gemv_check(wq, q, enc, workloads.activations(batch, k, workloads.LUT16, batch), rows=rows)


def test_gemv_bad_block_is_flagged_not_read(wq):
    """A width outside 3..5 or a block past packed_bytes contributes nothing and is flagged."""
    n, k = 4, 256
    w = _weights(19, n, k)
    q, enc = _oracle_encoding(wq, w, 0.0)                     # every block 5 bits
    x = to_dev_bits(workloads.activations(1, k, workloads.LUT16, 1))
    q.width[1, 2] = 7
    y = wq.gemv_wf(q, x)
    torch.cuda.synchronize()
    code = ctypes.c_int32(0)
    assert wq._lib.wq_device_error(ctypes.byref(code)) == wq.WQ_EDATA and code.value == 2002
    wd = oracle.bf16_to_f64(oracle.wf_dequant(*enc, n, k))
    wd[1, 128:192] = 0.0                                      # the flagged block drops out
    xd = oracle.bf16_to_f64(bits(x))
    y_ref, bound = xd @ wd.T, np.abs(xd) @ np.abs(wd).T
    assert np.all(np.abs(f32(y) - y_ref) <= matmul_tolerance(y_ref, bound))
    assert wq.device_error() == 0


@pytest.mark.parametrize("batch", [1, 2, 4])
def test_gemv_shifted_offset_drops_both_neighbours(wq, batch):
    """Batches 1-4 check each block against the next block's offset: shifting block 5's
    offset by 8 bytes breaks blocks 4 and 5 of that row (both flagged, both left out)."""
    n, k = 4, 1024
    w = _weights(23, n, k)
    q, enc = _oracle_encoding(wq, w, 0.0)                     # every block 5 bits
    x = to_dev_bits(workloads.activations(batch, k, workloads.LUT16, 2))
    kb = k // 64
    q.blk_off[2 * kb + 5] += 8
    y = wq.gemv_wf(q, x)
    torch.cuda.synchronize()
    code = ctypes.c_int32(0)
    assert wq._lib.wq_device_error(ctypes.byref(code)) == wq.WQ_EDATA and code.value == 2002
    wd = oracle.bf16_to_f64(oracle.wf_dequant(*enc, n, k))
    wd[2, 4 * 64:6 * 64] = 0.0
    xd = oracle.bf16_to_f64(bits(x))
    y_ref, bound = xd @ wd.T, np.abs(xd) @ np.abs(wd).T
    assert np.all(np.abs(f32(y) - y_ref) <= matmul_tolerance(y_ref, bound))
    assert wq.device_error() == 0


@pytest.mark.parametrize("batch", [1, 2, 3])
def test_gemv_run_ending_at_the_buffer_end(wq, batch):
    """All blocks at 3 bits (24 bytes): 9 blocks end 8 bytes short of a 16-byte boundary,
    exactly at the end of the buffer, so the last run's tail is read apart from its bulk
    copy; 3 rows leave a row of the warp empty."""
    n, k = 3, 192
    w = _weights(29, n, k)
    q, enc = _oracle_encoding(wq, w, float("inf"))
    assert q.total == 216 and q.packed.numel() == 216
    _gemv_check(wq, q, enc, workloads.activations(batch, k, workloads.LUT16, 4))
