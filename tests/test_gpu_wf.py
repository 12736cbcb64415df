"""GPU parity of water-filling ("MiniCPM5-1B 验证…" §2.1: 3/4/5-bit dyadic codebooks sharing one
level index space; §6: water-filling) with the oracle, through the C ABI: scales, widths,
the three fp64 distortions, block offsets, packed bit streams and the reconstruction are all
bit-exact, over water levels from zero to infinity, ragged shapes, zero blocks, scales far
outside the fast range, and sampled rows of a full-size launch; a too-small packed buffer is
flagged without any access past it."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, to_dev_bits

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
