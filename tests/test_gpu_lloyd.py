"""GPU parity of the codebook producers against the oracle.

Lloyd g32 ([G32] "int4-g32+warm 裸量化：原理与实验报告" §1.3): the GPU screens the 112
candidates in fp32 with bounds on each candidate's exact MSE and re-evaluates in fp64 every
candidate those bounds cannot rule out, so its choice is the oracle's argmin. A different
candidate is accepted only where the two MSEs are within 1e-6 relative (the near-tie the
comparison treats as ambiguous; such a group is re-run in the oracle from the GPU's
candidate and everything downstream is compared). Then: codes exactly wherever the
nearest-level margin exceeds 1e-6 * gmax, levels within 1e-5 * gmax, the parameter byte
exactly, the MSE trace within 1e-5 relative.

k-means LUT16 ([KM] "K-Means量化技术：突破LLM低比特部署瓶颈" §1.2): both sides decide in
fp64 and sum each centroid's members in index order, so codes and fp16 centroids must match
bit for bit, and repeated runs are identical.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, to_dev_bits

pytestmark = pytest.mark.gpu


def _cand_from_params(p):
    p = p.astype(np.int64)
    fam = p >> 7
    return np.where(fam == 0, 7 * ((p >> 3) & 15) + (p & 7), 105 + ((p >> 3) & 15))


NEAR_TIE = 1e-6          # relative MSE gap below which two candidates are a near-tie


def _near_tie_ok(gpu_c_mse, best, gmax):
    # fp64 levels carry ~1e-15 * gmax, so an MSE of zero is only known to ~1e-30 * gmax^2:
    # the floor keeps zero-MSE groups (built from a candidate's own levels) comparable
    return gpu_c_mse <= best * (1 + NEAR_TIE) + 1e-24 * gmax ** 2


def _check_lloyd(wq, w_bits, rounds=25):
    n, k = w_bits.shape
    pw, ex = wq.quantize_lloyd(to_dev_bits(w_bits), wq.LLOYD_G32_WARM, rounds, codes=True, trace=True)
    torch.cuda.synchronize()
    g_codes = ex["codes"].cpu().numpy()
    g_lv = pw.aux.cpu().numpy().astype(np.float64)
    g_par = ex["params"].cpu().numpy()
    g_tr = ex["trace"].cpu().numpy().astype(np.float64)
    ref = oracle.lloyd(w_bits, 32, rounds)
    gmax = np.abs(oracle.bf16_to_f64(w_bits)).reshape(n, k // 32, 32).max(-1)
    g_cand = _cand_from_params(g_par)
    mism = g_cand != ref["cand"]
    print(f"candidate mismatches: {mism.sum()} of {mism.size} groups")
    if mism.any():
        forced = oracle.lloyd(w_bits, 32, rounds, force_cand=np.where(mism, g_cand, -1).astype(np.int32))
        # the GPU's candidate is a near-tie of the oracle's best
        best = ref["trace"][..., 0]
        gpu_c_mse = forced["trace"][..., 0]
        assert np.all(_near_tie_ok(gpu_c_mse[mism], best[mism], gmax[mism])), \
            "a candidate mismatch that is not a near-tie"
        ref = forced
    assert np.array_equal(g_par, ref["params"])
    # the packed bytes hold the codes (the GPU's own unpack; nothing of the GPU's goes into
    # the oracle except the near-tie candidates above, which it validates first)
    assert np.array_equal(wq.unpack(pw.packed).cpu().numpy(), g_codes)
    # codes exact where the nearest-level margin is not a near-tie
    clear = ref["min_margin"] > 1e-6 * gmax
    cmatch = (g_codes.reshape(n, k // 32, 32) == ref["codes"].reshape(n, k // 32, 32)).all(-1)
    assert np.all(cmatch[clear]), f"{(~cmatch & clear).sum()} clear groups with different codes"
    lv_err = np.abs(g_lv - ref["levels"])[clear]
    assert np.all(lv_err <= 1e-5 * gmax[clear][:, None])
    # the trace is stored as fp32: compare where the MSE is inside fp32's range, with an
    # absolute floor of the smallest normal fp32
    tr = ref["trace"]
    inrange = (tr < 3.0e38)[clear]
    diff = np.abs(g_tr - tr)[clear]
    assert np.all((diff <= 1e-5 * tr[clear] + 2.0 ** -126)[inrange])
    assert np.all(np.isinf(g_tr[clear][~inrange]))
    # dequant of the oracle's codes and levels (as fp32, the stored format) is exactly the
    # oracle's reconstruction of them
    r_packed = oracle.pack(ref["codes"])
    r_levels = ref["levels"].astype(np.float32)
    rw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, torch.from_numpy(r_packed).cuda(),
                         torch.from_numpy(r_levels).cuda())
    d = wq.dequant(rw)
    assert np.array_equal(bits(d), oracle.dequant(oracle.LLOYD8S, r_packed, r_levels, 32))
    return mism.mean(), (~clear).mean()


def test_lloyd_g32_laplace_rowscaled(wq):
    w = workloads.laplace_rowscaled_weight(96, 2048, index=0)
    _check_lloyd(wq, w)


def test_lloyd_g32_edge_groups(wq):
    rng = np.random.default_rng(1)
    w = workloads.laplace_rowscaled_weight(8, 512, index=1)
    w[0, :32] = 0                                        # all zero (with a -0.0)
    w[0, 5] = 0x8000
    w[1, :32] = 0x3C80                                   # equal magnitudes, mixed signs
    w[1, :32:3] |= 0x8000
    w[2, :32] = 0
    w[2, 7] = 0x3F80                                     # a single nonzero weight
    w[3, :32] = workloads.f64_to_bf16_bits(rng.laplace(0, 1e-36, 32))   # tiny / subnormal
    w[4, :32] = workloads.f64_to_bf16_bits(rng.laplace(0, 1e35, 32))    # huge
    w[5, :32] = 0x3F80                                   # two magnitudes only
    w[5, ::2] = 0x3E80
    for rounds in (25, 0, 1):
        _check_lloyd(wq, w, rounds)


def test_lloyd_g32_full_size_matrix_sampled(wq):
    """A full 2048x2048 matrix of the 224-matrix workload on the GPU; 64 sampled rows
    (4096 groups) compared with the oracle. A group whose candidate differs must be a
    near-tie, and is then compared with the oracle re-run from the GPU's candidate."""
    w = workloads.laplace_rowscaled_weight(2048, 2048, index=7)
    pw, ex = wq.quantize_lloyd(to_dev_bits(w), wq.LLOYD_G32_WARM, 25, codes=True, trace=True)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(2).choice(2048, 64, replace=False))
    sub = w[rows]
    ref = oracle.lloyd(sub, 32, 25)
    g_par = ex["params"].cpu().numpy()[rows]
    g_cand = _cand_from_params(g_par)
    gmax = np.abs(oracle.bf16_to_f64(sub)).reshape(64, 64, 32).max(-1)
    mism = g_cand != ref["cand"]
    print(f"candidate mismatches: {mism.sum()} of {mism.size} groups")
    if mism.any():
        forced = oracle.lloyd(sub, 32, 25, force_cand=np.where(mism, g_cand, -1).astype(np.int32))
        assert np.all(_near_tie_ok(forced["trace"][..., 0][mism], ref["trace"][..., 0][mism], gmax[mism]))
        ref = forced
    assert np.array_equal(g_par, ref["params"])
    clear = ref["min_margin"] > 1e-6 * gmax
    g_codes = ex["codes"].cpu().numpy()[rows].reshape(64, 64, 32)
    assert np.all((g_codes == ref["codes"].reshape(64, 64, 32)).all(-1)[clear])
    g_lv = pw.aux.cpu().numpy()[rows].astype(np.float64)
    assert np.all(np.abs(g_lv - ref["levels"])[clear] <= 1e-5 * gmax[clear][:, None])
    assert (~clear).mean() < 1e-2


def _check_kmeans(wq, w_bits, rounds=25):
    n, k = w_bits.shape
    pw, ex = wq.quantize_lloyd(to_dev_bits(w_bits), wq.LLOYD_KMEANS16, rounds, codes=True, trace=True)
    pw2, ex2 = wq.quantize_lloyd(to_dev_bits(w_bits), wq.LLOYD_KMEANS16, rounds, codes=True, trace=True)
    torch.cuda.synchronize()
    ref = oracle.kmeans_lut16(w_bits, 64, rounds)
    assert np.array_equal(bits(pw.aux), ref["lut"])
    assert np.array_equal(ex["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(pw.packed.cpu().numpy(), oracle.pack(ref["codes"]))
    tr = ex["trace"].cpu().numpy().astype(np.float64)
    assert np.allclose(tr, ref["trace"], rtol=1e-6, atol=1e-30)
    # a second run gives the same bits (no order-dependent sums)
    assert np.array_equal(bits(pw2.aux), bits(pw.aux))
    assert np.array_equal(pw2.packed.cpu().numpy(), pw.packed.cpu().numpy())
    assert np.array_equal(ex2["trace"].cpu().numpy(), ex["trace"].cpu().numpy())


@pytest.mark.parametrize("heavy", [False, True])
def test_kmeans16_bit_exact(wq, heavy):
    w = workloads.lut16_weight(64, 2048, heavy_tail=heavy)
    _check_kmeans(wq, w)


def test_kmeans16_edge_blocks(wq):
    rng = np.random.default_rng(3)
    w = workloads.lut16_weight(4, 256, heavy_tail=True, index=5)
    w[0, :64] = 0x3C00                                  # all equal
    vals = workloads.f64_to_bf16_bits(np.sort(rng.standard_normal(16)) * 0.01)
    w[1, :64] = np.repeat(vals, 4)[rng.permutation(64)]  # 16 distinct values x 4
    w[2, :64] = 0                                        # all zero
    w[3, :64:2] = 0x8000                                 # zeros of both signs
    # a cluster near zero whose members have both signs and lie up to 100 binades apart
    # (an fp64 sum of them depends on its order), among 15 well separated values x 4
    wide = np.array([2.0 ** -20, -2.0 ** -20, 2.0 ** -100, -2.0 ** -60], dtype=np.float64)
    far = np.repeat(np.arange(1, 16, dtype=np.float64), 4)
    blk = np.concatenate([wide, far])[rng.permutation(64)]
    w[2, 64:128] = workloads.f64_to_bf16_bits(blk)
    for rounds in (25, 0, 3):
        _check_kmeans(wq, w, rounds)


def test_kmeans16_full_size_sampled(wq):
    """The 8192x28672 LUT16 workload (Student-t) quantised on the GPU; 16 sampled rows
    (7168 blocks) compared with the oracle bit for bit."""
    w = workloads.lut16_weight(8192, 28672, heavy_tail=True)
    pw, ex = wq.quantize_lloyd(to_dev_bits(w), wq.LLOYD_KMEANS16, 25)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(4).choice(8192, 16, replace=False))
    ref = oracle.kmeans_lut16(w[rows], 64, 25)
    assert np.array_equal(bits(pw.aux)[rows], ref["lut"])
    assert np.array_equal(pw.packed.cpu().numpy()[rows], oracle.pack(ref["codes"]))
