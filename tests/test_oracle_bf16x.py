"""Pins of the BF16X oracle ("同一个 1B 模型，我上了三种压缩方案…", section "第一剑·完美主义：
BF16X"): a lossless codec, so decode(encode(w)) must give back every bit; the escape count
is recomputed from the values by another route; a two-block example is worked by hand.
"""
import numpy as np
import pytest

import oracle
import workloads


def _f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def test_bf16x_hand_worked_blocks():
    # block 0: 1.0, -2.0, 0.0, 1.5, 2^-5, 2^-6, -0.0, then 1.0 x 9. Exponent fields 127,
    # 128, 0, 127, 122, 121, 0, 127...; E = 128; differences 1, 0, 128, 1, 6, 7, 128, 1...
    # Stored fields 1, 0, 7, 1, 6, 7, 7, 1 x 9 (6 still fits, 7 and more escape).
    #   plane 0 (bit 0 of each field): weights 0, 2, 3, 5, 6, 7..15 -> 0xFFED
    #   plane 1 (bit 1): weights 2, 4, 5, 6 -> 0x0074; plane 2 (bit 2): the same -> 0x0074
    # block 1: 1.0 x 16 except weight 9 = 2^-7 (field 120): E = 127, weight 9 escapes;
    #   planes 0x0200 each; three escapes precede it in the superblock.
    # Headers: E << 48 | plane2 << 32 | plane1 << 16 | plane0, prefix << 56.
    b0 = [0x3F80, 0xC000, 0x0000, 0x3FC0, 0x3D00, 0x3C80, 0x8000] + [0x3F80] * 9
    b1 = [0x3F80] * 16
    b1[9] = 0x3C00
    w = np.array([b0 + b1], np.uint16)
    enc = oracle.bf16x_encode(w)
    assert [hex(int(h)) for h in enc["hdr"][0]] == ["0x8000740074ffed", "0x37f020002000200"]
    assert enc["sm"][0, :16].tolist() == [0, 0x80, 0, 0x40, 0, 0, 0x80] + [0] * 9
    assert enc["sm"][0, 16:].tolist() == [0] * 16
    assert enc["ovf"].tolist() == [0, 121, 0, 120]
    assert enc["sb_off"].tolist() == [0, 4]
    assert np.array_equal(oracle.bf16x_decode(enc, 1, 32), w)


def test_bf16x_every_bf16_pattern_round_trips():
    allp = np.arange(65536, dtype=np.uint16)
    for order in (allp, np.random.default_rng(7).permutation(allp)):
        w = order.reshape(16, 4096)
        enc = oracle.bf16x_encode(w)
        assert np.array_equal(oracle.bf16x_decode(enc, 16, 4096), w)


@pytest.mark.parametrize("n,k", [(3, 16), (5, 48), (64, 4096), (7, 272)])
def test_bf16x_escape_count_by_frexp(n, k):
    w = workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, n * 1000 + k)
    # also some zeros, subnormals and an Inf to reach every exponent class
    w.reshape(-1)[::97] = 0
    w.reshape(-1)[5::211] = 0x0003
    w.reshape(-1)[-1] = 0x7F80
    v = _f32(w).astype(np.float64)
    mant, x = np.frexp(np.abs(v))
    e = np.where(v == 0, 0, np.maximum(x + 126, 0))
    e = np.where(np.isinf(v) | np.isnan(v), 255, e)
    blocks = e.reshape(-1, 16)
    esc = (blocks.max(axis=1, keepdims=True) - blocks) >= 7
    enc = oracle.bf16x_encode(w)
    assert enc["ovf"].size == esc.sum()
    per_sb = np.add.reduceat(esc.sum(axis=1), np.arange(0, blocks.shape[0], 16))
    assert enc["sb_off"].tolist() == [0] + np.cumsum(per_sb).tolist()
    assert np.array_equal(enc["ovf"], e.reshape(-1)[esc.reshape(-1)].astype(np.uint8))
    assert np.array_equal(oracle.bf16x_decode(enc, n, k), w)
    # structure: the block maximum is never escaped; an escape needs E >= 7
    hdr = enc["hdr"].reshape(-1)
    planes = [(hdr >> np.uint64(16 * p)) & np.uint64(0xFFFF) for p in range(3)]
    fields = sum(((planes[p][:, None] >> np.arange(16, dtype=np.uint64)) & np.uint64(1)) << np.uint64(p)
                 for p in range(3)).astype(np.int64)
    emax = ((hdr >> np.uint64(48)) & np.uint64(0xFF)).astype(np.int64)
    assert (fields == 0).any(axis=1).all()
    assert (emax[(fields == 7).any(axis=1)] >= 7).all()
    assert np.array_equal(enc["sm"] >> 7, (w >> 15).astype(np.uint8))


def test_bf16x_decode_rejects_a_wrong_prefix():
    w = workloads.gaussian_outlier_weight(4, 256, workloads.DECODE_SWEEP, 3)
    enc = oracle.bf16x_encode(w)
    assert enc["ovf"].size > 0
    bad = dict(enc, hdr=enc["hdr"].copy())
    i = int(np.argmax((bad["hdr"].reshape(-1) >> np.uint64(56)) > 0))
    bad["hdr"].reshape(-1)[i] += np.uint64(1) << np.uint64(56)
    with pytest.raises(ValueError):
        oracle.bf16x_decode(bad, 4, 256)
