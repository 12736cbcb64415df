"""GPU parity of the BF16X codec ("同一个 1B 模型，我上了三种压缩方案…", section "第一剑·完美主义：
BF16X") with the oracle: every field of the encoding (sign/mantissa bytes, headers,
superblock offsets, overflow table) bit-exact, decoding bit-exact both on the GPU's own
encoding and on the oracle's, over every bf16 pattern, ragged superblock tails and a
full-size projection of the decode-sweep stack; a too-short overflow table is flagged
without any access past it."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, to_dev_bits

pytestmark = pytest.mark.gpu


def _host(b):
    return dict(sm=b.sm.cpu().numpy(), hdr=b.hdr.cpu().numpy().view(np.uint64),
                sb_off=b.sb_off.cpu().numpy().view(np.uint32),
                ovf=b.ovf.cpu().numpy()[:b.escapes])


def _dev(wq, enc, n, k):
    ovf = np.zeros(max(enc["ovf"].size, 16), np.uint8)
    ovf[:enc["ovf"].size] = enc["ovf"]
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a).view(dt)).cuda()
    return wq.Bf16xWeight(n, k, t(enc["sm"], np.uint8), t(enc["hdr"], np.int64),
                          t(enc["sb_off"], np.int32), t(ovf, np.uint8), int(enc["ovf"].size))


def _check(wq, w_bits):
    n, k = w_bits.shape
    w = to_dev_bits(w_bits)
    b = wq.bf16x_encode(w)
    out = wq.bf16x_decode(b)
    torch.cuda.synchronize()
    ref = oracle.bf16x_encode(w_bits)
    got = _host(b)
    for key in ("sm", "hdr", "sb_off", "ovf"):
        assert np.array_equal(got[key], ref[key]), key
    assert b.escapes == ref["ovf"].size
    assert np.array_equal(bits(out), w_bits)
    # the GPU decoder on the oracle's encoding
    out2 = wq.bf16x_decode(_dev(wq, ref, n, k))
    assert np.array_equal(bits(out2), w_bits)
    assert wq.device_error() == 0
    return b


@pytest.mark.parametrize("n,k", [(1, 32), (3, 96), (5, 4128), (64, 4096), (7, 2080)])
def test_bf16x_matches_oracle(wq, n, k):
    w = workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, n * 100 + k)
    w.reshape(-1)[::61] = 0                                     # zeros escape below E >= 7
    _check(wq, w)


def test_bf16x_every_bf16_pattern(wq):
    allp = np.arange(65536, dtype=np.uint16)
    _check(wq, allp.reshape(16, 4096))
    _check(wq, np.random.default_rng(11).permutation(allp).reshape(64, 1024))


def test_bf16x_blocks_without_escapes_and_all_escaped(wq):
    w = np.full((2, 256), 0x3F80, np.uint16)                     # 1.0 everywhere: none
    w[1, ::16] = 0x7F80                                          # Inf heads: 15 escapes per block
    b = _check(wq, w)
    assert b.escapes == 16 * 15


def test_bf16x_full_size_projection(wq):
    # the gate projection of the decode-sweep stack (5632 x 2048), as the benchmark decodes it
    n, k = workloads.INTERMEDIATE, workloads.HIDDEN
    _check(wq, workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, 4))


def test_bf16x_short_overflow_table_is_flagged(wq):
    n, k = 8, 4096
    w_bits = workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, 9)
    ref = oracle.bf16x_encode(w_bits)
    assert ref["ovf"].size > 16
    b = _dev(wq, ref, n, k)
    short = wq.Bf16xWeight(n, k, b.sm, b.hdr, b.sb_off, b.ovf[:16].clone(), b.escapes)
    assert wq.device_error() == 0
    wq.bf16x_decode(short)
    torch.cuda.synchronize()
    assert wq.device_error() == 1000
    assert wq.device_error() == 0                                # read clears it
    # an encode whose offsets do not fit the table: skipped and flagged the same way
    w = to_dev_bits(w_bits)
    wq.bf16x_encode_into(w, short)
    torch.cuda.synchronize()
    assert wq.device_error() == 1001


def test_bf16x_argument_checks(wq):
    w = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")      # k % 32 != 0
    with pytest.raises(wq.WqError):
        wq.bf16x_encode(w)
    assert wq.bf16x_superblocks(4, 40) == -1
    assert wq.bf16x_superblocks(3, 96) == 2
