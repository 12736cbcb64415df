"""GPU parity of the STE fake-quantisation forward ("MiniCPM5-1B 验证…" §2.3) with the oracle:
codes, packed bytes and the fp32 forward values bit-exact, on random latents (some beyond
their scale, as a trained scale allows), on every midpoint and its neighbours, and on scales
that take the kernel's double-precision path."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, to_dev_bits

pytestmark = pytest.mark.gpu


def _run(wq, z, scale_bits, group):
    zt = torch.from_numpy(z).cuda()
    q, c, p = wq.fake_quant_ste(zt, to_dev_bits(scale_bits), group, codes=True, packed=True)
    torch.cuda.synchronize()
    return q.cpu().numpy(), c.cpu().numpy(), p.cpu().numpy()


def _compare(wq, z, scale_bits, group):
    q, c, p = _run(wq, z, scale_bits, group)
    q_ref, c_ref = oracle.fake_quant_ste(z, scale_bits, group)
    assert np.array_equal(c, c_ref)
    assert np.array_equal(q.view(np.uint32), q_ref.view(np.uint32))      # bit-exact, signs too
    assert np.array_equal(p, oracle.pack(c_ref))


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("n,k", [(1, 64), (7, 320), (64, 1024), (33, 2144)])
def test_fake_quant_matches_oracle(wq, n, k, group):
    if k % group:
        pytest.skip("k not a multiple of the group")
    g = np.random.default_rng(n * k + group)
    z = (g.standard_normal((n, k)) * 0.03).astype(np.float32)
    amax = np.abs(z.reshape(n, k // group, group)).max(-1)
    scale = workloads.f64_to_bf16_bits(amax * g.uniform(0.5, 1.2, amax.shape))
    _compare(wq, z, scale, group)


@pytest.mark.parametrize("scale_value", [1.0, 0.0371, 3.0e-3, 2.0 ** -100, 2.0 ** 100, 1e-40, 0.0])
def test_fake_quant_every_midpoint_and_neighbour(wq, scale_value):
    """z on every midpoint (2j - 17) s / 16, one fp32 ulp either side, every code value, and
    points beyond the range: the tie rule and both correction directions."""
    s_bits = workloads.f64_to_bf16_bits(np.array([scale_value]))
    s = float(oracle.bf16_to_f64(s_bits)[0])
    pts = []
    for j in range(0, 18):
        m = np.float32((2 * j - 17) * s / 16)
        pts += [m, np.nextafter(m, np.float32(np.inf)), np.nextafter(m, np.float32(-np.inf))]
    for j in range(16):
        pts.append(np.float32((j - 8) * s / 8))
    pts += [np.float32(3 * s + 1e-30), np.float32(-3 * s - 1e-30), np.float32(0.0), np.float32(-0.0)]
    z = np.array(pts, np.float32)
    z = np.concatenate([z, np.zeros((-z.size) % 64, np.float32)]).reshape(-1, 64)
    scale = np.full((z.shape[0], 1), s_bits[0], np.uint16)
    _compare(wq, z, scale, 64)


def test_fake_quant_large_matrix_sampled(wq):
    n, k = 2048, 8192
    g = np.random.default_rng(9)
    z = (g.standard_normal((n, k)) * 0.02).astype(np.float32)
    amax = np.abs(z.reshape(n, k // 64, 64)).max(-1)
    scale = workloads.f64_to_bf16_bits(amax)
    q, c, _ = _run(wq, z, scale, 64)
    rows = g.choice(n, 64, replace=False)
    q_ref, c_ref = oracle.fake_quant_ste(z[rows], scale[rows], 64)
    assert np.array_equal(c[rows], c_ref)
    assert np.array_equal(q[rows].view(np.uint32), q_ref.view(np.uint32))
