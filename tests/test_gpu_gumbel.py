"""GPU parity of the Gumbel-ST backward ("MiniCPM5-1B 验证…" §2.3 "Gumbel-ST": soft =
softmax(-dist/tau) . codes, q = hard + (soft - soft.detach())) with the oracle, through the C
ABI: the latent gradient per element and the scale gradient per group, across temperatures
from far below to far above step^2 (the page's own 5 -> 0.3 anneal included), latents beyond
a trained scale, zero scales, ragged shapes and sampled rows of a full-size launch.

Tolerance (fp32 kernel, fp64 oracle; wq.h states it): the kernel forms each softmax weight
with one ex2 of a logit taken relative to the nearest code (a few ulp of relative error,
plus ulps of the logit), sums 16 weights and their central moments in fp32 and multiplies a
handful of factors: about 1e-6 relative in all, against a bound of 1e-4. Weights below fp32's
normal range are flushed, hence the absolute floor 2^-100 |gq| (1 + 2 step^2 / tau). The
scale gradient is a signed sum over the group; it is held to 1e-4 of the sum of the absolute
values of the exact derivative's terms (the oracle's gscale_mag)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import to_dev_bits

pytestmark = pytest.mark.gpu


def _inputs(seed, n, k, group, zs=0.02, spread=0.4, zero_groups=False):
    g = np.random.default_rng(seed)
    z = (g.standard_normal((n, k)) * zs).astype(np.float32)
    amax = np.abs(z.astype(np.float64)).reshape(n, k // group, group).max(-1)
    scale = workloads.f64_to_bf16_bits(amax * g.uniform(1 - spread, 1 + spread, amax.shape))
    if zero_groups:
        scale.reshape(-1)[::5] = 0
    gq = g.standard_normal((n, k)).astype(np.float32)
    return z, scale, gq


def _run(wq, z, scale, gq, tau, group, scale_grad=True):
    gz, gs = wq.gumbel_st_backward(torch.from_numpy(z).cuda(), to_dev_bits(scale),
                                   torch.from_numpy(gq).cuda(), tau, group, scale_grad=scale_grad)
    torch.cuda.synchronize()
    return gz.cpu().numpy().astype(np.float64), None if gs is None else gs.cpu().numpy().astype(np.float64)


def _check(z, scale, gq, tau, group, gz, gs, rows=None):
    if rows is not None:
        z, scale, gq = z[rows], scale[rows], gq[rows]
        gz = gz[rows]
        gs = None if gs is None else gs[rows]
    gz_ref, gs_ref, _, gs_mag = oracle.gumbel_st_backward(z, scale, gq, tau, group)
    step = np.repeat(oracle.bf16_to_f64(scale), group, axis=1) / 8
    floor = 2.0 ** -100 * np.abs(gq.astype(np.float64)) * (1 + 2 * step * step / tau)
    err = np.abs(gz - gz_ref)
    assert np.all(err <= 1e-4 * np.abs(gz_ref.astype(np.float64)) + floor), \
        f"gz: worst {np.max(err / (np.abs(gz_ref) + floor)):.3e} relative"
    if gs is not None:
        assert np.all(np.abs(gs - gs_ref) <= 1e-4 * gs_mag + 1e-30), \
            f"gscale: worst {np.max(np.abs(gs - gs_ref) / (gs_mag + 1e-300)):.3e} of the term sum"
    return float(np.max(err / (np.abs(gz_ref) + floor)))


@pytest.mark.parametrize("group", [64, 32])
@pytest.mark.parametrize("tau_over_step2", [0.05, 0.3, 1.0, 30.0, 3000.0])
def test_matches_oracle_across_temperatures(wq, group, tau_over_step2):
    n, k = 9, 2 * 1024 + group                       # several warps and a ragged last one
    z, scale, gq = _inputs(int(tau_over_step2 * 100) + group, n, k, group)
    step = float(np.median(oracle.bf16_to_f64(scale))) / 8
    tau = tau_over_step2 * step * step
    gz, gs = _run(wq, z, scale, gq, tau, group)
    _check(z, scale, gq, tau, group, gz, gs)


@pytest.mark.parametrize("tau", [5.0, 3.0, 1.0, 0.5, 0.3])
def test_the_pages_temperatures(wq, tau):
    # the anneals of §3.4 (5 -> 0.3, 3 -> 0.5, 1 -> 0.5) on weight-magnitude latents
    z, scale, gq = _inputs(int(tau * 10), 16, 4096, 64)
    gz, gs = _run(wq, z, scale, gq, tau, 64)
    _check(z, scale, gq, tau, 64, gz, gs)


@pytest.mark.parametrize("n,k,group", [(1, 32, 32), (1, 64, 64), (3, 96, 32), (5, 4160, 64)])
def test_ragged_shapes_zero_scales_and_no_scale_gradient(wq, n, k, group):
    z, scale, gq = _inputs(n * k, n, k, group, zero_groups=True)
    tau = 2.0 * (float(np.max(oracle.bf16_to_f64(scale))) / 8) ** 2 + 1e-12
    gz, gs = _run(wq, z, scale, gq, tau, group)
    _check(z, scale, gq, tau, group, gz, gs)
    zero = np.repeat(scale == 0, group, axis=1)
    assert np.all(gz[zero] == 0)                     # every code is 0: no z gradient
    gz2, none = _run(wq, z, scale, gq, tau, group, scale_grad=False)
    assert none is None and np.array_equal(gz2, gz)


def test_full_size_launch_sampled_rows(wq):
    # the 8192 x 28672 shape of the LUT16 workload as one fp32 latent, rows checked by sample
    n, k = workloads.LUT16_SHAPE
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev).manual_seed(3)
    zt = torch.randn((n, k), device=dev, generator=gen).mul_(0.02)
    st = (zt.abs().reshape(n, k // 64, 64).amax(-1) * 1.1).to(torch.bfloat16)
    gqt = torch.randn((n, k), device=dev, generator=gen)
    tau = 1e-5
    gz, gs = wq.gumbel_st_backward(zt, st, gqt, tau, 64)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 4095, 5000, n - 1])
    sel = torch.from_numpy(rows).to(dev)
    z = zt[sel].cpu().numpy()
    scale = st[sel].view(torch.int16).cpu().numpy().view(np.uint16)
    gq = gqt[sel].cpu().numpy()
    _check(z, scale, gq, tau, 64, gz[sel].cpu().numpy().astype(np.float64),
           gs[sel].cpu().numpy().astype(np.float64))


def test_rejects_bad_temperature_through_the_c_abi(wq):
    z = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    s = torch.zeros((1, 1), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(z)
    for tau in (0.0, -1.0, float("nan"), float("inf"), 1e-39):
        st = wq._lib.wq_gumbel_st_backward(wq._ptr(z), 1, 64, 64, wq._ptr(s), ctypes.c_float(tau),
                                           wq._ptr(z), wq._ptr(out), None,
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == wq.WQ_EINVAL, tau
