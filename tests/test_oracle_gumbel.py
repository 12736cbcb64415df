"""Pins of the oracle's Gumbel-ST backward ("MiniCPM5-1B 验证…" §2.3 "Gumbel-ST": soft =
softmax(-dist/tau) . codes, hard = codes[argmin(dist)], q = hard + (soft - soft.detach())).

The oracle writes the chain rule out term by term. It is pinned against things that do not
share that derivation: torch autograd (float64) run on the page's own forward expression,
a complex-step derivative of the soft assignment, 50-digit numerical derivatives (mpmath)
where float64 autograd itself loses digits (low temperature, latents beyond the scale), and
closed forms at the degenerate points (zero scale, a midpoint at low temperature, the
uniform limit at high temperature)."""
import mpmath
import numpy as np
import torch

import oracle
import workloads


def _autograd(z, scale_bits, gq, tau, group):
    """The page's forward expression, differentiated by torch autograd in float64."""
    n, k = z.shape
    zt = torch.tensor(z.astype(np.float64), requires_grad=True)
    st = torch.tensor(oracle.bf16_to_f64(scale_bits), requires_grad=True)
    step = st.repeat_interleave(group, dim=1) / 8                     # [n, k]
    codes = step[..., None] * torch.arange(-8, 8, dtype=torch.float64)  # [n, k, 16]
    dist = (zt[..., None] - codes) ** 2
    soft = (torch.softmax(-dist / tau, dim=-1) * codes).sum(-1)
    idx = torch.argmin(dist, dim=-1)                                  # first minimum on a tie
    hard = torch.gather(codes, -1, idx[..., None])[..., 0]
    q = hard + (soft - soft.detach())
    (q * torch.tensor(gq.astype(np.float64))).sum().backward()
    return zt.grad.numpy(), st.grad.numpy(), q.detach().numpy()


def _case(seed, n=6, k=128, group=64, zs=0.02, tau_over_step2=None, tau=None, spread=0.0):
    """Latents N(0, zs^2), scales = group absmax times U(1 - spread, 1 + spread) (a trained
    scale: spread > 0 leaves some latents beyond it)."""
    g = np.random.default_rng(seed)
    z = (g.standard_normal((n, k)) * zs).astype(np.float32)
    scale = workloads.f64_to_bf16_bits(np.abs(z.astype(np.float64)).reshape(n, k // group, group).max(-1)
                                       * g.uniform(1 - spread, 1 + spread, (n, k // group)))
    gq = g.standard_normal((n, k)).astype(np.float32)
    if tau is None:
        step = float(np.median(oracle.bf16_to_f64(scale))) / 8
        tau = tau_over_step2 * step * step
    return z, scale, gq, tau


def test_matches_autograd_of_the_printed_forward():
    # latents within the scale and tau >= step^2: float64 autograd is accurate here
    for seed, t in [(1, 1.0), (2, 3.0), (3, 30.0), (4, 300.0)]:
        z, scale, gq, tau = _case(seed, tau_over_step2=t)
        gz, gs, gz_mag, gs_mag = oracle.gumbel_st_backward(z, scale, gq, tau, 64)
        gz_ref, gs_ref, q = _autograd(z, scale, gq, tau, 64)
        # gz is the float32 rounding of the oracle's double
        assert np.all(np.abs(gz - gz_ref) <= 2 ** -24 * np.abs(gz_ref) + 1e-11 * gz_mag)
        assert np.all(np.abs(gs - gs_ref) <= 1e-11 * gs_mag)
        # the forward value is the hard code value, which is the STE forward
        q_ste, _ = oracle.fake_quant_ste(z, scale, 64)
        assert np.array_equal(q.astype(np.float32), q_ste)


def test_the_pages_temperatures_on_weight_scale_latents():
    # tau annealed 5 -> 0.3 and 3 -> 0.5 on latents of weight magnitude (the ablation of §3.4)
    for seed, tau in [(5, 5.0), (6, 0.3), (7, 0.5)]:
        z, scale, gq, tau = _case(seed, group=32, tau=tau)
        gz, gs, gz_mag, gs_mag = oracle.gumbel_st_backward(z, scale, gq, tau, 32)
        gz_ref, gs_ref, _ = _autograd(z, scale, gq, tau, 32)
        assert np.all(np.abs(gz - gz_ref) <= 2 ** -24 * np.abs(gz_ref) + 1e-11 * gz_mag)
        assert np.all(np.abs(gs - gs_ref) <= 1e-11 * gs_mag)


def _mp_soft(zv, s, tau):
    step = s / 8
    codes = [step * (j - 8) for j in range(16)]
    lg = [-(zv - c) ** 2 / tau for c in codes]
    m = max(lg)
    p = [mpmath.e ** (x - m) for x in lg]
    return sum(pi * c for pi, c in zip(p, codes)) / sum(p)


def test_against_50_digit_derivatives_where_float64_autograd_loses_digits():
    # low temperature and latents up to 1.5x beyond a trained scale: d soft/d z is a small
    # difference of large softmax terms here (float64 autograd is off by ~1e-5 relative)
    mpmath.mp.dps = 50
    for seed, t in [(11, 0.3), (12, 0.05), (13, 2.0)]:
        z, scale, gq, tau = _case(seed, n=2, k=64, group=32, tau_over_step2=t, spread=0.4)
        gq = np.ones_like(gq)
        gz, gs, _, _ = oracle.gumbel_st_backward(z, scale, gq, tau, 32)
        sv = oracle.bf16_to_f64(scale)
        for r in range(2):
            for g in range(2):
                s = mpmath.mpf(float(sv[r, g]))
                want_s = mpmath.mpf(0)
                for c in range(32 * g, 32 * g + 32):
                    zv = mpmath.mpf(float(z[r, c]))
                    d_z = mpmath.diff(lambda x: _mp_soft(x, s, tau), zv)
                    assert abs(gz[r, c] - float(d_z)) <= 2 ** -24 * abs(float(d_z)) + 1e-300
                    idx = min(range(16), key=lambda j: (abs(zv - s / 8 * (j - 8)), j))
                    want_s += mpmath.mpf(idx - 8) / 8 + mpmath.diff(lambda y: _mp_soft(zv, y, tau), s)
                assert abs(gs[r, g] - float(want_s)) <= 1e-12 * (abs(float(want_s)) + 1)


def test_dz_against_a_complex_step_derivative():
    # d soft / d z by the complex step: soft(z + i h) evaluated in complex arithmetic, Im / h
    g = np.random.default_rng(8)
    s = 0.05
    step = s / 8
    codes = step * np.arange(-8, 8)
    for tau in (0.3 * step * step, 4 * step * step, 50 * step * step):
        zs = g.uniform(-1.2 * s, 1.2 * s, 40).astype(np.float32)
        z = np.tile(zs, (1, 1)).reshape(1, 40)
        z = np.concatenate([z, np.zeros((1, 24), np.float32)], axis=1)
        scale = workloads.f64_to_bf16_bits(np.array([[s]]))
        s_exact = float(oracle.bf16_to_f64(scale)[0, 0])
        codes = s_exact / 8 * np.arange(-8, 8)
        gz, _, _, _ = oracle.gumbel_st_backward(z, scale, np.ones((1, 64), np.float32), tau, 64)
        h = 1e-30
        for i, zz in enumerate(z[0, :40].astype(np.float64)):
            zc = zz + 1j * h
            lg = -(zc - codes) ** 2 / tau
            lg = lg - lg.real.max()
            p = np.exp(lg)
            soft = (p * codes).sum() / p.sum()
            assert abs(gz[0, i] - soft.imag / h) <= 1e-6 * abs(soft.imag / h) + 1e-30


def test_zero_scale():
    # every code is 0: p is uniform over 16 codes, the soft path has no z gradient, and
    # d q / d scale = (0 - 8)/8 (hard: idx 0 on the all-way tie) + mean of (j - 8)/8 = -17/16
    z = np.random.default_rng(9).standard_normal((2, 64)).astype(np.float32)
    gq = np.random.default_rng(10).standard_normal((2, 64)).astype(np.float32)
    scale = np.zeros((2, 1), np.uint16)
    gz, gs, _, _ = oracle.gumbel_st_backward(z, scale, gq, 0.7, 64)
    assert np.all(gz == 0)
    assert np.allclose(gs[:, 0], gq.astype(np.float64).sum(1) * (-17 / 16), rtol=1e-14)


def test_midpoint_at_low_temperature():
    # z halfway between two codes, tau = step^2/100: the two codes share the mass, every
    # other code is e^-200 smaller, so Var = (step/2)^2 and d soft/d z = step^2 / (2 tau) = 50
    s = 0.0625
    step = s / 8
    scale = workloads.f64_to_bf16_bits(np.array([[s]]))
    z = np.zeros((1, 32), np.float32)
    mids = [(j - 8 + 0.5) * step for j in range(15)]
    z[0, :15] = np.array(mids, np.float32)            # exact: step is a power of two here
    tau = step * step / 100
    gz, _, _, _ = oracle.gumbel_st_backward(z, scale, np.ones((1, 32), np.float32), tau, 32)
    assert np.allclose(gz[0, :15], 50.0, rtol=1e-12)


def test_uniform_limit_at_high_temperature():
    # tau >> (scale)^2: p -> uniform, d soft / d z -> (2/tau) Var(codes) = (2/tau) step^2 * 21.25
    s = 0.04
    scale = workloads.f64_to_bf16_bits(np.array([[s]]))
    step = float(oracle.bf16_to_f64(scale)[0, 0]) / 8
    tau = 1e9 * step * step
    z = np.linspace(-s, s, 64).astype(np.float32).reshape(1, 64)
    gz, _, _, _ = oracle.gumbel_st_backward(z, scale, np.ones((1, 64), np.float32), tau, 64)
    assert np.allclose(gz[0], 2 / tau * step * step * 21.25, rtol=1e-6)
