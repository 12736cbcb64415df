"""Pins for the oracle's Lloyd g32 producer ([G32] = "int4-g32+warm 裸量化：原理与实验报告")
and its LUT16 k-means producer ([KM] = "K-Means量化技术：突破LLM低比特部署瓶颈").

What pins what:
  * the candidate grid against the lists printed in [G32] §1.2 (tests/golden);
  * the inverse transforms against the page's own fixed-point iteration and closed forms;
  * the search against groups built from a candidate's own levels (MSE must reach 0);
  * Lloyd against the k-means properties of [G32] §1.3 step 3 (non-increasing MSE,
    levels equal to their members' means, every code nearest);
  * special cases (all-equal magnitudes, all zero);
  * ordering claims of [G32] §1.4 on synthetic Laplace data (warm <= parametric,
    g32 < g64 < g128). The absolute MSE figures of [G32] §1.4 are parity unpinned.
"""
import math
import os

import numpy as np
import pytest

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden", "lloyd_candidates.txt")


def _golden():
    vals = {}
    for line in open(GOLD):
        line = line.split("#")[0].split()
        if line:
            vals[line[0]] = [float(v) for v in line[1:]]
    return vals


def test_candidate_grid_matches_page_lists():
    gold = _golden()
    assert len(gold["rational_b_rel_endpoints"]) == 2
    cands = [oracle.lloyd_candidate(c) for c in range(112)]
    rat = [c for c in cands if c[0] == 0]
    tnh = [c for c in cands if c[0] == 1]
    assert len(rat) == 105 and len(tnh) == 7
    brel = sorted({round(c[1], 12) for c in rat})
    assert len(brel) == 15
    assert brel[0] == pytest.approx(gold["rational_b_rel_endpoints"][0], rel=1e-15)
    assert brel[-1] == pytest.approx(gold["rational_b_rel_endpoints"][1], rel=1e-15)
    ratios = np.diff(np.log10(brel))                                   # logspace: equal steps
    assert np.allclose(ratios, 5.0 / 14.0, rtol=1e-9)
    assert sorted({c[2] for c in rat}) == gold["rational_beta"]
    assert [c[1] for c in tnh] == gold["tanh_b_rel"]
    # params byte: family(1) | b_rel index(4) | beta index(3), [G32] §2
    bytes_ = [oracle.lloyd_params_byte(c) for c in range(112)]
    assert len(set(bytes_)) == 112 and max(bytes_) < 256
    for c in range(112):
        fam, brel_c, beta = cands[c]
        b = bytes_[c]
        assert (b >> 7) == fam
        if fam == 0:
            assert math.isclose(10 ** (-3 + 5 * ((b >> 3) & 15) / 14), brel_c, rel_tol=1e-12)
            assert gold["rational_beta"][b & 7] == beta
        else:
            assert gold["tanh_b_rel"][(b >> 3) & 15] == brel_c and (b & 7) == 0


@pytest.mark.parametrize("beta", [0.5, 0.55, 0.65, 0.75, 0.85, 0.95])
def test_rational_inverse_matches_page_fixed_point(beta):
    """[G32] §1.2: for beta < 1 the page inverts by iterating w <- fd*b + fd*w^beta. Run that
    iteration to convergence in Python and compare with the oracle's root."""
    gmax = 0.0731
    for b_rel in (1e-3, 0.05, 1.0, 30.0):
        b = b_rel * gmax
        fmax = gmax / (b + gmax ** beta)
        for q in range(1, 7):
            fd = q / 7 * fmax
            w = gmax
            for _ in range(20000):
                w_new = fd * b + fd * w ** beta
                if abs(w_new - w) <= 1e-18:
                    break
                w = w_new
            got = oracle.lloyd_inverse(0, fd, b, beta, gmax)
            assert got == pytest.approx(w, rel=1e-9, abs=1e-15)
            assert got / (b + got ** beta) == pytest.approx(fd, rel=1e-13)


def test_closed_form_inverses():
    gmax = 0.25
    for b_rel in (1e-3, 0.3, 100.0):                  # beta = 1: w = fd*b / (1 - fd)
        b = b_rel * gmax
        for fd in (0.01, 0.3, 0.9 * gmax / (b + gmax)):
            w = oracle.lloyd_inverse(0, fd, b, 1.0, gmax)
            assert w / (b + w) == pytest.approx(fd, rel=1e-13)
    for b_rel in (0.25, 0.4, 3.0):                    # tanh: w = b * atanh(fd)
        b = b_rel * gmax
        for fd in (0.05, 0.5, 0.9 * math.tanh(gmax / b)):
            w = oracle.lloyd_inverse(1, fd, b, 1.0, gmax)
            assert math.tanh(w / b) == pytest.approx(fd, rel=1e-13)


def _levels_of(c, gmax):
    fam, b_rel, beta = oracle.lloyd_candidate(c)
    b = b_rel * gmax
    f = (lambda a: a / (b + a ** beta)) if fam == 0 else (lambda a: math.tanh(a / b))
    fmax = f(gmax)
    return [0.0] + [oracle.lloyd_inverse(fam, q / 7 * fmax, b, beta, gmax) for q in range(1, 7)] + [gmax]


@pytest.mark.parametrize("c", [0, 3, 6, 50, 97, 104, 105, 108, 111])
def test_group_made_of_a_candidates_levels_reaches_zero_mse(c):
    """Weights that are exactly (bf16 copies of) the 8 levels of candidate c for their gmax:
    the search must find a candidate whose MSE is 0 up to the bf16 rounding of the levels,
    and Lloyd must then reproduce the weights exactly."""
    gmax_bits = 0x3D96                                 # 0.0732421875
    gmax = oracle.bf16_to_f64(np.array([gmax_bits], np.uint16))[0]
    lv = _levels_of(c, gmax)
    lv_bits = oracle.f64_to_bf16(np.array(lv))
    lv_bits[-1] = gmax_bits
    w = np.tile(lv_bits, 4).reshape(1, 32)
    w[0, 1::2] |= 0x8000                               # signs must not matter
    res = oracle.lloyd(w, 32, 25, threads=1)
    lvq = oracle.bf16_to_f64(lv_bits)
    cand_mse = res["trace"][0, 0, 0]
    assert cand_mse <= np.max(np.abs(lvq - np.array(lv))) ** 2 + 1e-30
    assert res["trace"][0, 0, -1] == 0.0
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.LLOYD8S, oracle.pack(res["codes"]),
                                           res["levels"].astype(np.float32), 32))
    assert np.array_equal(wd, oracle.bf16_to_f64(w))


def test_all_equal_magnitudes_and_all_zero():
    w = np.full((1, 32), 0x3C80, np.uint16)
    w[0, ::3] |= 0x8000
    res = oracle.lloyd(w, 32, 25, threads=1)
    assert res["cand"][0, 0] == 0 and res["trace"][0, 0, 0] == 0.0
    assert np.array_equal(res["codes"][0] & 7, np.full(32, 7))
    assert np.array_equal(res["codes"][0] >> 3, (w[0] >> 15).astype(np.uint8))
    z = np.zeros((1, 64), np.uint16)
    z[0, 7] = 0x8000
    res = oracle.lloyd(z, 32, 25, threads=1)
    assert np.all(res["codes"] == 0) and np.all(res["levels"] == 0) and np.all(res["cand"] == 0)


def _check_kmeans_properties(a, codes_q, levels):
    """Every magnitude is assigned to a nearest level (lowest index on a tie)."""
    d = np.abs(a[..., None] - levels[..., None, :])
    nearest = np.argmin(d, axis=-1)
    assert np.array_equal(codes_q, nearest)


def test_lloyd_properties_on_laplace_workload():
    w = workloads.laplace_rowscaled_weight(48, 512)
    res = oracle.lloyd(w, 32, 25)
    tr = res["trace"]
    assert np.all(np.diff(tr, axis=-1) <= 1e-18)                     # non-increasing
    assert np.all(tr[..., -1] <= tr[..., 0])
    a = np.abs(oracle.bf16_to_f64(w)).reshape(48, 16, 32)
    q = (res["codes"] & 7).reshape(48, 16, 32)
    s = (res["codes"] >> 3).reshape(48, 16, 32)
    assert np.array_equal(s, (oracle.bf16_to_f64(w) < 0).reshape(48, 16, 32))
    _check_kmeans_properties(a, q, res["levels"])
    lv = res["levels"]
    assert np.all(np.diff(lv, axis=-1) >= 0)                          # sorted
    assert np.all(lv[..., 0] >= 0) and np.all(lv[..., -1] <= a.max(-1) + 0)
    # reported final MSE equals the MSE recomputed from codes and levels
    rec = np.take_along_axis(lv, q, axis=-1)
    assert np.allclose(((a - rec) ** 2).mean(-1), tr[..., -1], rtol=1e-12, atol=0)
    # the candidate really is the argmin: forcing any other candidate never does better
    for other in (0, 55, 104, 110):
        fc = np.full((48, 16), other, np.int32)
        r2 = oracle.lloyd(w, 32, 0, force_cand=fc)
        assert np.all(r2["trace"][..., 0] >= tr[..., 0])


def test_ordering_claims_on_synthetic_laplace():
    """[G32] §1.4: warm start never loses to the parametric solution alone; smaller groups
    give a smaller error (g32 < g64 < g128). Values are parity unpinned."""
    w = workloads.laplace_rowscaled_weight(64, 1024)
    warm = oracle.lloyd(w, 32, 25)
    assert warm["trace"][..., -1].mean() < warm["trace"][..., 0].mean()
    cold = oracle.lloyd(w, 32, 25, cold_start=True)
    assert warm["trace"][..., -1].mean() < cold["trace"][..., -1].mean()
    mse = {g: oracle.lloyd(w, g, 25)["trace"][..., -1].mean() for g in (32, 64, 128)}
    assert mse[32] < mse[64] < mse[128]


# --- LUT16 k-means ---------------------------------------------------------------------------

def test_kmeans_sixteen_distinct_values_repeated_four_times():
    g = np.random.default_rng(9)
    vals = workloads.f64_to_bf16_bits(np.sort(g.standard_normal(16)) * 0.01)
    assert len(np.unique(vals)) == 16
    w = np.repeat(vals, 4)
    w = w[g.permutation(64)].reshape(1, 64)
    res = oracle.kmeans_lut16(w, 64, 25, threads=1)
    cen = oracle.fp16_to_f64(res["lut"][0, 0])
    wv = oracle.bf16_to_f64(w[0])
    assert np.array_equal(cen[res["codes"][0]], oracle.fp16_to_f64(oracle.f64_to_fp16(wv)))
    assert np.array_equal(np.sort(cen), cen)


def test_kmeans_init_reading_and_properties():
    w = workloads.lut16_weight(16, 256, heavy_tail=True)
    r0 = oracle.kmeans_lut16(w, 64, 0)
    v = oracle.bf16_to_f64(w).reshape(16, 4, 64)
    init = np.sort(v, axis=-1)[..., 2::4]                               # (4i+2)-th smallest
    assert np.array_equal(oracle.fp16_to_f64(r0["lut"]), oracle.fp16_to_f64(oracle.f64_to_fp16(init)))
    res = oracle.kmeans_lut16(w, 64, 25)
    tr = res["trace"]
    assert np.all(np.diff(tr[..., :-1], axis=-1) <= 1e-18)               # Lloyd rounds
    cen = oracle.fp16_to_f64(res["lut"])
    _check_kmeans_properties(v, res["codes"].reshape(16, 4, 64), cen)
    assert tr[..., -1].mean() < tr[..., 0].mean()
    wd = oracle.fp16_to_f64(oracle.dequant(oracle.LUT16, oracle.pack(res["codes"]), res["lut"], 64))
    err = ((wd.reshape(16, 4, 64) - v) ** 2).mean(-1)
    assert np.allclose(err, tr[..., -1], rtol=1e-12)


# ---------------------------------------------------------------------------------------
# Brute force of the candidate search ([G32] §1.2 grid, §1.3 step 1), written apart from the
# oracle: the grid from the page's printed lists, the transforms with Python's own pow and
# tanh, every inverse level by scipy's Brent root finder on f(L) = q/7 * fmax (no closed
# forms), round half to even, and all 112 MSEs compared one by one with the oracle forced to
# each candidate.
# ---------------------------------------------------------------------------------------

def _page_grid():
    gold = _golden()
    lo, hi = (math.log10(v) for v in gold["rational_b_rel_endpoints"])
    grid = []
    for r in range(15):
        for beta in gold["rational_beta"]:
            grid.append((0, 10 ** (lo + (hi - lo) * r / 14), beta))
    grid += [(1, br, 1.0) for br in gold["tanh_b_rel"]]
    return grid


def _brute_mses(a):
    from scipy.optimize import brentq
    gmax = max(a)
    out = []
    for fam, b_rel, beta in _page_grid():
        b = b_rel * gmax
        if fam == 0:
            f = lambda v, b=b, beta=beta: v / (b + v ** beta)
        else:
            f = lambda v, b=b: math.tanh(v / b)
        fmax = f(gmax)
        levels = [0.0] + [brentq(lambda v, t=q / 7 * fmax: f(v) - t, 0.0, gmax, xtol=1e-300,
                                 rtol=8.9e-16, maxiter=400) for q in range(1, 7)] + [gmax]
        se = 0.0
        for v in a:
            q = min(max(int(np.rint(7 * f(v) / fmax)), 0), 7)      # rint: half to even
            se += (v - levels[q]) ** 2
        out.append(se / len(a))
    return np.array(out)


def _groups_for_brute_force():
    rng = np.random.default_rng(11)
    groups = [workloads.f64_to_bf16_bits(rng.laplace(0, 0.015, 32) * s) for s in (0.5, 1.0, 2.0)]
    g = workloads.f64_to_bf16_bits(rng.normal(0, 0.02, 32))
    g[rng.integers(32)] = workloads.f64_to_bf16_bits(np.array([0.4]))[0]      # one outlier x20
    groups.append(g)
    groups.append(workloads.f64_to_bf16_bits(rng.laplace(0, 1.0, 8)))          # a tiny group
    return groups


@pytest.mark.parametrize("gi", range(5))
def test_candidate_search_matches_brute_force(gi):
    g = _groups_for_brute_force()[gi]
    a = [abs(float(v)) for v in oracle.bf16_to_f64(g)]
    brute = _brute_mses(a)
    size = len(a)
    w = g.reshape(1, size)
    ref = oracle.lloyd(w, size, 0)
    # every candidate's MSE, the oracle forced to it
    for c in range(112):
        forced = oracle.lloyd(w, size, 0, force_cand=np.array([c], np.int32))
        assert forced["trace"][0, 0, 0] == pytest.approx(brute[c], rel=1e-9, abs=1e-30), c
    order = np.argsort(brute, kind="stable")
    best, second = brute[order[0]], brute[order[1]]
    assert second > best * (1 + 1e-6)          # a clear winner: no near-tie in these groups
    assert ref["cand"][0, 0] == order[0]
    assert ref["trace"][0, 0, 0] == pytest.approx(best, rel=1e-12)
    assert ref["cand_gap"][0, 0] == pytest.approx(second - best, rel=1e-6)


def test_candidate_search_exact_tie_takes_lowest_index():
    """Magnitudes only 0 and gmax (and one just below gmax, which every candidate's concave
    transform sends to the top level): every candidate reconstructs them with its exact end
    levels, so all 112 MSEs are the same number and the lowest index, 0, must win."""
    vals = np.array([0.0, 1.5, -1.5, 0.0, 1.5, -1.4921875] * 5 + [1.5, -0.0])
    g = workloads.f64_to_bf16_bits(vals)
    a = [abs(float(v)) for v in oracle.bf16_to_f64(g)]
    brute = _brute_mses(a)
    assert np.all(brute == brute[0]) and brute[0] > 0
    ref = oracle.lloyd(g.reshape(1, 32), 32, 0)
    assert ref["cand"][0, 0] == 0 and ref["params"][0, 0] == 0
    assert ref["trace"][0, 0, 0] == brute[0]
