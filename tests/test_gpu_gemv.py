"""GPU parity of the W4A16 GEMV against the oracle's fp64 product of its own
reconstruction: |y - y_ref| <= 2e-3 * sum_c |Wdeq[r, c]| |x[b, c]| per output element
(the stated tolerance), plus exact special cases."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _util import bits, f32, matmul_tolerance, to_dev, to_dev_bits

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _dyadic_weight(wq, n, k, group, seed):
    w_bits = workloads.gaussian_outlier_weight(n, k, workloads.DYADIC_1, seed)
    s, c = oracle.dyadic_quantize(w_bits, group)
    packed = oracle.pack(c)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, group, n, k, to_dev(packed), to_dev_bits(s))
    return pw, packed, s


def _check(y, y_ref, bound, rows=None):
    y = f32(y)
    if rows is not None:
        y = y[:, rows]
    err = np.abs(y - y_ref)
    ok = err <= matmul_tolerance(y_ref, bound, TOL)
    assert ok.all(), f"max err/bound {np.max(err / np.maximum(bound, 1e-300)):.3g}"
    return float(np.max(err / np.maximum(bound, 1e-300)))


@pytest.mark.parametrize("batch", [1, 2, 4, 8, 9, 16])
@pytest.mark.parametrize("n,k,group", [(8, 256, 64), (13, 320, 64), (37, 1088, 64),
                                       (300, 2048, 64), (24, 2144, 32), (5, 32, 32)])
def test_gemv_dyadic_matches_oracle(wq, n, k, group, batch):
    pw, packed, s = _dyadic_weight(wq, n, k, group, n + k + group)
    x_bits = workloads.activations(batch, k, workloads.DECODE_SWEEP, n)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, group, x_bits)
    _check(y, y_ref, bound)


@pytest.mark.parametrize("group", [64, 32])
def test_gemv_one_hot_reproduces_dequantised_column_exactly(wq, group):
    n, k = 40, 512
    pw, packed, s = _dyadic_weight(wq, n, k, group, 5)
    wd = oracle.dequant(oracle.DYADIC4, packed, s, group)
    cols = [0, 1, 7, 31, 32, 63, 64, 255, 256, 511]
    x = np.zeros((len(cols), k))
    for i, c in enumerate(cols):
        x[i, c] = 1.0
    y = wq.gemv(pw, to_dev_bits(workloads.f64_to_bf16_bits(x)))
    got = f32(y)
    for i, c in enumerate(cols):
        assert np.array_equal(got[i], oracle.bf16_to_f64(wd[:, c]))


def test_gemv_all_codes_eight_is_exact_zero_and_unit_group_sums(wq):
    n, k = 24, 384
    packed = np.full((n, k // 2), 0x88, np.uint8)
    s = workloads.f64_to_bf16_bits(np.random.default_rng(1).uniform(0.01, 3, (n, k // 64)))
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(s))
    x = workloads.activations(16, k, workloads.DECODE_SWEEP, 3)
    assert np.all(f32(wq.gemv(pw, to_dev_bits(x))) == 0.0)
    g = np.random.default_rng(2)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    scale = np.full((n, k // 64), 0x3E00, np.uint16)          # step 1/64: sums exact in bf16
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(oracle.pack(codes)), to_dev_bits(scale))
    xs = np.zeros((6, k))
    for grp in range(6):
        xs[grp, grp * 64:(grp + 1) * 64] = 1.0
    y = f32(wq.gemv(pw, to_dev_bits(workloads.f64_to_bf16_bits(xs))))
    for grp in range(6):
        expect = (codes[:, grp * 64:(grp + 1) * 64].astype(np.int64) - 8).sum(1) / 64.0
        assert np.array_equal(y[grp], expect)


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_grouped_gemv_equals_single_calls(wq, batch):
    shapes = [(2048, 2048), (256, 2048), (300, 1088), (5632, 2048), (2048, 5632)]
    ws, xs, xbits, packs = [], [], [], []
    for i, (n, k) in enumerate(shapes):
        pw, packed, s = _dyadic_weight(wq, n, k, 64, 100 + i)
        ws.append(pw)
        packs.append((packed, s))
        xb = workloads.activations(batch, k, workloads.DECODE_SWEEP, 100 + i)
        xbits.append(xb)
        xs.append(to_dev_bits(xb))
    ys = wq.gemv_grouped(ws, xs)
    # the grouped launch may split K differently from a single launch (fp32 summation
    # order): both must meet the tolerance on the same sampled rows
    rng = np.random.default_rng(3)
    for (packed, s), xb, y, w, x in zip(packs, xbits, ys, ws, xs):
        rows = rng.choice(packed.shape[0], 64, replace=False)
        y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, xb, rows=rows)
        _check(y, y_ref, bound, rows)
        _check(wq.gemv(w, x), y_ref, bound, rows)


def test_decode_sweep_layer_full_size_sampled(wq):
    """One layer of the decode-sweep stack at full size, quantised by the oracle, in one
    grouped launch; sampled rows of every projection against the oracle, at batch 1 and 16."""
    mats = [m for m in workloads.sweep_matrices(1)]
    ws, pk = [], []
    for layer, name, n, k, idx in mats:
        # quantised by the oracle on the host: the GEMV's inputs never come from the GPU path
        w_bits = workloads.gaussian_outlier_weight(n, k, workloads.DECODE_SWEEP, idx)
        s, c = oracle.dyadic_quantize(w_bits, 64)
        packed = oracle.pack(c)
        ws.append(wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(s)))
        pk.append((packed, s))
    rng = np.random.default_rng(4)
    for batch in (1, 16):
        xb = [workloads.activations(batch, k, workloads.DECODE_SWEEP, idx) for _, _, _, k, idx in mats]
        ys = wq.gemv_grouped(ws, [to_dev_bits(x) for x in xb])
        for (packed, s), x, y in zip(pk, xb, ys):
            rows = rng.choice(packed.shape[0], 48, replace=False)
            y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, x, rows=rows)
            _check(y, y_ref, bound, rows)


def test_gemv_host_input_path(wq):
    pw, packed, s = _dyadic_weight(wq, 64, 512, 64, 9)
    x_bits = workloads.activations(2, 512, workloads.DECODE_SWEEP, 9)
    xc = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    y = wq.gemv(pw, xc)
    assert y.device.type == "cpu"
    assert torch.equal(y, wq.gemv(pw, xc.cuda()).cpu())


def test_gemv_lut16_matches_oracle(wq):
    n, k = 96, 1024
    g = np.random.default_rng(11)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    lut = oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(lut, torch.float16))
    for batch in (1, 8, 16):
        x_bits = workloads.activations(batch, k, workloads.LUT16, batch)
        y = wq.gemv(pw, to_dev_bits(x_bits))
        y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, x_bits)
        _check(y, y_ref, bound)
    # one-hot: the fp16 centroid rounded once to bf16
    x = np.zeros((3, k))
    x[0, 0] = x[1, 65] = x[2, 1023] = 1.0
    y = f32(wq.gemv(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
    wd = oracle.fp16_to_f64(oracle.dequant(oracle.LUT16, packed, lut, 64))
    for i, c in enumerate([0, 65, 1023]):
        assert np.array_equal(y[i], oracle.bf16_to_f64(oracle.f64_to_bf16(wd[:, c])))


SCALE_REGIMES = [0x0001, 0x0031, 0x007F, 0x0080, 0x00FF, 0x3D4C, 0x3F80, 0x3FFF, 0x7C00, 0x7D80,
                 0x7E55, 0x7F7F, 0x0000]


@pytest.mark.parametrize("group", [64, 32])
def test_gemv_one_hot_every_scale_regime(wq, group):
    """Every scale regime (subnormal, smallest normal, typical, 2^121, >= 2^124 where the
    fp32 path takes over, the largest bf16, zero): one-hot activations reproduce the
    dequantised column exactly, so the in-register reconstruction is bit-exact."""
    n, k = 16 * len(SCALE_REGIMES), 256
    g = np.random.default_rng(13)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    scale = np.repeat(np.array(SCALE_REGIMES, np.uint16), 16)[:, None].repeat(k // group, 1)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, group, n, k, to_dev(packed), to_dev_bits(scale))
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.DYADIC4, packed, scale, group))
    cols = np.arange(0, k, 17)
    for lo in range(0, len(cols), 16):
        cc = cols[lo:lo + 16]
        x = np.zeros((len(cc), k))
        x[np.arange(len(cc)), cc] = 1.0
        y = f32(wq.gemv(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
        assert np.array_equal(y, wd[:, cc].T)


@pytest.mark.parametrize("batch", [1, 5, 16])
def test_gemv_plan_matches_grouped_call_and_reads_current_inputs(wq, batch):
    """A prepared plan launches the kernel the grouped call would (bit-identical output),
    and reads whatever its bound x buffers hold when it runs."""
    shapes = [(2048, 2048), (300, 1088), (5632, 2048), (2048, 5632)]
    ws, packs, xs, ys = [], [], [], []
    for i, (n, k) in enumerate(shapes):
        pw, packed, s = _dyadic_weight(wq, n, k, 64, 200 + i)
        ws.append(pw)
        packs.append((packed, s))
        xs.append(to_dev_bits(workloads.activations(batch, k, workloads.DECODE_SWEEP, 300 + i)))
        ys.append(torch.empty((batch, n), dtype=torch.bfloat16, device="cuda"))
    plan = wq.GroupedGemv(ws, xs, ys)
    plan()
    ref = wq.gemv_grouped(ws, xs)
    for y, r in zip(ys, ref):
        assert torch.equal(y, r)
    # new activations written into the bound buffers: the next launch sees them
    rng = np.random.default_rng(5)
    new_bits = []
    for x, (n, k) in zip(xs, shapes):
        nb = workloads.activations(batch, k, workloads.DECODE_SWEEP, 400 + n)
        x.copy_(to_dev_bits(nb))
        new_bits.append(nb)
    plan()
    torch.cuda.synchronize()
    for (packed, s), nb, y in zip(packs, new_bits, ys):
        rows = rng.choice(packed.shape[0], 48, replace=False)
        y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, s, 64, nb, rows=rows)
        _check(y, y_ref, bound, rows)
    plan.close()
    plan.close()                                         # idempotent


def test_gemv_plan_replays_in_a_cuda_graph(wq):
    pw, packed, s = _dyadic_weight(wq, 1024, 2048, 64, 31)
    x = to_dev_bits(workloads.activations(1, 2048, workloads.DECODE_SWEEP, 31))
    y = torch.empty((1, 1024), dtype=torch.bfloat16, device="cuda")
    plan = wq.GroupedGemv([pw], [x], [y])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan()
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, wq.gemv(pw, x))


@pytest.mark.parametrize("graph", [False, True])
def test_gemv_plan_overlap_keeps_stream_order_for_data(wq, graph):
    """A plan with overlap enabled (programmatic dependent launch) may start beside the
    kernel before it, but must read its activations only after that kernel's writes: a torch
    kernel rewrites x right before each launch of plan A, plan B reads A's output (a layer
    feeding the next), and A's launch follows B's. Every output must be bit-identical to
    the same chain in plain stream order, eagerly and captured in a CUDA graph; the large
    first problem (a cluster launch) and the small ones (plain launches) take both paths."""
    shapes_a = [(5632, 2048), (2048, 2048)]
    wa = [_dyadic_weight(wq, n, k, 64, 500 + i)[0] for i, (n, k) in enumerate(shapes_a)]
    wb, _, _ = _dyadic_weight(wq, 1024, 5632, 64, 510)
    big = wq.PackedWeight(*_lut_args(wq, 8192, 4096, 511))
    src = [to_dev_bits(workloads.activations(1, k, workloads.DECODE_SWEEP, 600 + i)).float()
           for i, (_, k) in enumerate(shapes_a)]
    src_big = to_dev_bits(workloads.activations(1, 4096, workloads.DECODE_SWEEP, 610)).float()

    def chain(overlap, steps=6):
        xa = [torch.empty((1, k), dtype=torch.bfloat16, device="cuda") for _, k in shapes_a]
        ya = [torch.empty((1, n), dtype=torch.bfloat16, device="cuda") for n, _ in shapes_a]
        yb = torch.empty((1, 1024), dtype=torch.bfloat16, device="cuda")
        xl = torch.empty((1, 4096), dtype=torch.bfloat16, device="cuda")
        yl = torch.empty((1, 8192), dtype=torch.bfloat16, device="cuda")
        plan_a = wq.GroupedGemv(wa, xa, ya, overlap=overlap)
        plan_b = wq.GroupedGemv([wb], [ya[0]], [yb], overlap=overlap)
        plan_l = wq.GroupedGemv([big], [xl], [yl], overlap=overlap)
        outs = []

        def run():
            outs.clear()
            for t in range(steps):
                for x, s0 in zip(xa, src):
                    x.copy_(s0 * ((t + 1) / 4))              # a conversion kernel writes x
                plan_a()
                plan_b()
                xl.copy_(src_big * (t + 1))
                plan_l()
                outs.append(torch.cat([ya[0][0], ya[1][0], yb[0], yl[0]]).clone())

        if graph:
            run()                                          # warm up outside the capture
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run()
            g.replay()
        else:
            run()
        torch.cuda.synchronize()
        res = torch.stack(outs)
        for p in (plan_a, plan_b, plan_l):
            p.close()
        return res

    plain = chain(False)
    over = chain(True)
    assert torch.equal(over, plain)
    # and the plain chain is the product it should be (spot check of the last step)
    assert torch.isfinite(plain.float()).all()


def _lut_args(wq, n, k, seed):
    g = np.random.default_rng(seed)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    lut = oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    return wq.FMT_LUT16, 64, n, k, to_dev(oracle.pack(codes)), to_dev_bits(lut, torch.float16)


def _lloyd_weight(wq, n, k, seed, signed_levels=False):
    """Random LLOYD8S weights: codes 0..15 (level index | sign << 3) and 8 fp32 levels per
    group of 32 (sorted magnitudes, as the producer makes them; optionally of either sign,
    which the format allows)."""
    g = np.random.default_rng(seed)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    levels = np.sort(np.abs(g.standard_normal((n, k // 32, 8))) * 0.02, -1).astype(np.float32)
    if signed_levels:
        levels *= np.where(g.random(levels.shape) < 0.5, -1.0, 1.0).astype(np.float32)
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, n, k, to_dev(packed), torch.from_numpy(levels).cuda())
    return pw, packed, levels


@pytest.mark.parametrize("batch", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("n,k", [(16, 32), (37, 1088), (300, 2048), (24, 2144)])
def test_gemv_lloyd8s_matches_oracle(wq, n, k, batch):
    """The fused LLOYD8S consumer ("int4-g32+warm" §5.2: 8-level codebook plus sign bit held
    in registers) against the oracle's product of its bf16(+/-level) reconstruction."""
    pw, packed, levels = _lloyd_weight(wq, n, k, n + k + batch)
    x_bits = workloads.activations(batch, k, workloads.DECODE_SWEEP, n + batch)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    y_ref, bound = oracle.matmul_rows(oracle.LLOYD8S, packed, levels, 32, x_bits)
    _check(y, y_ref, bound)


def test_gemv_lloyd8s_one_hot_reproduces_dequant_exactly(wq):
    n, k = 48, 256
    pw, packed, levels = _lloyd_weight(wq, n, k, 7, signed_levels=True)
    wd = oracle.bf16_to_f64(oracle.dequant(oracle.LLOYD8S, packed, levels, 32))
    cols = np.arange(0, k, 5)
    for lo in range(0, len(cols), 16):
        cc = cols[lo:lo + 16]
        x = np.zeros((len(cc), k))
        x[np.arange(len(cc)), cc] = 1.0
        y = f32(wq.gemv(pw, to_dev_bits(workloads.f64_to_bf16_bits(x))))
        assert np.array_equal(y, wd[:, cc].T)


def test_gemv_lloyd8s_on_lloyd_quantised_weights(wq):
    """Codes and levels of the g32 Lloyd producer (the oracle's, on the host) on rows of the
    Lloyd workload, consumed by the fused GEMV and by the oracle (sampled rows)."""
    w_bits = workloads.laplace_rowscaled_weight(128, 2048, index=3)
    ref = oracle.lloyd(w_bits, 32, 25)
    packed = oracle.pack(ref["codes"])
    levels = ref["levels"].astype(np.float32)
    pw = wq.PackedWeight(wq.FMT_LLOYD8S, 32, 128, 2048, to_dev(packed), torch.from_numpy(levels).cuda())
    rng = np.random.default_rng(8)
    rows = rng.choice(128, 64, replace=False)
    for batch in (1, 16):
        x_bits = workloads.activations(batch, 2048, workloads.DECODE_SWEEP, 40 + batch)
        y = wq.gemv(pw, to_dev_bits(x_bits))
        y_ref, bound = oracle.matmul_rows(oracle.LLOYD8S, packed, levels, 32, x_bits, rows=rows)
        _check(y, y_ref, bound, rows)


@pytest.mark.parametrize("n,k", [(4096, 4096), (4100, 4160)])
@pytest.mark.parametrize("batch", [1, 3, 16])
def test_gemv_cluster_split_k_matches_oracle(wq, n, k, batch):
    """Single launches of >= 16 M weights with too few rows to fill the GPU split K across a
    thread-block cluster (partial sums reduced through distributed shared memory); ragged
    rows and a ragged last step included. Sampled rows against the oracle."""
    g = np.random.default_rng(n + k + batch)
    codes = g.integers(0, 16, (n, k), dtype=np.uint8)
    scale = workloads.f64_to_bf16_bits(g.uniform(0.005, 0.05, (n, k // 64)))
    packed = oracle.pack(codes)
    pw = wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(scale))
    x_bits = workloads.activations(batch, k, workloads.DECODE_SWEEP, batch)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    rows = np.concatenate([g.choice(n, 96, replace=False), np.arange(n - 8, n)])
    y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, scale, 64, x_bits, rows=rows)
    _check(y, y_ref, bound, rows)


@pytest.mark.parametrize("batch", [1, 4, 16])
def test_full_decode_sweep_in_the_benchmarked_launch(wq, batch):
    """All 168 matrices of the decode-sweep stack (1,056,964,608 weights) in the one grouped,
    prepared launch the benchmark times (the full-K kernel variant that only a launch of this
    size selects). Seeded codes and scales from the host; 6 sampled rows of every matrix,
    plus its last row, against the oracle."""
    mats = workloads.sweep_matrices()
    g = np.random.default_rng(77 + batch)
    ws, host, xs_bits = [], [], []
    for layer, name, n, k, idx in mats:
        packed = g.integers(0, 256, (n, k // 2), dtype=np.uint8)
        scale = workloads.f64_to_bf16_bits(g.uniform(0.002, 0.08, (n, k // 64)))
        ws.append(wq.PackedWeight(wq.FMT_DYADIC4, 64, n, k, to_dev(packed), to_dev_bits(scale)))
        host.append((packed, scale))
        xs_bits.append(workloads.activations(batch, k, workloads.DECODE_SWEEP, idx))
    xs = [to_dev_bits(x) for x in xs_bits]
    ys = [torch.empty((batch, n), dtype=torch.bfloat16, device="cuda") for _, _, n, _, _ in mats]
    plan = wq.GroupedGemv(ws, xs, ys)
    plan()
    torch.cuda.synchronize()
    plan.close()
    assert wq.device_error() == 0
    for (packed, scale), x, y in zip(host, xs_bits, ys):
        n = packed.shape[0]
        rows = np.concatenate([g.choice(n, 6, replace=False), [n - 1]])
        y_ref, bound = oracle.matmul_rows(oracle.DYADIC4, packed, scale, 64, x, rows=rows)
        _check(y, y_ref, bound, rows)


@pytest.mark.parametrize("batch", [1, 8, 16])
def test_lut16_full_size_in_the_benchmarked_launch(wq, batch):
    """The 16-centroid LUT workload at full size (8192 x 28672: K split across a cluster of
    CTAs, the launch the benchmark times), seeded codes and sorted fp16 centroid tables from
    the host; 64 sampled rows, plus the last row, against the oracle."""
    n, k = workloads.LUT16_SHAPE
    g = np.random.default_rng(91 + batch)
    packed = g.integers(0, 256, (n, k // 2), dtype=np.uint8)
    lut = oracle.f64_to_fp16(np.sort(g.standard_normal((n, k // 64, 16)), -1) * 0.01)
    pw = wq.PackedWeight(wq.FMT_LUT16, 64, n, k, to_dev(packed), to_dev_bits(lut, torch.float16))
    x_bits = workloads.activations(batch, k, workloads.LUT16, batch)
    y = wq.gemv(pw, to_dev_bits(x_bits))
    torch.cuda.synchronize()
    assert wq.device_error() == 0
    rows = np.concatenate([np.sort(g.choice(n, 64, replace=False)), [n - 1]])
    y_ref, bound = oracle.matmul_rows(oracle.LUT16, packed, lut, 64, x_bits, rows=rows)
    _check(y, y_ref, bound, rows)
