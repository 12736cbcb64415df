"""fp64 CPU oracle for group-wise 4-bit weight coding and W4A16 matmul.

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package. The CUDA library never
does, and this package never imports the CUDA library: the two share no code.

The arithmetic lives in ``wq_oracle.c`` (plain C, double precision), compiled with gcc
into ``_liboracle.so`` next to this file. This module only marshals numpy arrays and
splits row ranges across host threads (ctypes releases the GIL during each call).

Sources, cited by key in the C file and below:
  [DG]  "MiniCPM5-1B 验证: 6× 压缩, ppl 反超 fp, 1.2GB 显存, 50ms Triton 推理"
  [KM]  "K-Means量化技术：突破LLM低比特部署瓶颈"
  [G32] "int4-g32+warm 裸量化：原理与实验报告"
  [BX]  "同一个 1B 模型，我上了三种压缩方案：无损的、4bit 的、还有没跑通的" (BF16X)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wq_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")

DYADIC4, LLOYD8S, LUT16 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no GPU involved). Returns the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib_lock = threading.Lock()


def _L():
    global _lib
    if _lib is not None:
        return _lib
    with _lib_lock:                 # the row-parallel callers arrive from several threads
        return _load()


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        sig = {
            "orc_bf16_to_double_array": [vp, i64, vp],
            "orc_double_to_bf16_array": [vp, i64, vp],
            "orc_fp16_to_double_array": [vp, i64, vp],
            "orc_double_to_fp16_array": [vp, i64, vp],
            "orc_dyadic_quantize": [vp, i64, i64, i32, i64, i64, vp, vp],
            "orc_dyadic_dequant": [vp, vp, i64, i64, i32, i64, i64, vp],
            "orc_fake_quant_ste": [vp, vp, i64, i64, i32, i64, i64, vp, vp],
            "orc_gumbel_st_backward": [vp, vp, vp, i64, i64, i32, ctypes.c_double, i64, i64, vp, vp,
                                       vp, vp],
            "orc_pack": [vp, i64, i64, i64, i64, vp],
            "orc_unpack": [vp, i64, i64, i64, i64, vp],
            "orc_dequant": [i32, vp, vp, i64, i64, i32, i64, i64, vp],
            "orc_matmul_rows": [i32, vp, vp, i64, i32, vp, i64, vp, i64, i64, i64, vp, vp],
            "orc_lloyd": [vp, i64, i64, i32, i32, vp, vp, i64, i64, vp, vp, vp, vp, vp, vp, vp],
            "orc_kmeans_lut16": [vp, i64, i64, i32, i32, i64, i64, vp, vp, vp, vp],
            "orc_lloyd_candidate": [i32, vp, vp, vp],
            "orc_lloyd_params_byte": [i32],
            "orc_lloyd_num_candidates": [],
            "orc_bf16x_encode": [vp, i64, i64, vp, vp, vp, vp, i64, vp],
            "orc_bf16x_decode": [vp, vp, vp, vp, i64, i64, i64, vp],
            "orc_wf_analyze": [vp, i64, i64, ctypes.c_double, i64, i64, vp, vp, vp],
            "orc_wf_offsets": [vp, i64, vp],
            "orc_wf_pack": [vp, i64, i64, vp, vp, vp, i64, i64, vp],
            "orc_wf_dequant": [vp, vp, vp, vp, i64, i64, i64, i64, vp],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        lib.orc_lloyd_inverse.argtypes = [i32, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_double]
        lib.orc_lloyd_inverse.restype = ctypes.c_double
        lib.orc_bf16x_superblocks.argtypes = [i64, i64]
        lib.orc_bf16x_superblocks.restype = i64
        lib.orc_storage_bytes.argtypes = [i32, ctypes.c_double, i32]
        lib.orc_storage_bytes.restype = ctypes.c_double
        lib.orc_storage_lloyd_codebook_bytes.argtypes = [ctypes.c_double, i32]
        lib.orc_storage_lloyd_codebook_bytes.restype = ctypes.c_double
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _rows_parallel(n: int, fn, threads: int | None):
    """Run fn(r0, r1) over [0, n) split into contiguous chunks on `threads` threads."""
    threads = threads or default_threads()
    threads = max(1, min(threads, n))
    bounds = np.linspace(0, n, threads + 1).astype(np.int64)
    if threads == 1:
        rcs = [fn(0, n)]
    else:
        with ThreadPoolExecutor(threads) as ex:
            rcs = list(ex.map(lambda i: fn(int(bounds[i]), int(bounds[i + 1])), range(threads)))
    for rc in rcs:
        if rc != 0:
            raise ValueError(f"oracle call failed with code {rc}")


# --- number formats -------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float64)
    _L().orc_bf16_to_double_array(_p(bits), bits.size, _p(out))
    return out


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _L().orc_double_to_bf16_array(_p(v), v.size, _p(out))
    return out


def fp16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, np.float64)
    _L().orc_fp16_to_double_array(_p(bits), bits.size, _p(out))
    return out


def f64_to_fp16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    _L().orc_double_to_fp16_array(_p(v), v.size, _p(out))
    return out


# --- dyadic code, pack, dequant ----------------------------------------------------------

def dyadic_quantize(w_bits: np.ndarray, group: int = 64, threads: int | None = None):
    """[DG] §2.1-2.3: per-group bf16 absmax scale and nearest-code index (lowest on tie).
    Returns (scale_bits [n, k/group] uint16, codes [n, k] uint8)."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    scale = np.empty((n, k // group), np.uint16)
    codes = np.empty((n, k), np.uint8)
    _rows_parallel(n, lambda r0, r1: _L().orc_dyadic_quantize(_p(w), n, k, group, r0, r1,
                                                              _p(scale), _p(codes)), threads)
    return scale, codes


def fake_quant_ste(z: np.ndarray, scale_bits: np.ndarray, group: int = 64,
                   threads: int | None = None):
    """[DG] §2.3 STE forward on an fp32 latent z: (q fp32 [n, k], codes uint8 [n, k]) with
    codes the nearest of the 16 dyadic code values (lowest index on a tie) and q that value."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    scale = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    n, k = z.shape
    q = np.empty((n, k), np.float32)
    codes = np.empty((n, k), np.uint8)
    _rows_parallel(n, lambda r0, r1: _L().orc_fake_quant_ste(_p(z), _p(scale), n, k, group, r0, r1,
                                                             _p(q), _p(codes)), threads)
    return q, codes


def gumbel_st_backward(z: np.ndarray, scale_bits: np.ndarray, gq: np.ndarray, tau: float,
                       group: int = 64, threads: int | None = None):
    """[DG] §2.3 Gumbel-ST (q = hard + (soft - soft.detach()), soft = softmax(-dist/tau).codes)
    backward for the upstream gradient gq: (gz fp32 [n, k], gscale fp64 [n, k/group], gz_mag,
    gscale_mag), the *_mag arrays being the same sums over absolute values of every term."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    gq = np.ascontiguousarray(gq, dtype=np.float32)
    scale = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    n, k = z.shape
    gz = np.empty((n, k), np.float32)
    gz_mag = np.empty((n, k), np.float64)
    gs = np.empty((n, k // group), np.float64)
    gs_mag = np.empty((n, k // group), np.float64)
    _rows_parallel(n, lambda r0, r1: _L().orc_gumbel_st_backward(
        _p(z), _p(scale), _p(gq), n, k, group, float(tau), r0, r1, _p(gz), _p(gs), _p(gz_mag),
        _p(gs_mag)), threads)
    return gz, gs, gz_mag, gs_mag


def dyadic_dequant(codes: np.ndarray, scale_bits: np.ndarray, group: int = 64,
                   threads: int | None = None) -> np.ndarray:
    """[DG] §2.2: bf16(step * (idx - 8)), step = scale / 8, from unpacked codes."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scale = np.ascontiguousarray(scale_bits, dtype=np.uint16)
    n, k = codes.shape
    out = np.empty((n, k), np.uint16)
    _rows_parallel(n, lambda r0, r1: _L().orc_dyadic_dequant(_p(codes), _p(scale), n, k, group,
                                                             r0, r1, _p(out)), threads)
    return out


def pack(codes: np.ndarray, threads: int | None = None) -> np.ndarray:
    """[DG] §2.5: byte j of a row = code[2j] | code[2j+1] << 4."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    n, k = codes.shape
    out = np.empty((n, k // 2), np.uint8)
    _rows_parallel(n, lambda r0, r1: _L().orc_pack(_p(codes), n, k, r0, r1, _p(out)), threads)
    return out


def unpack(packed: np.ndarray, threads: int | None = None) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n, kh = packed.shape
    k = 2 * kh
    out = np.empty((n, k), np.uint8)
    _rows_parallel(n, lambda r0, r1: _L().orc_unpack(_p(packed), n, k, r0, r1, _p(out)), threads)
    return out


def dequant(fmt: int, packed: np.ndarray, aux: np.ndarray, group: int,
            threads: int | None = None) -> np.ndarray:
    """Dequantised weights as 16-bit patterns (bf16; fp16 centroids for LUT16)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    aux = np.ascontiguousarray(aux)
    n, kh = packed.shape
    k = 2 * kh
    out = np.empty((n, k), np.uint16)
    _rows_parallel(n, lambda r0, r1: _L().orc_dequant(fmt, _p(packed), _p(aux), n, k, group,
                                                      r0, r1, _p(out)), threads)
    return out


def matmul_rows(fmt: int, packed: np.ndarray, aux: np.ndarray, group: int, x_bits: np.ndarray,
                rows: np.ndarray | None = None, threads: int | None = None):
    """y[b, j] = sum_c Wdeq[rows[j], c] * x[b, c] in double, and the per-element error scale
    bound[b, j] = sum_c |Wdeq[rows[j], c]| * |x[b, c]|. x is bf16 bits [m, k]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    aux = np.ascontiguousarray(aux)
    x = np.ascontiguousarray(np.atleast_2d(x_bits), dtype=np.uint16)
    n, kh = packed.shape
    k = 2 * kh
    m = x.shape[0]
    assert x.shape[1] == k
    rows = np.arange(n, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    nr = rows.size
    y = np.empty((m, nr), np.float64)
    bound = np.empty((m, nr), np.float64)
    _rows_parallel(nr, lambda j0, j1: _L().orc_matmul_rows(fmt, _p(packed), _p(aux), k, group,
                                                           _p(x), m, _p(rows), nr, j0, j1,
                                                           _p(y), _p(bound)), threads)
    return y, bound


# --- Lloyd g32 and LUT16 k-means producers ---------------------------------------------------

def lloyd_candidate(c: int):
    fam, brel, beta = ctypes.c_int32(), ctypes.c_double(), ctypes.c_double()
    if _L().orc_lloyd_candidate(c, ctypes.byref(fam), ctypes.byref(brel), ctypes.byref(beta)) != 0:
        raise ValueError(c)
    return fam.value, brel.value, beta.value


def lloyd_params_byte(c: int) -> int:
    return _L().orc_lloyd_params_byte(c)


def lloyd_inverse(family: int, fd: float, b: float, beta: float, hi: float) -> float:
    return _L().orc_lloyd_inverse(family, fd, b, beta, hi)


def lloyd(w_bits: np.ndarray, group: int = 32, rounds: int = 25, force_cand: np.ndarray | None = None,
          cold_start: bool = False, threads: int | None = None) -> dict:
    """[G32] §1.3 / §5.1 producer. Returns a dict with codes [n,k] (q | sign<<3), levels
    [n, k/group, 8] (double), params [n, k/group] (the [G32] §2 byte), cand, trace
    [n, k/group, rounds+2], cand_gap and min_margin (both per group)."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    ng = k // group
    codes = np.empty((n, k), np.uint8)
    levels = np.empty((n, ng, 8), np.float64)
    params = np.empty((n, ng), np.uint8)
    cand = np.empty((n, ng), np.int32)
    trace = np.empty((n, ng, rounds + 2), np.float64)
    gap = np.empty((n, ng), np.float64)
    margin = np.empty((n, ng), np.float64)
    fc = None if force_cand is None else np.ascontiguousarray(force_cand, dtype=np.int32).reshape(-1)
    mode = np.array([1 if cold_start else 0], np.int32)
    _rows_parallel(n, lambda r0, r1: _L().orc_lloyd(_p(w), n, k, group, rounds, _p(fc), _p(mode),
                                                    r0, r1, _p(codes), _p(levels), _p(params),
                                                    _p(cand), _p(trace), _p(gap), _p(margin)),
                   threads)
    return dict(codes=codes, levels=levels, params=params, cand=cand, trace=trace,
                cand_gap=gap, min_margin=margin)


def kmeans_lut16(w_bits: np.ndarray, group: int = 64, rounds: int = 25,
                 threads: int | None = None) -> dict:
    """[KM] §1.2 per-block k-means with 16 centroids. Returns codes [n, k], lut fp16 bits
    [n, k/group, 16], trace [n, k/group, rounds+1], min_margin [n, k/group]."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    ng = k // group
    codes = np.empty((n, k), np.uint8)
    lut = np.empty((n, ng, 16), np.uint16)
    trace = np.empty((n, ng, rounds + 1), np.float64)
    margin = np.empty((n, ng), np.float64)
    _rows_parallel(n, lambda r0, r1: _L().orc_kmeans_lut16(_p(w), n, k, group, rounds, r0, r1,
                                                           _p(codes), _p(lut), _p(trace),
                                                           _p(margin)), threads)
    return dict(codes=codes, lut=lut, trace=trace, min_margin=margin)


def storage_bytes(fmt: int, nweights: float, group: int) -> float:
    return _L().orc_storage_bytes(fmt, float(nweights), group)


def storage_lloyd_codebook_bytes(nweights: float, group: int) -> float:
    return _L().orc_storage_lloyd_codebook_bytes(float(nweights), group)


def bf16x_encode(w_bits: np.ndarray) -> dict:
    """[BX] BF16X encoding of a bf16 [n, k] matrix (k % 16 == 0): dict of sm uint8 [n, k],
    hdr uint64 [n, k/16], sb_off uint32 [S + 1], ovf uint8 [escaped]."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    L = _L()
    S = L.orc_bf16x_superblocks(n, k)
    sm = np.empty((n, k), np.uint8)
    hdr = np.empty((n, k // 16), np.uint64)
    sb = np.empty(S + 1, np.uint32)
    ovf = np.empty(max(n * k, 1), np.uint8)
    cnt = np.zeros(1, np.int64)
    rc = L.orc_bf16x_encode(_p(w), n, k, _p(sm), _p(hdr), _p(sb), _p(ovf), ovf.size, _p(cnt))
    if rc != 0:
        raise ValueError(f"orc_bf16x_encode: {rc}")
    return dict(sm=sm, hdr=hdr, sb_off=sb, ovf=ovf[:int(cnt[0])].copy())


def bf16x_decode(enc: dict, n: int, k: int) -> np.ndarray:
    """Inverse of bf16x_encode: bf16 bits [n, k]. Raises if the index fields disagree with
    the escape table."""
    out = np.empty((n, k), np.uint16)
    ovf = np.ascontiguousarray(enc["ovf"], np.uint8)
    ovf_buf = ovf if ovf.size else np.zeros(1, np.uint8)
    rc = _L().orc_bf16x_decode(_p(np.ascontiguousarray(enc["sm"], np.uint8)),
                               _p(np.ascontiguousarray(enc["hdr"], np.uint64)),
                               _p(np.ascontiguousarray(enc["sb_off"], np.uint32)), _p(ovf_buf),
                               ovf.size, n, k, _p(out))
    if rc != 0:
        raise ValueError(f"orc_bf16x_decode: {rc}")
    return out


# --- [DG] water-filling (3/4/5-bit blocks in one index space) ------------------------------

def wf_analyze(w_bits: np.ndarray, lam: float, threads: int | None = None):
    """Per 64-weight block: (scale bf16 bits [n, k/64], width uint8 [n, k/64], dist fp64
    [n, k/64, 3] = squared error at 3, 4, 5 bits)."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    scale = np.empty((n, k // 64), np.uint16)
    width = np.empty((n, k // 64), np.uint8)
    dist = np.empty((n, k // 64, 3), np.float64)
    _rows_parallel(n, lambda r0, r1: _L().orc_wf_analyze(_p(w), n, k, float(lam), r0, r1, _p(scale),
                                                         _p(width), _p(dist)), threads)
    return scale, width, dist


def wf_offsets(width: np.ndarray) -> np.ndarray:
    """Byte offset of every block (8 * width bytes each, row-major) and the total."""
    wd = np.ascontiguousarray(width, dtype=np.uint8).reshape(-1)
    off = np.empty(wd.size + 1, np.uint32)
    rc = _L().orc_wf_offsets(_p(wd), wd.size, _p(off))
    if rc != 0:
        raise ValueError(f"orc_wf_offsets: {rc}")
    return off


def wf_pack(w_bits: np.ndarray, scale: np.ndarray, width: np.ndarray, blk_off: np.ndarray,
            threads: int | None = None) -> np.ndarray:
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    n, k = w.shape
    scale = np.ascontiguousarray(scale, dtype=np.uint16)
    width = np.ascontiguousarray(width, dtype=np.uint8)
    blk_off = np.ascontiguousarray(blk_off, dtype=np.uint32)
    packed = np.zeros(int(blk_off[-1]), np.uint8)
    _rows_parallel(n, lambda r0, r1: _L().orc_wf_pack(_p(w), n, k, _p(scale), _p(width), _p(blk_off),
                                                      r0, r1, _p(packed)), threads)
    return packed


def wf_dequant(packed: np.ndarray, scale: np.ndarray, width: np.ndarray, blk_off: np.ndarray,
               n: int, k: int, threads: int | None = None) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    if packed.size == 0:
        packed = np.zeros(1, np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.uint16)
    width = np.ascontiguousarray(width, dtype=np.uint8)
    blk_off = np.ascontiguousarray(blk_off, dtype=np.uint32)
    out = np.empty((n, k), np.uint16)
    _rows_parallel(n, lambda r0, r1: _L().orc_wf_dequant(_p(packed), _p(scale), _p(width), _p(blk_off),
                                                         n, k, r0, r1, _p(out)), threads)
    return out


def wf_matmul_rows(packed: np.ndarray, scale: np.ndarray, width: np.ndarray, blk_off: np.ndarray,
                   n: int, k: int, x_bits: np.ndarray, rows: np.ndarray | None = None):
    """The product a consumer of the water-filled format computes, by its definition:
    y[b, j] = sum_c Wdeq[rows[j], c] * x[b, c] in double with Wdeq = wf_dequant (the
    reconstruction through the 5-bit index space, "MiniCPM5-1B 验证…" §2.1), and the error
    scale bound[b, j] = sum_c |Wdeq[rows[j], c]| |x[b, c]|. x is bf16 bits [m, k]."""
    wd = bf16_to_f64(wf_dequant(packed, scale, width, blk_off, n, k))
    if rows is not None:
        wd = wd[np.asarray(rows, np.int64)]
    x = bf16_to_f64(np.atleast_2d(np.asarray(x_bits, np.uint16)))
    return x @ wd.T, np.abs(x) @ np.abs(wd).T
