"""Thin Python binding of libwq (include/wq.h): group-wise 4-bit weight coding and W4A16
matmul on B200.

Every function marshals torch CUDA tensors into the C ABI and calls one entry point of
libwq.so; all arithmetic runs in the library's CUDA kernels. There is no CPU or
PyTorch fallback: importing the package fails if libwq.so has not been built
(``python w4a16_matmul_b200/build.py``), and every call fails if the tensors are not on
a CUDA device. PyTorch supplies device memory and the current stream only.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# WQ_DEBUG=1 selects the debug build of the same library (device-side index and finite-input
# checks, reported through device_error()); it is built with `build.py --debug`
DEBUG = os.environ.get("WQ_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libwq_debug.so" if DEBUG else "libwq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "wq.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python w4a16_matmul_b200/build.py"
                      f"{' --debug' if DEBUG else ''}` (nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

# --- constants mirrored from include/wq.h -----------------------------------------------
WQ_OK, WQ_EINVAL, WQ_EALIGN, WQ_EUNSUPPORTED, WQ_ECUDA, WQ_ETIMEOUT, WQ_EDATA = range(7)
FMT_DYADIC4, FMT_LLOYD8S, FMT_LUT16 = 0, 1, 2
LLOYD_G32_WARM, LLOYD_KMEANS16 = 0, 1
GEMV_MAX_GROUPED = 192


class WqWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("group", ctypes.c_int32), ("n", ctypes.c_int64),
                ("k", ctypes.c_int64), ("packed", ctypes.c_void_p), ("aux", ctypes.c_void_p)]


class WqLloydParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("rounds", ctypes.c_int32)]


_i32, _i64, _vp, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
_WP = ctypes.POINTER(WqWeight)
_SIG = {
    "wq_status_string": ([_i32], ctypes.c_char_p),
    "wq_last_error": ([], ctypes.c_char_p),
    "wq_version": ([], _i32),
    "wq_quantize_dyadic": ([_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp], _i32),
    "wq_quantize_lloyd": ([_vp, _i64, _i64, ctypes.POINTER(WqLloydParams), _vp, _vp, _vp, _vp,
                           _vp, _vp], _i32),
    "wq_pack": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "wq_fake_quant_ste": ([_vp, _i64, _i64, _i32, _vp, _vp, _vp, _vp, _vp], _i32),
    "wq_gumbel_st_backward": ([_vp, _i64, _i64, _i32, _vp, ctypes.c_float, _vp, _vp, _vp, _vp], _i32),
    "wq_unpack": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "wq_dequant": ([_WP, _vp, _vp], _i32),
    "wq_gemv_w4a16": ([_WP, _vp, _i32, _vp, _vp], _i32),
    "wq_gemv_w4a16_grouped": ([_WP, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i32, _i32, _vp], _i32),
    "wq_gemv_plan_create": ([_WP, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i32, _i32,
                             ctypes.POINTER(_vp)], _i32),
    "wq_gemv_plan_launch": ([_vp, _vp], _i32),
    "wq_gemv_plan_destroy": ([_vp], None),
    "wq_gemv_plan_set_overlap": ([_vp, _i32], _i32),
    "wq_gemm_workspace_bytes": ([_WP, _i64], _sz),
    "wq_gemm_w4a16": ([_WP, _vp, _i64, _vp, _vp, _sz, _vp], _i32),
    "wq_gemm_w4a16_static": ([_WP, _vp, _i64, _vp, _vp], _i32),
    "wq_debug_fail_next_launches": ([_i32], None),
    "wq_device_error": ([ctypes.POINTER(_i32)], _i32),
    "wq_quantize_wf_analyze": ([_vp, _i64, _i64, ctypes.c_double, _vp, _vp, _vp, _vp, _vp], _i32),
    "wq_quantize_wf_pack": ([_vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp], _i32),
    "wq_dequant_wf": ([_vp, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _vp], _i32),
    "wq_gemv_wf": ([_vp, _i64, _vp, _vp, _vp, _i64, _i64, _vp, _i32, _vp, _vp], _i32),
    "wq_bf16x_superblocks": ([_i64, _i64], _i64),
    "wq_bf16x_count": ([_vp, _i64, _i64, _vp, _vp], _i32),
    "wq_bf16x_encode": ([_vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp], _i32),
    "wq_bf16x_decode": ([_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp], _i32),
}
for _name, (_args, _res) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


def header_functions() -> list[str]:
    """Names of the functions include/wq.h declares (for export checks)."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(wq_\w+)\s*\(", text, re.M)))


class WqError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_lib.wq_status_string(status).decode()}: {detail}")


def _check(status: int) -> None:
    if status != WQ_OK:
        raise WqError(status, (_lib.wq_last_error() or b"").decode())


def last_error() -> str:
    return (_lib.wq_last_error() or b"").decode()


def device_error() -> int:
    """Reads and clears the device error words (nonzero: a bounded GPU wait expired, a BF16X
    kernel met an overflow index past its table, or a water-filling kernel met a block whose
    width or offset does not fit its buffer)."""
    code = _i32(0)
    st = _lib.wq_device_error(ctypes.byref(code))
    if st not in (WQ_OK, WQ_ETIMEOUT, WQ_EDATA):
        _check(st)
    return code.value


def version() -> int:
    return _lib.wq_version()


def debug_fail_next_launches(count: int) -> None:
    _lib.wq_debug_fail_next_launches(count)


def _stream(t: torch.Tensor | None = None):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device if t is not None else None).cuda_stream)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _u16(t: torch.Tensor) -> torch.Tensor:
    """View of a 16-bit tensor (bf16 / fp16 / int16) as raw 16-bit storage."""
    return t


@dataclass
class PackedWeight:
    """A packed 4-bit weight: codes two per byte plus per-group scale / levels / centroids."""
    fmt: int
    group: int
    n: int
    k: int
    packed: torch.Tensor          # uint8 [n, k/2]
    aux: torch.Tensor             # bf16 [n, k/g] | fp32 [n, k/32, 8] | fp16 [n, k/64, 16]

    def desc(self) -> WqWeight:
        return WqWeight(self.fmt, self.group, self.n, self.k, self.packed.data_ptr(), self.aux.data_ptr())


# --- producers ---------------------------------------------------------------------------

def quantize_dyadic(w: torch.Tensor, group: int = 64, codes: bool = False, packed: bool = True):
    """Dyadic 4-bit quantisation of a bf16 [n, k] weight. Returns (PackedWeight, codes|None);
    PackedWeight is None when packed=False."""
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    scale = torch.empty((n, k // group), dtype=torch.bfloat16, device=w.device)
    c = torch.empty((n, k), dtype=torch.uint8, device=w.device) if codes else None
    p = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device) if packed else None
    _check(_lib.wq_quantize_dyadic(_ptr(w), n, k, group, _ptr(scale), _ptr(c), _ptr(p), _stream(w)))
    pw = PackedWeight(FMT_DYADIC4, group, n, k, p, scale) if packed else None
    return pw, c


def fake_quant_ste(z: torch.Tensor, scale: torch.Tensor, group: int = 64, codes: bool = False,
                   packed: bool = False):
    """STE forward on an fp32 latent z [n, k] with bf16 scales [n, k/group]: returns
    (q fp32 [n, k], codes uint8 [n, k] | None, packed uint8 [n, k/2] | None). The backward of
    the straight-through estimator is the identity."""
    _cuda(z, torch.float32, "z")
    _cuda(scale, torch.bfloat16, "scale")
    n, k = z.shape
    q = torch.empty_like(z)
    c = torch.empty((n, k), dtype=torch.uint8, device=z.device) if codes else None
    p = torch.empty((n, k // 2), dtype=torch.uint8, device=z.device) if packed else None
    _check(_lib.wq_fake_quant_ste(_ptr(z), n, k, group, _ptr(scale), _ptr(q), _ptr(c), _ptr(p),
                                  _stream(z)))
    return q, c, p


def gumbel_st_backward(z: torch.Tensor, scale: torch.Tensor, gq: torch.Tensor, tau: float,
                       group: int = 64, scale_grad: bool = True):
    """Gumbel-ST backward (soft = softmax(-dist/tau).codes, q = hard + (soft - soft.detach()))
    for the upstream gradient gq: returns (gz fp32 [n, k], gscale fp32 [n, k/group] | None).
    The forward value of Gumbel-ST is the hard code, i.e. fake_quant_ste's q."""
    _cuda(z, torch.float32, "z")
    _cuda(gq, torch.float32, "gq")
    _cuda(scale, torch.bfloat16, "scale")
    n, k = z.shape
    gz = torch.empty_like(z)
    gs = torch.empty((n, k // group), dtype=torch.float32, device=z.device) if scale_grad else None
    _check(_lib.wq_gumbel_st_backward(_ptr(z), n, k, group, _ptr(scale), float(tau), _ptr(gq),
                                      _ptr(gz), _ptr(gs), _stream(z)))
    return gz, gs


def quantize_lloyd(w: torch.Tensor, mode: int = LLOYD_G32_WARM, rounds: int = 25,
                   codes: bool = False, trace: bool = False):
    """Codebook quantisation: mode LLOYD_G32_WARM (8 levels + sign per group of 32) or
    LLOYD_KMEANS16 (16 fp16 centroids per block of 64). Returns (PackedWeight, extras dict)."""
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    dev = w.device
    p = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
    c = torch.empty((n, k), dtype=torch.uint8, device=dev) if codes else None
    if mode == LLOYD_G32_WARM:
        g = 32
        book = torch.empty((n, k // g, 8), dtype=torch.float32, device=dev)
        params = torch.empty((n, k // g), dtype=torch.uint8, device=dev)
        tr = torch.empty((n, k // g, rounds + 2), dtype=torch.float32, device=dev) if trace else None
        fmt = FMT_LLOYD8S
    else:
        g = 64
        book = torch.empty((n, k // g, 16), dtype=torch.float16, device=dev)
        params = None
        tr = torch.empty((n, k // g, rounds + 1), dtype=torch.float32, device=dev) if trace else None
        fmt = FMT_LUT16
    prm = WqLloydParams(mode, rounds)
    _check(_lib.wq_quantize_lloyd(_ptr(w), n, k, ctypes.byref(prm), _ptr(c), _ptr(p), _ptr(book),
                                  _ptr(params), _ptr(tr), _stream(w)))
    return PackedWeight(fmt, g, n, k, p, book), dict(codes=c, params=params, trace=tr)


def pack(codes: torch.Tensor) -> torch.Tensor:
    _cuda(codes, torch.uint8, "codes")
    n, k = codes.shape
    out = torch.empty((n, k // 2), dtype=torch.uint8, device=codes.device)
    _check(_lib.wq_pack(_ptr(codes), n, k, _ptr(out), _stream(codes)))
    return out


def unpack(packed: torch.Tensor) -> torch.Tensor:
    _cuda(packed, torch.uint8, "packed")
    n, kh = packed.shape
    out = torch.empty((n, 2 * kh), dtype=torch.uint8, device=packed.device)
    _check(_lib.wq_unpack(_ptr(packed), n, 2 * kh, _ptr(out), _stream(packed)))
    return out


def dequant(w: PackedWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """Dense reconstruction: bf16 [n, k] (fp16 [n, k] for LUT16), into `out` if given."""
    dt = torch.float16 if w.fmt == FMT_LUT16 else torch.bfloat16
    if out is None:
        out = torch.empty((w.n, w.k), dtype=dt, device=w.packed.device)
    else:
        _cuda(out, dt, "out")
        if tuple(out.shape) != (w.n, w.k):
            raise ValueError(f"out must be [{w.n}, {w.k}]")
    d = w.desc()
    _check(_lib.wq_dequant(ctypes.byref(d), _ptr(out), _stream(w.packed)))
    return out


# --- consumers ---------------------------------------------------------------------------

def gemv(w: PackedWeight, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """y = Wdeq x for x bf16 [batch, k] (batch <= 16) -> bf16 [batch, n]. A CPU x is copied to
    the weight's device (pinned, non-blocking) and the result copied back."""
    host = not x.is_cuda
    if host:
        x = x.pin_memory().to(w.packed.device, non_blocking=True) if x.device.type == "cpu" else x
    x2 = x if x.dim() == 2 else x.reshape(1, -1)
    _cuda(x2, torch.bfloat16, "x")
    b = x2.shape[0]
    y = out if out is not None else torch.empty((b, w.n), dtype=torch.bfloat16, device=x2.device)
    d = w.desc()
    _check(_lib.wq_gemv_w4a16(ctypes.byref(d), _ptr(x2), b, _ptr(y), _stream(x2)))
    if host:
        return y.to("cpu")
    return y if x.dim() == 2 else y.reshape(-1)


def gemv_grouped(ws: list[PackedWeight], xs: list[torch.Tensor],
                 ys: list[torch.Tensor] | None = None) -> list[torch.Tensor]:
    """Independent GEMVs ys[i] = Wdeq(ws[i]) xs[i] in one launch (same format/group/batch)."""
    cnt = len(ws)
    b = xs[0].shape[0]
    for x in xs:
        _cuda(x, torch.bfloat16, "x")
    if ys is None:
        ys = [torch.empty((b, w.n), dtype=torch.bfloat16, device=xs[0].device) for w in ws]
    arr = (WqWeight * cnt)(*[w.desc() for w in ws])
    xp = (_vp * cnt)(*[x.data_ptr() for x in xs])
    yp = (_vp * cnt)(*[y.data_ptr() for y in ys])
    _check(_lib.wq_gemv_w4a16_grouped(arr, xp, yp, cnt, b, _stream(xs[0])))
    return ys


class GroupedGemv:
    """A prepared grouped GEMV (wq_gemv_plan): the arguments are checked and the kernel is
    chosen once, at construction; each call only enqueues the kernel, on the current stream
    (or `stream`), reading whatever the bound x buffers hold by then. The tensors are kept
    alive for the plan's lifetime. overlap=True lets each launch overlap the kernel before it
    in the stream (wq_gemv_plan_set_overlap): only where that kernel does not write the
    weights."""

    def __init__(self, ws: list[PackedWeight], xs: list[torch.Tensor], ys: list[torch.Tensor],
                 overlap: bool = False):
        if not (len(ws) == len(xs) == len(ys)):
            raise ValueError("ws, xs and ys must have the same length")
        for x in xs:
            _cuda(x, torch.bfloat16, "x")
        for y in ys:
            _cuda(y, torch.bfloat16, "y")
        self.cnt = len(ws)
        self.batch = xs[0].shape[0]
        self._keep = (ws, xs, ys)
        arr = (WqWeight * self.cnt)(*[w.desc() for w in ws])
        xp = (_vp * self.cnt)(*[x.data_ptr() for x in xs])
        yp = (_vp * self.cnt)(*[y.data_ptr() for y in ys])
        self._plan = _vp(None)
        _check(_lib.wq_gemv_plan_create(arr, xp, yp, self.cnt, self.batch, ctypes.byref(self._plan)))
        if overlap:
            self.set_overlap(True)

    def set_overlap(self, on: bool) -> None:
        _check(_lib.wq_gemv_plan_set_overlap(self._plan, 1 if on else 0))

    def __call__(self, stream=None) -> None:
        s = ctypes.c_void_p(stream if stream is not None else torch.cuda.current_stream().cuda_stream)
        _check(_lib.wq_gemv_plan_launch(self._plan, s))

    def close(self) -> None:
        # at interpreter shutdown the module globals may already be gone: the process is
        # exiting and the plan's host memory goes with it
        if getattr(self, "_plan", None) and self._plan.value and _lib is not None:
            _lib.wq_gemv_plan_destroy(self._plan)
            self._plan = _vp(None)

    def __del__(self):
        self.close()


def gemm_workspace_bytes(w: PackedWeight, m: int) -> int:
    d = w.desc()
    return int(_lib.wq_gemm_workspace_bytes(ctypes.byref(d), m))


def gemm(w: PackedWeight, x: torch.Tensor, out: torch.Tensor | None = None,
         workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = x Wdeq^T for x bf16 [m, k] -> bf16 [m, n] on the tcgen05 tensor cores."""
    _cuda(x, torch.bfloat16, "x")
    m = x.shape[0]
    y = out if out is not None else torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    need = gemm_workspace_bytes(w, m)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    d = w.desc()
    _check(_lib.wq_gemm_w4a16(ctypes.byref(d), _ptr(x), m, _ptr(y), _ptr(workspace),
                              need, _stream(x)))
    return y


def gemm_static(w: PackedWeight, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """gemm() with its scratch in the library's static device array (wq_gemm_w4a16_static):
    no workspace is allocated for the call."""
    _cuda(x, torch.bfloat16, "x")
    m = x.shape[0]
    y = out if out is not None else torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    d = w.desc()
    _check(_lib.wq_gemm_w4a16_static(ctypes.byref(d), _ptr(x), m, _ptr(y), _stream(x)))
    return y


# --- BF16X lossless codec ------------------------------------------------------------------
@dataclass
class Bf16xWeight:
    """A bf16 [n, k] matrix in the BF16X layout of include/wq.h. Unsigned fields are held in
    signed tensors of the same width (hdr: int64 for uint64, sb_off: int32 for uint32)."""
    n: int
    k: int
    sm: torch.Tensor        # uint8 [n, k]
    hdr: torch.Tensor       # int64 [n, k/16]
    sb_off: torch.Tensor    # int32 [S + 1]
    ovf: torch.Tensor       # uint8 [max(escapes, 16)]
    escapes: int

    def nbytes(self) -> int:
        """Bytes the encoding needs (the overflow table at its exact length)."""
        return self.sm.numel() + 8 * self.hdr.numel() + 4 * self.sb_off.numel() + self.escapes


def bf16x_superblocks(n: int, k: int) -> int:
    return int(_lib.wq_bf16x_superblocks(n, k))


def bf16x_count(w: torch.Tensor, sb_off: torch.Tensor) -> None:
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    _check(_lib.wq_bf16x_count(_ptr(w), n, k, _ptr(sb_off), _stream(w)))


def bf16x_encode(w: torch.Tensor) -> Bf16xWeight:
    """Encodes a bf16 [n, k] CUDA matrix. Synchronises once, to size the overflow table."""
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    dev = w.device
    S = bf16x_superblocks(n, k)
    if S < 0:
        raise WqError(WQ_EINVAL, f"k={k} is not a multiple of 16")
    sb = torch.empty(S + 1, dtype=torch.int32, device=dev)
    _check(_lib.wq_bf16x_count(_ptr(w), n, k, _ptr(sb), _stream(w)))
    total = int(sb[S].item()) & 0xFFFFFFFF
    sm = torch.empty((n, k), dtype=torch.uint8, device=dev)
    hdr = torch.empty((n, k // 16), dtype=torch.int64, device=dev)
    ovf = torch.empty(max(total, 16), dtype=torch.uint8, device=dev)
    _check(_lib.wq_bf16x_encode(_ptr(w), n, k, _ptr(sb), _ptr(sm), _ptr(hdr), _ptr(ovf), ovf.numel(),
                                _stream(w)))
    return Bf16xWeight(n, k, sm, hdr, sb, ovf, total)


def bf16x_encode_into(w: torch.Tensor, b: Bf16xWeight) -> None:
    """Both passes into an existing encoding of the same matrix (no allocation, no sync)."""
    n, k = w.shape
    _check(_lib.wq_bf16x_count(_ptr(w), n, k, _ptr(b.sb_off), _stream(w)))
    _check(_lib.wq_bf16x_encode(_ptr(w), n, k, _ptr(b.sb_off), _ptr(b.sm), _ptr(b.hdr), _ptr(b.ovf),
                                b.ovf.numel(), _stream(w)))


def bf16x_decode(b: Bf16xWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """The bf16 [n, k] matrix the encoding holds, bit for bit."""
    if out is None:
        out = torch.empty((b.n, b.k), dtype=torch.bfloat16, device=b.sm.device)
    _check(_lib.wq_bf16x_decode(_ptr(b.sm), _ptr(b.hdr), _ptr(b.sb_off), _ptr(b.ovf), b.ovf.numel(),
                                b.n, b.k, _ptr(out), _stream(out)))
    return out


# --- water-filling 3/4/5-bit dyadic blocks --------------------------------------------------
@dataclass
class WfWeight:
    """A bf16 [n, k] matrix as water-filled dyadic blocks (layout in include/wq.h). blk_off is
    uint32 held in an int32 tensor."""
    n: int
    k: int
    scale: torch.Tensor     # bf16 [n, k/64]
    width: torch.Tensor     # uint8 [n, k/64]
    blk_off: torch.Tensor   # int32 [n k/64 + 1]
    packed: torch.Tensor    # uint8 [max(total, 16)]
    total: int              # bytes of packed in use


def wf_analyze(w: torch.Tensor, lam: float, dist: bool = False):
    """Pass 1 of water-filling: (scale, width, blk_off, dist | None)."""
    _cuda(w, torch.bfloat16, "w")
    n, k = w.shape
    dev = w.device
    scale = torch.empty((n, k // 64), dtype=torch.bfloat16, device=dev)
    width = torch.empty((n, k // 64), dtype=torch.uint8, device=dev)
    off = torch.empty(n * (k // 64) + 1, dtype=torch.int32, device=dev)
    d = torch.empty((n, k // 64, 3), dtype=torch.float64, device=dev) if dist else None
    _check(_lib.wq_quantize_wf_analyze(_ptr(w), n, k, float(lam), _ptr(scale), _ptr(width), _ptr(off),
                                       _ptr(d), _stream(w)))
    return scale, width, off, d


def quantize_wf(w: torch.Tensor, lam: float) -> WfWeight:
    """Water-filling quantisation at water level lam. Synchronises once, to size packed."""
    n, k = w.shape
    scale, width, off, _ = wf_analyze(w, lam)
    total = int(off[-1].item()) & 0xFFFFFFFF
    packed = torch.empty(max(total, 16), dtype=torch.uint8, device=w.device)
    _check(_lib.wq_quantize_wf_pack(_ptr(w), n, k, _ptr(scale), _ptr(width), _ptr(off), _ptr(packed),
                                    packed.numel(), _stream(w)))
    return WfWeight(n, k, scale, width, off, packed, total)


def dequant_wf(q: WfWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    if out is None:
        out = torch.empty((q.n, q.k), dtype=torch.bfloat16, device=q.packed.device)
    _check(_lib.wq_dequant_wf(_ptr(q.packed), q.packed.numel(), _ptr(q.scale), _ptr(q.width),
                              _ptr(q.blk_off), q.n, q.k, _ptr(out), _stream(out)))
    return out


def gemv_wf(q: WfWeight, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """y = x Wdeq^T for water-filled weights; x bf16 [batch, k] (batch 1..16) -> bf16 [batch, n]."""
    _cuda(x, torch.bfloat16, "x")
    batch = x.shape[0]
    if out is None:
        out = torch.empty((batch, q.n), dtype=torch.bfloat16, device=x.device)
    _check(_lib.wq_gemv_wf(_ptr(q.packed), q.packed.numel(), _ptr(q.scale), _ptr(q.width), _ptr(q.blk_off),
                           q.n, q.k, _ptr(x), batch, _ptr(out), _stream(x)))
    return out
