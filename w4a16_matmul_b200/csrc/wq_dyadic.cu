// wq_dyadic.cu -- dyadic 4-bit quantisation ("MiniCPM5-1B 验证: 6× 压缩…" §2.1-2.3),
// nibble pack / unpack (§2.5) and dense reconstruction of all three packed formats.
//
// All four kernels are HBM-bound streams: one thread owns a 16-byte chunk of the widest
// array it touches, loads are 128-bit and coalesced, grids are a multiple of the SM count
// and loop grid-stride.
#include "wq_internal.cuh"

namespace wq {

WQ_DEBUG_WORD(dyadic)
namespace {

constexpr int kThreads = 256;

int stream_grid(int64_t items, int per_sm_blocks = 8) {
    int64_t blocks = (items + kThreads - 1) / kThreads;
    int64_t cap = (int64_t)sm_count() * per_sm_blocks;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

// ---------------------------------------------------------------------------------------
// Quantisation: scale = max|w| per group; idx = #{j in 1..15 : w > (2j-17) * scale/16}.
//
// That count is the argmin over the 16 codes with the lowest index on a tie (the
// midpoint between codes j-1 and j is (2j-17) * scale / 16, and a weight exactly on a
// midpoint stays with the lower code). With t = 16 w / scale it equals
// (ceil(t) + 16) >> 1 clamped to 0..15: the count only changes where t crosses an odd
// integer. t is formed with one correctly rounded reciprocal per group and one multiply
// (relative error <= 2^-23, |t| <= 16, so |error| < 2e-6). For bf16 w and scale with
// 16 w / scale != u (u odd, |u| <= 15) the distance |16 w / scale - u| is at least
// 2^-16, so t is on the right side of every odd integer except when w sits exactly on
// a midpoint; that case can only overshoot by one, and is corrected by an exact
// comparison against the midpoint below (a bf16 times an odd integer <= 17 over 16, exact
// in fp32).
// ---------------------------------------------------------------------------------------
// One warp-contiguous block of 32 chunks (8 weights each) per unrolled step u: each thread
// issues its U 128-bit loads before it computes, so U loads per thread are in flight.
// 1/x from the special-function unit (relative error below 2^-22 for normal x).
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

template <int G, typename I>
__device__ __forceinline__ void quantize_chunk(uint4 v, bool live, I c, uint16_t* __restrict__ scale,
                                               uint2* __restrict__ codes, uint32_t* __restrict__ packed) {
    constexpr int LANES = G / 8;                 // threads per group (8 or 4)
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(wv[i] << 16);
        f[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
    // group absmax: |w| pairs by clearing the sign bits, a packed bf16 max over the chunk,
    // then the two halves and the group's lanes
    uint32_t m2;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m2) : "r"(v.x & 0x7FFF7FFFu), "r"(v.y & 0x7FFF7FFFu));
    uint32_t m3;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m3) : "r"(v.z & 0x7FFF7FFFu), "r"(v.w & 0x7FFF7FFFu));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m2) : "r"(m2), "r"(m3));
    float amax = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
#pragma unroll
    for (int off = 1; off < LANES; off <<= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, off));

    uint32_t p;
    if (amax == 0.f) {
        p = 0;                                   // every code ties: code 0
    } else if (amax >= 0x1p-96f && amax <= 0x1p96f) {
        // idx = #{j in 1..15 : w > m_j}, m_j = (2j - 17) s / 16, is ceil(u) - 1 (at most 15)
        // with u = 8 w / s + 8.5 (w > m_j <=> u > j; u >= 0.5 as |w| <= s). u is formed with
        // the hardware reciprocal (relative error below 2^-22) and one FMA: |error| < 2^-18,
        // while a u that is not an integer is at least 2^-17 from one (w and s being bf16);
        // ceil is an add of 2^23 rounded upward. Only an exact midpoint (u an integer) can come out one too high;
        // the exact comparison against the midpoint below corrects it (for idx 0 that
        // midpoint, -17 s / 16, is below every weight, so no check is needed).
        const float c8 = 8.0f * rcp_approx(amax);
        const float s8 = amax * 0.125f, m17 = -17.0f * amax * 0.0625f;
        // weights j and j + 4 side by side on the packed fp32x2 pipe (each lane of an x2
        // instruction rounds exactly as its scalar form), so the nibble packing below also
        // runs as pairs: (low half of the word, high half)
        float2 cf[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 fw = make_float2(f[j], f[j + 4]);
            const float2 u = __ffma2_rn(fw, make_float2(c8, c8), make_float2(8.5f, 8.5f));
            float2 x = __fadd2_rn(__fadd2_ru(u, make_float2(8388608.0f, 8388608.0f)),
                                  make_float2(-8388609.0f, -8388609.0f));               // ceil(u) - 1
            x = make_float2(fminf(x.x, 15.0f), fminf(x.y, 15.0f));
            const float2 mlo = __ffma2_rn(x, make_float2(s8, s8), make_float2(m17, m17));   // exact midpoint
            const float2 xm1 = __fadd2_rn(x, make_float2(-1.0f, -1.0f));
            cf[j] = make_float2(fw.x > mlo.x ? x.x : xm1.x, fw.y > mlo.y ? x.y : xm1.y);
        }
        // nibbles packed with exact float arithmetic: 2^23 + sum cf_i 16^i (< 2^24) holds the
        // 16-bit half of the packed word in its low mantissa bits (both halves at once)
        float2 acc = __fadd2_rn(cf[0], make_float2(8388608.0f, 8388608.0f));
        acc = __ffma2_rn(cf[1], make_float2(16.0f, 16.0f), acc);
        acc = __ffma2_rn(cf[2], make_float2(256.0f, 256.0f), acc);
        acc = __ffma2_rn(cf[3], make_float2(4096.0f, 4096.0f), acc);
        p = prmt(__float_as_uint(acc.x), __float_as_uint(acc.y), 0x5410u);
    } else {
        // keep 16/s and 17*s/16 finite for tiny and huge scales: rescale w and s by a power
        // of two (exact; a weight that underflows is far below the smallest step)
        const float ps = amax < 0x1p-96f ? 0x1p32f : 0x1p-32f;
        const float s = amax * ps;
        const float c16 = 16.0f * __frcp_rn(s);
        const float s16 = s * 0.0625f;
        const float two_s16 = 2.0f * s16, m17 = -17.0f * s16;
        p = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float ws = f[i] * ps;
            int cnt = (__float2int_ru(ws * c16) + 16) >> 1;
            cnt = min(max(cnt, 0), 15);
            // exact midpoint below code cnt: (2 cnt - 17) * s/16
            const float mlo = fmaf((float)cnt, two_s16, m17);
            if (cnt > 0 && !(ws > mlo)) cnt -= 1;
            p |= (uint32_t)cnt << (4 * i);
        }
    }
    if (live) {
        if (packed) packed[c] = p;
        if (codes) {
            // nibbles -> bytes: c0 c1 c2 c3 | c4 c5 c6 c7
            const uint32_t e = p & 0x0F0F0F0Fu, o = (p >> 4) & 0x0F0F0F0Fu;
            codes[c] = make_uint2(prmt(e, o, 0x5140u), prmt(e, o, 0x7362u));
        }
        // the scale array [n, k/G] tiles the rows exactly, so group (row, col/G) is number
        // c / LANES in row-major order
        if ((threadIdx.x & (LANES - 1)) == 0) scale[c / LANES] = (uint16_t)float_to_bf16_bits(amax);
    }
}

// I: the chunk index type (uint32_t when every chunk index fits, else uint64_t).
template <int G, typename I>
__global__ void __launch_bounds__(kThreads)
quantize_dyadic_kernel(const uint4* __restrict__ w, I n_chunks, uint16_t* __restrict__ scale,
                       uint2* __restrict__ codes, uint32_t* __restrict__ packed) {
    constexpr int U = 4;
    const I stride = (I)gridDim.x * blockDim.x * U;
    const I lane = threadIdx.x & 31;
    // a warp covers U consecutive blocks of 32 chunks; groups never straddle n_chunks
    for (I c0 = ((I)blockIdx.x * blockDim.x + (threadIdx.x & ~31u)) * U; c0 < n_chunks; c0 += stride) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const I c = c0 + 32 * u + lane;
            v[u] = c < n_chunks ? ldg_nc_v4(w + c) : make_uint4(0, 0, 0, 0);
            WQ_DCHECK(bf16x8_finite(v[u]), kDbgNonFiniteWeight + 1);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const I c = c0 + 32 * u + lane;
            quantize_chunk<G, I>(v[u], c < n_chunks, c, scale, codes, packed);
        }
    }
}

__global__ void __launch_bounds__(kThreads)
pack_kernel(const uint4* __restrict__ codes, int64_t n16, uint2* __restrict__ packed) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 c = ldg_nc_v4(codes + i);
        const uint32_t in[4] = {c.x, c.y, c.z, c.w};
        uint32_t out[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t a = in[2 * j], b = in[2 * j + 1];
            // bytes a = c0 c1 c2 c3 -> (c0 | c1 << 4) | (c2 | c3 << 4) << 8, then b above
            const uint32_t lo = (a & 0x0F) | ((a >> 4) & 0xF0) | ((a >> 8) & 0x0F00) | ((a >> 12) & 0xF000);
            const uint32_t hi = (b & 0x0F) | ((b >> 4) & 0xF0) | ((b >> 8) & 0x0F00) | ((b >> 12) & 0xF000);
            out[j] = lo | hi << 16;
        }
        packed[i] = make_uint2(out[0], out[1]);
    }
}

__global__ void __launch_bounds__(kThreads)
unpack_kernel(const uint2* __restrict__ packed, int64_t n16, uint4* __restrict__ codes) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint2 p = packed[i];
        const uint32_t in[2] = {p.x, p.y};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t v = in[j];
            out[2 * j] = (v & 0x0F) | ((v & 0xF0) << 4) | ((v & 0x0F00) << 8) | ((v & 0xF000) << 12);
            const uint32_t u = v >> 16;
            out[2 * j + 1] = (u & 0x0F) | ((u & 0xF0) << 4) | ((u & 0x0F00) << 8) | ((u & 0xF000) << 12);
        }
        codes[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ---------------------------------------------------------------------------------------
// Dense reconstruction. One thread: 8 codes (one 32-bit packed word) -> 16 bytes.
// ---------------------------------------------------------------------------------------

// DYADIC4: bf16(step * (idx - 8)), step = scale / 8. The product is exact in fp32 (an
// 8-bit significand times an integer of magnitude <= 8, scaled by 2^-3), so the bf16
// conversion is the one and only rounding.
// A warp takes 128 consecutive packed words per trip, lane l the words l, l + 32, l + 64 and
// l + 96, so every 4-byte load covers 128 contiguous bytes and every 16-byte store 512
// contiguous bytes of the output (four 16-byte stores per thread at a 64-byte stride ran
// 30 % slower: each store instruction then touches 32 sectors half-way). Groups and rows are
// contiguous in the flat packed array, so word i's scale is scale[8 i / group].
__global__ void __launch_bounds__(kThreads)
dequant_dyadic_kernel(const uint32_t* __restrict__ packed, const uint16_t* __restrict__ scale,
                      int64_t n_words, int gshift, uint4* __restrict__ out) {
    constexpr int U = 4;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * (32 * U);
         base < n_words; base += warps * (32 * U)) {
        uint32_t p[U], sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + 32 * u + lane;
            p[u] = 0x88888888u;
            sc[u] = 0;
            if (i < n_words) {
                WQ_DCHECK((i >> gshift) <= ((n_words - 1) >> gshift), kDbgIndex + 1);
                p[u] = __ldg(packed + i);
                sc[u] = ldg_u16(scale + (i >> gshift));
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = base + 32 * u + lane;
            if (i >= n_words) break;
            uint4 o;
            if ((sc[u] & 0x7FFFu) >= 0x0380u) {
                // scale >= 2^-120: every nonzero step * (idx - 8) is a normal bf16. Two codes
                // at a time: (w >> 4j) & 0x000F000F | 0x4300 in each half is the bf16 pair
                // (128 + idx_j, 128 + idx_j+4); minus 136 gives idx - 8 exactly, and one bf16x2
                // multiply by (step, step) (step = scale / 8: the exponent field minus 3)
                // rounds step * (idx - 8) once, which is the definition.
                const uint32_t st2 = prmt(sc[u] - 0x0180u, 0u, 0x1010u);
                uint32_t q[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t m = ((p[u] >> (4 * j)) & 0x000F000Fu) | 0x43004300u;
                    const uint32_t d = bf16x2_fma(m, 0x3F803F80u, 0xC308C308u);    // idx - 8
                    q[j] = bf16x2_fma(d, st2, 0x80008000u);                        // + (-0)
                }
                // q[j] = (code j, code j + 4): regroup into (0, 1) (2, 3) (4, 5) (6, 7)
                o = make_uint4(prmt(q[0], q[1], 0x5410u), prmt(q[2], q[3], 0x5410u),
                               prmt(q[0], q[1], 0x7632u), prmt(q[2], q[3], 0x7632u));
            } else {
                // tiny (or zero) scales: exact in fp32, rounded once to bf16
                const float step = bf16_bits_to_float(sc[u]) * 0.125f;
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) v[j] = step * (float)((int)((p[u] >> (4 * j)) & 15) - 8);
                o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7]));
            }
            stg_cs_v4(out + i, o);
        }
    }
}

// LLOYD8S: code = q | sign << 3; bf16(+/- level[q]) from the group's 8 fp32 levels.
__global__ void __launch_bounds__(kThreads)
dequant_lloyd_kernel(const uint32_t* __restrict__ packed, const float4* __restrict__ levels,
                     int64_t n_words, uint4* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t p = packed[i];
        const int64_t g = i / 4;                    // 32 codes per group = 4 words
        const float4 l0 = levels[2 * g], l1 = levels[2 * g + 1];
        const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = (p >> (4 * j)) & 15;
            float a = lv[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) a = ((c & 7) == (uint32_t)q) ? lv[q] : a;
            v[j] = (c & 8) ? -a : a;
        }
        out[i] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
}

// LUT16: the fp16 centroid itself.
__global__ void __launch_bounds__(kThreads)
dequant_lut16_kernel(const uint32_t* __restrict__ packed, const uint4* __restrict__ lut,
                     int64_t n_words, uint4* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t p = packed[i];
        const int64_t g = i / 8;                    // 64 codes per block = 8 words
        const uint4 a = lut[2 * g], b = lut[2 * g + 1];
        const uint32_t L[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t h[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t c = (p >> (4 * j)) & 15;
            uint32_t r = L[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) r = ((c >> 1) == (uint32_t)q) ? L[q] : r;
            h[j] = (c & 1) ? (r >> 16) : (r & 0xFFFF);
        }
        out[i] = make_uint4(h[0] | h[1] << 16, h[2] | h[3] << 16, h[4] | h[5] << 16, h[6] | h[7] << 16);
    }
}

}  // namespace

wq_status launch_quantize_dyadic(const uint16_t* w, int64_t n, int64_t k, int group,
                                 uint16_t* scale, uint8_t* codes, uint8_t* packed,
                                 cudaStream_t s) {
    const int64_t chunks = n * k / 8;
    const int grid = stream_grid((chunks + 3) / 4);
    // 32-bit chunk indices while c0 + stride stays below 2^32
    const bool narrow = chunks + (int64_t)grid * kThreads * 4 < (int64_t)1 << 32;
#define WQ_QUANT(G, I)                                                                          \
    quantize_dyadic_kernel<G, I><<<grid, kThreads, 0, s>>>((const uint4*)w, (I)chunks, scale,   \
                                                          (uint2*)codes, (uint32_t*)packed)
    if (group == 64) {
        if (narrow) WQ_QUANT(64, uint32_t); else WQ_QUANT(64, uint64_t);
    } else {
        if (narrow) WQ_QUANT(32, uint32_t); else WQ_QUANT(32, uint64_t);
    }
#undef WQ_QUANT
    return check_launch("quantize_dyadic");
}

wq_status launch_pack(const uint8_t* codes, int64_t n, int64_t k, uint8_t* packed, cudaStream_t s) {
    const int64_t n16 = n * k / 16;
    pack_kernel<<<stream_grid(n16), kThreads, 0, s>>>((const uint4*)codes, n16, (uint2*)packed);
    return check_launch("pack");
}

wq_status launch_unpack(const uint8_t* packed, int64_t n, int64_t k, uint8_t* codes, cudaStream_t s) {
    const int64_t n16 = n * k / 16;
    unpack_kernel<<<stream_grid(n16), kThreads, 0, s>>>((const uint2*)packed, n16, (uint4*)codes);
    return check_launch("unpack");
}

wq_status launch_dequant(const wq_weight& w, uint16_t* out, cudaStream_t s) {
    const int64_t n_words = w.n * w.k / 8;
    const int grid = stream_grid(n_words);
    if (w.fmt == WQ_FMT_DYADIC4) {
        dequant_dyadic_kernel<<<stream_grid((n_words + 3) / 4), kThreads, 0, s>>>(
            (const uint32_t*)w.packed, (const uint16_t*)w.aux, n_words, w.group == 64 ? 3 : 2, (uint4*)out);
    }
    else if (w.fmt == WQ_FMT_LLOYD8S)
        dequant_lloyd_kernel<<<grid, kThreads, 0, s>>>((const uint32_t*)w.packed,
                                                       (const float4*)w.aux, n_words, (uint4*)out);
    else
        dequant_lut16_kernel<<<grid, kThreads, 0, s>>>((const uint32_t*)w.packed,
                                                       (const uint4*)w.aux, n_words, (uint4*)out);
    return check_launch("dequant");
}

}  // namespace wq
