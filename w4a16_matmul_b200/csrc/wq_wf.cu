// wq_wf.cu -- water-filling dyadic blocks of 3, 4 or 5 bits in one level index space
// ("MiniCPM5-1B 验证: 6× 压缩…" §2.1 dyadic codebook, §6 water-filling).
//
// With half = 2^(b-1) and step = scale / half the b-bit codebook is step * {-half .. half-1},
// and the codebooks of different b line up: code idx_b of a b-bit block is code
// idx_5 = idx_b << (5 - b) of the 5-bit codebook of the same scale, so one reconstruction,
// bf16((scale / 16) * (idx_5 - 16)), serves every width. Per 64-weight block (the §2.2
// block, scale = max |w|) the width is the smallest b in {3, 4, 5} whose squared error
// D_b = sum (w - code)^2 lies at or under the water level 64 * lambda, else 5.
//
// Exactness: every midpoint between two codes, scale * odd / 2^b, is exact in fp32 for
// scales in [2^-100, 2^100] (in double otherwise), so the nearest-code search is exact;
// each error w - code is exact (the code is zero or within a factor of two of w), its
// square is exact in double, and D_b is summed over the block's weights in order, in double
// (one thread per block). Widths, codes and distortions are therefore bit-identical with a
// plain double-precision evaluation.
//
// Layout: scale bf16 [n, k/64]; width uint8 [n, k/64]; the blocks' bit streams back to back
// in row-major block order, block i taking 8 * width_i bytes with code j in bits
// [b j, b j + b) from bit 0 of its first byte (b = 4 is the nibble layout of §2.5);
// blk_off uint32 [n k/64 + 1] holds every block's byte offset and the total.
//
// Kernels: analyze (scale, the three distortions, width, the scan's tile totals), the shared
// in-place tile scan of the block sizes, pack (codes at the chosen width), dequant (eight
// threads per block: each rebuilds 8 weights from b whole bytes and stores 16 bytes, so a
// block's 128 output bytes leave in one coalesced run), and two GEMVs (the format's
// decode-side consumers) that rebuild the weights as the dequant does and multiply them on
// the tensor cores with fp32 accumulation: batches of 1 and 2 with the packed bytes staged
// in shared memory by bulk copies, larger batches 16 rows per warp.
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kThreads = 256;                   // one block of weights per thread
static_assert(kThreads == kScanTile, "an analyze CTA covers one scan tile");
constexpr int kPad = 33;                        // staged words per block (32 + 1: no bank conflicts)

__device__ int g_wf_error;                      // 0, or the first inconsistent-data code

__device__ __forceinline__ void report(int code) { atomicCAS(&g_wf_error, 0, code); }

// Stage this warp's 32 blocks (32 x 128 bytes) into shared memory, one block per 33 words.
__device__ __forceinline__ void stage_blocks(const uint4* __restrict__ w, int64_t nblk, int64_t first,
                                             uint32_t* sw) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int v = q * 32 + lane;             // 16-byte piece of the warp's 4 KB
        const int blk = v >> 3, word = 4 * (v & 7);
        uint4 x = make_uint4(0, 0, 0, 0);
        if (first + blk < nblk) x = ldg_nc_v4(w + (first + blk) * 8 + (v & 7));
        uint32_t* d = sw + blk * kPad + word;
        d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
    }
    __syncwarp();
}

// Largest |w| of the block as bf16 bits (the magnitude order of finite bf16 patterns).
__device__ __forceinline__ uint32_t block_absmax(const uint32_t* b) {
    uint32_t m = 0;
#pragma unroll 8
    for (int t = 0; t < 32; ++t) m = max(m, max(b[t] & 0x7FFFu, (b[t] >> 16) & 0x7FFFu));
    return m;
}

// idx_b of w: the number of midpoints (between codes x - 1 and x, x = 1 .. 2^b - 1) below w,
// found bit by bit (the midpoints increase with x; a tie goes to the lower code).
__device__ __forceinline__ int index_b(float w, float s, int b, bool fast) {
    const int half = 1 << (b - 1);
    int idx = 0;
    if (fast) {
        const float inv = __int_as_float((127 - b) << 23);          // 2^-b
        for (int bit = b - 1; bit >= 0; --bit) {
            const int cand = idx | (1 << bit);
            const float m = s * (float)(2 * cand - 2 * half - 1) * inv;
            if (w > m) idx = cand;
        }
    } else {
        const double sd = (double)s, wd = (double)w;
        for (int bit = b - 1; bit >= 0; --bit) {
            const int cand = idx | (1 << bit);
            const double m = sd * (double)(2 * cand - 2 * half - 1) / (double)(2 * half);
            if (wd > m) idx = cand;
        }
    }
    return idx;
}

// idx_5, idx_4 and idx_3 of w from one 5-bit search. The 4-bit midpoints are the 5-bit codes
// of odd index (s (2x - 17) / 16 = code_5(2x - 1)), and idx_5 places w against every 5-bit
// code but code_5(idx_5) itself, so idx_4 = idx_5 / 2, plus one when idx_5 is odd (and below
// 31) and w lies above code_5(idx_5); likewise idx_3 from idx_4 and the 4-bit codes.
__device__ __forceinline__ void index_543(float w, float s, bool fast, int& i5, int& i4, int& i3) {
    i5 = index_b(w, s, 5, fast);
    if (fast) {
        i4 = (i5 >> 1) + (((i5 & 1) && i5 < 31 && w > s * (float)(i5 - 16) * 0.0625f) ? 1 : 0);
        i3 = (i4 >> 1) + (((i4 & 1) && i4 < 15 && w > s * (float)(i4 - 8) * 0.125f) ? 1 : 0);
    } else {
        const double sd = (double)s, wd = (double)w;
        i4 = (i5 >> 1) + (((i5 & 1) && i5 < 31 && wd > sd * (double)(i5 - 16) / 16.0) ? 1 : 0);
        i3 = (i4 >> 1) + (((i4 & 1) && i4 < 15 && wd > sd * (double)(i4 - 8) / 8.0) ? 1 : 0);
    }
}

// The code value step * (idx - half) and the exact error w - code, as a double.
__device__ __forceinline__ double error_b(float w, float s, int b, int idx, bool fast) {
    const int half = 1 << (b - 1);
    if (fast) {
        const float c = s * (float)(idx - half) * __int_as_float((128 - b) << 23);   // 2^-(b-1)
        return (double)(w - c);
    }
    return (double)w - (double)s * (double)(idx - half) / (double)half;
}

__global__ void __launch_bounds__(kThreads)
wf_analyze_kernel(const uint4* __restrict__ w, int64_t nblk, double lambda64, uint16_t* __restrict__ scale,
                  uint8_t* __restrict__ width, uint32_t* __restrict__ blk_off, double* __restrict__ dist) {
    __shared__ uint32_t sw[kThreads / 32][32 * kPad];
    __shared__ uint32_t s_sum[kThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t ntiles = (nblk + kScanTile - 1) / kScanTile;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t t0 = tile * kScanTile, t1 = min(t0 + (int64_t)kScanTile, nblk);
        const int64_t first = t0 + 32 * wid;
        stage_blocks(w, nblk, first, sw[wid]);
        const int64_t i = first + lane;
        uint32_t size = 0;
        if (i < t1) {
            const uint32_t* b = sw[wid] + lane * kPad;
            const uint32_t sbits = block_absmax(b);
            const float s = bf16_bits_to_float(sbits);
            const bool fast = s >= 0x1p-100f && s <= 0x1p100f;
            // the three sums run side by side, each over the block's weights in order
            double D3 = 0.0, D4 = 0.0, D5 = 0.0;
            for (int j = 0; j < 64; ++j) {
                const float v = bf16_bits_to_float((j & 1) ? (b[j >> 1] >> 16) : (b[j >> 1] & 0xFFFFu));
                int i5, i4, i3;
                index_543(v, s, fast, i5, i4, i3);
                const double e3 = error_b(v, s, 3, i3, fast), e4 = error_b(v, s, 4, i4, fast),
                             e5 = error_b(v, s, 5, i5, fast);
                D3 = fma(e3, e3, D3);
                D4 = fma(e4, e4, D4);
                D5 = fma(e5, e5, D5);
            }
            if (dist) {
                dist[i * 3] = D3;
                dist[i * 3 + 1] = D4;
                dist[i * 3 + 2] = D5;
            }
            const int chosen = D3 <= lambda64 ? 3 : D4 <= lambda64 ? 4 : 5;
            scale[i] = (uint16_t)sbits;
            width[i] = (uint8_t)chosen;
            size = 8u * (uint32_t)chosen;
            blk_off[i] = size;
        }
        // the tile's total into bits 8..31 of its last entry, for the scan
        const uint32_t wsum = __reduce_add_sync(0xFFFFFFFFu, size);
        if (lane == 0) s_sum[wid] = wsum;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t tot = 0;
#pragma unroll
            for (int q = 0; q < kThreads / 32; ++q) tot += s_sum[q];
            blk_off[t1 - 1] |= tot << 8;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads)
wf_pack_kernel(const uint4* __restrict__ w, int64_t nblk, const uint16_t* __restrict__ scale,
               const uint8_t* __restrict__ width, const uint32_t* __restrict__ blk_off,
               uint8_t* __restrict__ packed, int64_t packed_bytes) {
    __shared__ uint32_t sw[kThreads / 32][32 * kPad];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
    for (int64_t first = ((int64_t)blockIdx.x * (kThreads / 32) + wid) * 32; first < nblk; first += warps * 32) {
        stage_blocks(w, nblk, first, sw[wid]);
        const int64_t i = first + lane;
        if (i < nblk) {
            const int bw = width[i];
            const int64_t off = (int64_t)blk_off[i];
            if (bw < 3 || bw > 5 || (off & 7) != 0 || off + 8 * bw > packed_bytes) {
                report(2001);
            } else {
                const uint32_t* b = sw[wid] + lane * kPad;
                const float s = bf16_bits_to_float(scale[i]);
                const bool fast = s >= 0x1p-100f && s <= 0x1p100f;
                unsigned long long* out = reinterpret_cast<unsigned long long*>(packed + off);
                unsigned long long acc = 0;
                int nbits = 0, word = 0;
                for (int t = 0; t < 64; ++t) {
                    const uint32_t h = (t & 1) ? (b[t >> 1] >> 16) : (b[t >> 1] & 0xFFFFu);
                    const unsigned long long idx = (unsigned long long)index_b(bf16_bits_to_float(h), s, bw, fast);
                    acc |= idx << nbits;
                    nbits += bw;
                    if (nbits >= 64) {
                        out[word++] = acc;
                        nbits -= 64;
                        acc = nbits > 0 ? idx >> (bw - nbits) : 0ull;
                    }
                }
            }
        }
        __syncwarp();                            // the staging buffer is reused next trip
    }
}

// The b bytes at byte0 of the bit streams (8 codes of b bits), as the low bits of a 64-bit
// word. Reads the 8-byte word holding byte0 and, when the bytes run past it, the next one:
// both lie inside the block when byte0 = off + b t (t < 8) with off a multiple of 8 and the
// block's 8 b bytes inside the buffer.
// The bytes are read once, so they bypass L1 (which then keeps what is reused, such as the
// GEMV's activations).
__device__ __forceinline__ unsigned long long ldg_na_u64(const unsigned long long* p) {
    unsigned long long v;
    asm("ld.global.nc.L1::no_allocate.u64 %0, [%1];" : "=l"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ unsigned long long wf_bytes(const uint8_t* packed, int64_t byte0, int bw) {
    const unsigned long long* src = reinterpret_cast<const unsigned long long*>(packed);
    const int64_t q = byte0 >> 3;
    const int sh = (int)(byte0 & 7) * 8;
    unsigned long long v = ldg_na_u64(src + q) >> sh;
    if (sh + 8 * bw > 64) v |= ldg_na_u64(src + q + 1) << (64 - sh);
    return v;
}

// idx_5 of the 8 codes of b bits in v (code j in bits b j ..), as pairs in column order (the
// two halves of each word). Each code is brought to bits 5 - b .. 4, where its value is
// idx_5 = code << (5 - b), by one 32-bit funnel shift of the 40 bits (the bits below it hold
// its neighbour and are masked off); a pair of codes is joined into one word by a byte
// permute. wf_decode8 then gives bf16((scale / 16) * (idx_5 - 16)) of each, as bf16 pairs;
// sb = the block's bf16 scale bits.
__device__ __forceinline__ void wf_fields8(unsigned long long v, int bw, uint32_t (&m)[4]) {
    const uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    const int s5 = 5 - bw;
    const uint32_t mp = (((1u << bw) - 1u) * 0x00010001u) << s5;      // idx_5 fields of a pair
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // code 2j starts at bit 2 j b, code 2j + 1 at (2j + 1) b; shifted right by that minus
        // s5 (>= 0 but for code 0, which is shifted left; < 32 but for code 7 at b = 5, bit 35)
        const uint32_t c0 = j == 0 ? lo << s5 : __funnelshift_r(lo, hi, 2 * j * bw - s5);
        const uint32_t c1 = (j == 3 && bw == 5) ? hi >> 3 : __funnelshift_r(lo, hi, (2 * j + 1) * bw - s5);
        m[j] = prmt(c0, c1, 0x5410u) & mp;                               // (idx_5 of 2j, of 2j + 1)
    }
}

// The reconstruction for a scale >= 2^-119, where every nonzero (scale / 16) (idx_5 - 16) is
// a normal bf16: idx_5 | 0x4300 is the bf16 number 128 + idx_5, minus 144 is idx_5 - 16
// exactly, and one bf16x2 multiply by scale / 16 (the exponent field minus 4) rounds the
// product once, as the definition reads.
__device__ __forceinline__ void wf_finish_normal(const uint32_t (&m)[4], uint32_t sb, uint32_t (&o)[4]) {
    const uint32_t s16x2 = prmt(sb - 0x0200u, 0u, 0x1010u);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t d = bf16x2_fma(m[j] | 0x43004300u, 0x3F803F80u, 0xC310C310u);   // idx_5 - 16
        o[j] = bf16x2_fma(d, s16x2, 0x80008000u);
    }
}

__device__ __forceinline__ bool wf_scale_normal(uint32_t sb) { return (sb & 0x7FFFu) >= 0x0400u; }

__device__ __forceinline__ void wf_decode8(unsigned long long v, int bw, uint32_t sb, uint32_t (&o)[4]) {
    uint32_t m[4];
    wf_fields8(v, bw, m);
    if (wf_scale_normal(sb)) {
        wf_finish_normal(m, sb, o);
    } else {
        const float s16 = bf16_bits_to_float(sb) * 0.0625f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = pack_bf16x2(s16 * (float)((int)(m[j] & 0xFFFFu) - 16), s16 * (float)((int)(m[j] >> 16) - 16));
    }
}

// True when a block's width and offset are consistent with a buffer of packed_bytes.
__device__ __forceinline__ bool wf_block_ok(int bw, int64_t off, int64_t packed_bytes) {
    return bw >= 3 && bw <= 5 && (off & 7) == 0 && off + 8 * bw <= packed_bytes;
}

__global__ void __launch_bounds__(kThreads)
wf_dequant_kernel(const uint8_t* __restrict__ packed, int64_t packed_bytes, const uint16_t* __restrict__ scale,
                  const uint8_t* __restrict__ width, const uint32_t* __restrict__ blk_off, int64_t nblk,
                  uint4* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gid < nblk * 8; gid += stride) {
        const int64_t i = gid >> 3;
        const int t = (int)(gid & 7);
        const int bw = __ldg(width + i);
        const int64_t off = (int64_t)ldg_u32(blk_off + i);
        uint32_t o[4] = {0, 0, 0, 0};
        if (!wf_block_ok(bw, off, packed_bytes)) {
            report(2000);
        } else {
            // this thread's 8 codes are the b bytes at off + b t (8 codes of b bits)
            wf_decode8(wf_bytes(packed, off + (int64_t)bw * t, bw), bw, ldg_u16(scale + i), o);
        }
        stg_cs_v4(out + gid, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

// Larger batches: y[i, r] = sum_c Wdeq[r, c] x[i, c] for up to 16 activation rows in one
// pass over the weights, Wdeq rebuilt exactly as wf_dequant_kernel does (bf16), products on
// the tensor cores (mma.sync m16n8k16, fp32 accumulation).
//   * A warp owns 16 weight rows; step = one 64-weight block column. Lane (g, t) decodes
//     words t and t + 4 (codes 8t .. 8t + 7 and 32 + 8t .. 32 + 8t + 7) of the blocks of rows
//     g and g + 8. Pair u of word t (codes 8t + 2u, + 1) is its A operand at k-slots 2t, 2t + 1
//     of the step's MMA u, pair u of word t + 4 at k-slots 2t + 8, 2t + 9: every lane's A
//     comes from its own words, and the 4 MMAs of a step cover the block's 64 columns.
//   * The B operand is then x[g][block + 8t .. + 7] and x[g][block + 32 + 8t .. + 7] in
//     natural order (word u of each 16-byte load for MMA u), read through L1 (every warp
//     of the SM reads the same activations).
//   * The 8 warps of a CTA take every 8th block of the same 16 rows and add up their sums
//     in shared memory at the end.
//   * Software pipeline: a block's metadata is read two steps ahead, its packed words and
//     activations one step ahead.
// A block whose width or offset is inconsistent with the buffer is reported (2002) and
// contributes nothing.
#ifndef WQ_WF_WARPS
#define WQ_WF_WARPS 4                  // warps per CTA (splitting the row group's blocks)
#endif
#ifndef WQ_WF_BPS
#define WQ_WF_BPS 1                    // blocks per warp step (loads issued together)
#endif
constexpr int kWfWarps = WQ_WF_WARPS;
constexpr int kWfBps = WQ_WF_BPS;

struct WfMeta {
    int b[2];            // widths of rows g, g + 8 (0: none)
    uint32_t off[2];
    uint32_t sb[2];
};

template <int NB>
__global__ void __launch_bounds__(32 * kWfWarps)
wf_gemv_kernel(const uint8_t* __restrict__ packed, int64_t packed_bytes, const uint16_t* __restrict__ scale,
               const uint8_t* __restrict__ width, const uint32_t* __restrict__ blk_off, int n, int k,
               const uint16_t* __restrict__ x, int batch, uint16_t* __restrict__ y) {
    __shared__ float red[kWfWarps][NB][4][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int kb = k >> 6;
    const int row[2] = {(int)blockIdx.x * 16 + g, (int)blockIdx.x * 16 + g + 8};
    const uint16_t* xr[2] = {x + (size_t)min(g, batch - 1) * k, x + (size_t)min(g + 8, batch - 1) * k};
    constexpr int STRIDE = kWfWarps * kWfBps;     // blocks between a warp's steps

    auto meta = [&](int blk, WfMeta& m) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            m.b[h] = 0; m.off[h] = 0; m.sb[h] = 0;
            if (blk < kb && row[h] < n) {
                const int64_t i = (int64_t)row[h] * kb + blk;
                m.b[h] = __ldg(width + i);
                m.off[h] = ldg_u32(blk_off + i);
                m.sb[h] = ldg_u16(scale + i);
                if (!wf_block_ok(m.b[h], m.off[h], packed_bytes)) {
                    report(2002);
                    m.b[h] = 0;
                }
            }
        }
    };
    auto words = [&](const WfMeta& m, unsigned long long (&v)[2][2]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int b = m.b[h];
            v[h][0] = b ? wf_bytes(packed, (int64_t)m.off[h] + b * t, b) : 0ull;
            v[h][1] = b ? wf_bytes(packed, (int64_t)m.off[h] + b * (t + 4), b) : 0ull;
        }
    };
    auto acts = [&](int blk, uint4 (&xa)[NB][2]) {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            xa[nb][0] = xa[nb][1] = make_uint4(0, 0, 0, 0);
            if (blk < kb) {
                xa[nb][0] = __ldg(reinterpret_cast<const uint4*>(xr[nb] + blk * 64 + 8 * t));
                xa[nb][1] = __ldg(reinterpret_cast<const uint4*>(xr[nb] + blk * 64 + 32 + 8 * t));
            }
        }
    };

    float acc[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;

    // step = kWfBps blocks kWfWarps apart, starting at block warp; pipeline: a step's
    // metadata two steps ahead, its words and activations one step ahead
    WfMeta m0[kWfBps], m1[kWfBps];
    unsigned long long v0[kWfBps][2][2];
    uint4 x0[kWfBps][NB][2];
#pragma unroll
    for (int q = 0; q < kWfBps; ++q) {
        meta(warp + q * kWfWarps, m0[q]);
        words(m0[q], v0[q]);
        acts(warp + q * kWfWarps, x0[q]);
        meta(warp + q * kWfWarps + STRIDE, m1[q]);
    }
    for (int blk = warp; blk < kb; blk += STRIDE) {
        unsigned long long v1[kWfBps][2][2];
        uint4 x1[kWfBps][NB][2];
        WfMeta m2[kWfBps];
#pragma unroll
        for (int q = 0; q < kWfBps; ++q) {
            words(m1[q], v1[q]);
            acts(blk + q * kWfWarps + STRIDE, x1[q]);
            meta(blk + q * kWfWarps + 2 * STRIDE, m2[q]);
        }
#pragma unroll
        for (int q = 0; q < kWfBps; ++q) {
            // decode rows g, g + 8 (4 bf16 pairs per word), 4 MMAs per 8 batch rows
            uint32_t a[2][2][4];                 // [row][word][pair]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (m0[q].b[h]) {
                        wf_decode8(v0[q][h][w], m0[q].b[h], m0[q].sb[h], a[h][w]);
                    } else {
                        a[h][w][0] = a[h][w][1] = a[h][w][2] = a[h][w][3] = 0u;
                    }
                }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const uint32_t xb0[4] = {x0[q][nb][0].x, x0[q][nb][0].y, x0[q][nb][0].z, x0[q][nb][0].w};
                const uint32_t xb1[4] = {x0[q][nb][1].x, x0[q][nb][1].y, x0[q][nb][1].z, x0[q][nb][1].w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    mma_bf16_16816(acc[nb], a[0][0][u], a[1][0][u], a[0][1][u], a[1][1][u], xb0[u], xb1[u]);
            }
        }
#pragma unroll
        for (int q = 0; q < kWfBps; ++q) {
            m0[q] = m1[q]; m1[q] = m2[q];
#pragma unroll
            for (int h = 0; h < 2; ++h) { v0[q][h][0] = v1[q][h][0]; v0[q][h][1] = v1[q][h][1]; }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) { x0[q][nb][0] = x1[q][nb][0]; x0[q][nb][1] = x1[q][nb][1]; }
        }
    }
    // the CTA's warps add up their K slices; lane (g, t) holds rows g, g + 8 and batch
    // columns 8 nb + 2t, + 1
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp][nb][j][lane] = acc[nb][j];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWfWarps; ++w) v += red[w][nb][j][lane];
            const int r = row[j >> 1], bcol = 8 * nb + 2 * t + (j & 1);
            if (r < n && bcol < batch) y[(size_t)bcol * n + r] = (uint16_t)float_to_bf16_bits(v);
        }
}

// Batches of 1 to 4: y[i, r] = sum_c Wdeq[r, c] x[i, c] with the packed bytes staged in
// shared memory by bulk asynchronous copies, products on the tensor cores (one MMA per
// block column and pair of batch rows, all from the same decoded weights).
//   * A warp owns 4 weight rows. Its blocks come in chunks of 32 block columns: one lane
//     reads each block's offset, width and scale (coalesced), checks them, and writes a
//     16-byte descriptor to shared memory; lanes 0-3 each copy one row's bytes of the chunk,
//     a contiguous run of the bit streams, into shared memory with one cp.async.bulk (from
//     the 16-byte boundary at or below the run's start to the one at or past its end; at
//     the end of the buffer, to the one below, and the run's last 8 bytes by a plain load),
//     completing on the stage's mbarrier. WQ_WF_ST_STAGES stages per warp: while one chunk
//     is decoded the next ones are in flight, with no registers held for them.
//   * One mma.sync m16n8k16 per block column covers the 4 rows x 64 columns: lane (g, t)
//     decodes word t + 4 (g >> 2) (codes 8w .. 8w + 7) of row g & 3's block, its pairs
//     0 and 1 as A row g (quarter g >> 2 of the columns), pairs 2 and 3 as A row g + 8
//     (quarter 2 + (g >> 2)). B column 4 i + q holds activation row i at the columns of
//     quarter q (4 consecutive values per lane: one 8-byte load), so D[rho][4 i + q(rho)]
//     are the useful sums (16 of the 128 outputs) and y[i][row] adds four of them.
// A chunk whose first or end offset is not a multiple of 8, or whose run does not lie inside
// packed_bytes, is not read; inside a run, a block is decoded only when its width is 3..5
// and the next block's offset (or the run's end) lies 8 * width bytes past its own. Both
// are reported (2002) and contribute nothing. An expired wait for a copy is reported as
// 2100.
#ifndef WQ_WF_ST_WARPS
#define WQ_WF_ST_WARPS 1               // warps per CTA (each independent)
#endif
#ifndef WQ_WF_ST_STAGES
#define WQ_WF_ST_STAGES 2              // chunks staged per warp
#endif
constexpr int kStWarps = WQ_WF_ST_WARPS;
constexpr int kStStages = WQ_WF_ST_STAGES;
constexpr int kStRowBytes = 32 * 40 + 32;      // a chunk of 5-bit blocks, the alignment and read slack

struct WfStage {
    alignas(16) uint8_t data[4][kStRowBytes];  // row i's run, from its 16-byte boundary
    uint4 meta[4][33];                         // per block: its descriptor (wf_st_desc); rows one
                                               // entry apart in the banks, so that a column's four
                                               // descriptors load without a bank conflict
};
struct WfWarpSmem {
    WfStage st[kStStages];
    uint4 tbl[3];                              // descriptor words .y (the mask), .z, .w for b = 3, 4, 5
    uint64_t bar[kStStages];
};

// Block descriptor of the staged GEMV (zero for a block that is not decoded):
//   .x  the bf16x2 pair (scale * 4, scale * 4), or, where that pair would not give the exact
//       reconstruction (a scale below 2^-119, from 2^126 on, negative or not finite), the
//       scale's bf16 bits with bit 31 set;
//   .y  the block's byte offset in its row's staged run << 21 | width b << 8 | the mask of
//       the idx_5 fields of a code pair (bits 5 - b .. 4 and 21 - b .. 20);
//   .z  2^(32 - 2b);  .w  2^21 + 2^(5 + b).
__device__ __forceinline__ bool wf_st_pair_scale(uint32_t sb) { return sb >= 0x0400u && sb < 0x7E80u; }

__device__ __forceinline__ uint4 wf_st_desc(uint32_t sb, uint32_t b, uint32_t off) {
    const uint32_t sx = wf_st_pair_scale(sb) ? prmt(sb + 0x0100u, 0u, 0x1010u) : (sb | 0x80000000u);
    const uint32_t mp = (((1u << b) - 1u) << (5 - b)) * 0x00010001u;
    return make_uint4(sx, (off << 21) | (b << 8) | mp, 1u << (32 - 2 * b), (1u << 21) + (1u << (5 + b)));
}

// Shared-memory loads by 32-bit shared address (volatile: they stay after the stage's
// mbarrier wait, which the compiler sees only as an asm with a memory clobber).
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

// One block column of the staged GEMV: the lane decodes word wd (codes 8 wd .. 8 wd + 7) of
// its row's block and issues the column's MMA. The word's b bytes start at byte b wd of the
// block. Pair j (codes 2j, 2j + 1) is the window shifted right by 2jb (a funnel shift, h);
// h * 2^(32 - 2b) keeps just the pair, at the top of the word, and the high half of its
// product with 2^21 + 2^(5 + b) is the pair shifted right by 11 (code 2j + 1 at bits
// 21 - b .. 20) plus the pair shifted right by 27 - b (code 2j at bits 5 - b .. 4): both
// shifts are exact and the two ranges do not overlap, so no carry disturbs the idx_5
// fields, which the mask then isolates. As bf16 numbers the fields are idx_5 * 2^-133;
// times 2^127 minus 1/4 that is (idx_5 - 16) * 2^-6 exactly, and times (scale * 4) it is
// (scale / 16) (idx_5 - 16) rounded once, the reconstruction. FAST: every block of the
// chunk is valid with a pair-form scale, so nothing branches.
template <bool FAST, int NM>
__device__ __forceinline__ void wf_st_step(uint4 d, uint32_t b, uint32_t w0, uint32_t w1, uint32_t sh,
                                           const uint2 (&xv)[NM], float (&acc)[NM][4]) {
    const uint32_t lo = __funnelshift_r(w0, w1, sh), hi = w1 >> sh;
    const uint32_t h[4] = {lo, __funnelshift_r(lo, hi, 2 * b), __funnelshift_r(lo, hi, 4 * b),
                           __funnelshift_r(lo, hi, 6 * b)};
    uint32_t m[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) m[j] = __umulhi(h[j] * d.z, d.w) & d.y & 0x001F001Fu;
    uint32_t o[4];
    if (FAST || (d.x >> 31) == 0u) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = bf16x2_fma(bf16x2_fma(m[j], 0x7F007F00u, 0xBE80BE80u), d.x, 0x80008000u);
    } else {
        const float s16 = bf16_bits_to_float(d.x & 0xFFFFu) * 0.0625f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = pack_bf16x2(s16 * (float)((int)(m[j] & 0xFFFFu) - 16), s16 * (float)((int)(m[j] >> 16) - 16));
    }
    if (!FAST && d.y == 0u) o[0] = o[1] = o[2] = o[3] = 0u;
#pragma unroll
    for (int mi = 0; mi < NM; ++mi) mma_bf16_16816(acc[mi], o[0], o[2], o[1], o[3], xv[mi].x, xv[mi].y);
}

// Four block columns: the shared-memory loads of all four (descriptors, then the words) are
// issued before any is decoded, so that their latencies overlap.
template <bool FAST, int NM>
__device__ __forceinline__ void wf_st_group(uint32_t rowdata, uint32_t meta, uint32_t wd, int nvalid,
                                            const uint2 (&xv)[NM][4], float (&acc)[2][NM][4]) {
    uint4 d[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) d[u] = lds_v4(meta + 16 * u);
    uint32_t b[4], w0[4], w1[4], sh[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        b[u] = FAST ? (d[u].y >> 8) & 7u : max((d[u].y >> 8) & 7u, 3u);     // 0: not decoded
        const uint32_t bw = b[u] * wd;
        const uint32_t wa = rowdata + (d[u].y >> 21) + (bw & ~3u);
        w0[u] = lds_u32(wa);
        w1[u] = lds_u32(wa + 4);
        sh[u] = (bw & 3u) * 8;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (u < nvalid) {
            uint2 xs[NM];
#pragma unroll
            for (int mi = 0; mi < NM; ++mi) xs[mi] = xv[mi][u];
            wf_st_step<FAST, NM>(d[u], b[u], w0[u], w1[u], sh[u], xs, acc[u & 1]);
        }
}

// The block columns J0 .. J0 + nb - 1 of one staged chunk, in groups of 4 whose activation
// pieces were loaded 8 columns ahead (xa: the group at hand, xb: the next); after a group
// is used its registers take the pieces 8 columns further on. FULL: nb == 32.
template <bool FAST, bool FULL, int NM, typename XLoad>
__device__ __forceinline__ void wf_st_chunk(const WfStage& st, int ri, uint32_t wd, int J0, int nb, XLoad& xload4,
                                            uint2 (&xa)[NM][4], uint2 (&xb)[NM][4], float (&acc)[2][NM][4]) {
    const uint32_t rowdata = smem_u32(st.data[ri]);
    const uint32_t meta = smem_u32(st.meta[ri]);
#pragma unroll 1
    for (int jg = 0; jg < 32; jg += 8) {
        if (!FULL && jg >= nb) break;
        wf_st_group<FAST, NM>(rowdata, meta + 16 * jg, wd, FULL ? 4 : nb - jg, xa, acc);
        xload4(J0 + jg + 8, xa);
        wf_st_group<FAST, NM>(rowdata, meta + 16 * (jg + 4), wd, FULL ? 4 : nb - jg - 4, xb, acc);
        xload4(J0 + jg + 12, xb);
    }
}

template <int NB>
__global__ void __launch_bounds__(32 * kStWarps)
wf_gemv_staged_kernel(const uint8_t* __restrict__ packed, int64_t packed_bytes, const uint16_t* __restrict__ scale,
                      const uint8_t* __restrict__ width, const uint32_t* __restrict__ blk_off, int n, int k,
                      const uint16_t* __restrict__ x, int batch, uint16_t* __restrict__ y) {
    __shared__ WfWarpSmem smem[kStWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    WfWarpSmem& S = smem[warp];
    const int g = lane >> 2, t = lane & 3;
    const int row0 = ((int)blockIdx.x * kStWarps + warp) * 4;
    if (row0 >= n) return;                       // the whole warp leaves; warps share nothing
    const int kb = k >> 6, nch = (kb + 31) >> 5;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kStStages; ++s) mbar_init(&S.bar[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (lane < 3) {
        const uint4 d = wf_st_desc(0x3F80u, (uint32_t)lane + 3, 0);
        S.tbl[lane] = make_uint4(0u, d.y & 0x001F001Fu, d.z, d.w);
    }
    __syncwarp();

    // lane l's block of chunk c in each row (offset; scale << 16 | width); lanes 0-3: the
    // offsets of the first block of row `lane`'s chunk and just past its last block
    const uint32_t rb0 = (uint32_t)row0 * (uint32_t)kb;          // n * kb < 2^27
    uint32_t m_off[4], m_wsb[4], m_lo, m_end;
    auto load_meta = [&](int c) {
        const int j = 32 * c + lane;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m_off[i] = 0; m_wsb[i] = 0;
            if (row0 + i < n && j < kb) {
                const uint32_t bi = rb0 + (uint32_t)(i * kb + j);
                m_off[i] = ldg_u32(blk_off + bi);
                m_wsb[i] = (uint32_t)__ldg(width + bi) | (ldg_u16(scale + bi) << 16);
            }
        }
        m_lo = 0; m_end = 0;
        if (lane < 4 && row0 + lane < n) {
            const uint32_t bi = rb0 + (uint32_t)(lane * kb + 32 * c);
            m_lo = ldg_u32(blk_off + bi);
            m_end = ldg_u32(blk_off + bi + min(32, kb - 32 * c));
        }
    };
    // start the copies of chunk c into stage s, check its blocks and write their
    // descriptors; true when some block of the chunk is missing, inconsistent or has a
    // scale without the pair form, so that the chunk takes the general decode
    auto publish = [&](int c, int s) -> bool {
        WfStage& st = S.st[s];
        const int nb = min(32, kb - 32 * c);
        // lanes 0-3: row `lane`'s run [lo, hi) must be whole 8-byte blocks, at least one and
        // at most 32 of them at 5 bits, inside the buffer
        const bool rok = lane < 4 && row0 + lane < n && ((m_lo | m_end) & 7u) == 0 && m_end >= m_lo + 24 &&
                         m_end - m_lo <= 32 * 40 && (int64_t)m_end <= packed_bytes;
        const uint32_t base = m_lo & ~15u;
        // the copy runs to the 16-byte boundary at or past the run's end when that stays
        // inside the buffer (a few bytes of the next run come along), else to the one below
        const uint32_t up = (m_end + 15u) & ~15u;
        const bool whole = (int64_t)up <= packed_bytes;
        const uint32_t bytes = rok ? (whole ? up : m_end & ~15u) - base : 0u;   // >= 16 when sound
        uint32_t tot = bytes;
        tot += __shfl_xor_sync(0xFFFFFFFFu, tot, 1);
        tot += __shfl_xor_sync(0xFFFFFFFFu, tot, 2);
        if (lane == 0) mbar_expect_tx(&S.bar[s], tot);
        if (rok) {
            bulk_load(st.data[lane], packed + base, bytes, &S.bar[s]);
            if (!whole && (m_end & 15u) == 8u)   // the run's last 8 bytes, at the buffer's end
                *reinterpret_cast<unsigned long long*>(st.data[lane] + (m_end - 8 - base)) =
                    ldg_na_u64(reinterpret_cast<const unsigned long long*>(packed + m_end - 8));
        }
        const uint32_t lr = m_lo | (rok ? 1u : 0u);
        bool special = false;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lri = __shfl_sync(0xFFFFFFFFu, lr, i), hi = __shfl_sync(0xFFFFFFFFu, m_end, i);
            const uint32_t lo = lri & ~1u, off = m_off[i], b = m_wsb[i] & 0xFFu, sb = m_wsb[i] >> 16;
            uint32_t nxt = __shfl_down_sync(0xFFFFFFFFu, off, 1);
            if (lane == nb - 1) nxt = hi;
            // a decodable block: inside the run, 8-byte aligned, b in 3..5, and followed by
            // the next block (or the run's end) exactly 8 b bytes later
            const bool ok = (lri & 1u) && lane < nb && b - 3u <= 2u && (off & 7u) == 0 && off >= lo &&
                            nxt <= hi && nxt - off == 8 * b;
            const bool rv = row0 + i < n;
            if (rv && lane < nb && !ok) report(2002);
            const uint4 tb = S.tbl[ok ? b - 3 : 0];
            uint4 d = make_uint4(0u, 0u, 0u, 0u);
            if (ok) {
                d.x = wf_st_pair_scale(sb) ? prmt(sb + 0x0100u, 0u, 0x1010u) : (sb | 0x80000000u);
                d.y = ((off - (lo & ~15u)) << 21) | (b << 8) | tb.y;
                d.z = tb.z;
                d.w = tb.w;
            }
            st.meta[i][lane] = d;
            special |= !rv || (lane < nb && !(ok && wf_st_pair_scale(sb)));
        }
        return __any_sync(0xFFFFFFFFu, special);
    };

    // this lane's activation columns: in MMA mi, row 2 mi + (g >> 2) (row 0 at batch 1),
    // quarter q = g & 3 of each block column
    constexpr int NM = (NB + 1) / 2;             // MMAs per block column (2 batch rows each)
    const int q = g & 3;
    const uint16_t* xl[NM];
#pragma unroll
    for (int mi = 0; mi < NM; ++mi) {
        const int bi = min(NB == 1 ? 0 : 2 * mi + (g >> 2), batch - 1);
        xl[mi] = x + (size_t)bi * k + 32 * (q & 1) + 8 * t + 4 * (q >> 1);
    }
    const int ri = g & 3;
    const uint32_t wd = (uint32_t)(t + 4 * (g >> 2));   // decoded row and word
    // the activation pieces of steps J .. J + 3 (J: block column; past the row's end a
    // repeated in-bounds load whose value is not used)
    auto xload4 = [&](int J, uint2 (&xr)[NM][4]) {
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) {
            if (J + 3 < kb) {
                const uint2* p = reinterpret_cast<const uint2*>(xl[mi] + (size_t)J * 64);
#pragma unroll
                for (int u = 0; u < 4; ++u) xr[mi][u] = __ldg(p + 16 * u);
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    xr[mi][u] = __ldg(reinterpret_cast<const uint2*>(xl[mi] + (size_t)min(J + u, kb - 1) * 64));
            }
        }
    };

    float acc[2][NM][4];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int mi = 0; mi < NM; ++mi) acc[e][mi][0] = acc[e][mi][1] = acc[e][mi][2] = acc[e][mi][3] = 0.f;
    uint2 xa[NM][4], xb[NM][4];                  // steps 8 apart: the next two groups of 4
    xload4(0, xa);
    xload4(4, xb);
    uint32_t slow = 0;                           // bit s: stage s holds a chunk for the general loop
    bool dead = false;
    load_meta(0);
    for (int p = 0; p < kStStages - 1 && p < nch; ++p) {
        slow |= (uint32_t)publish(p, p) << p;
        if (p + 1 < nch) load_meta(p + 1);
    }
    int c = 0;
    for (; c < nch; ++c) {
        const int pc = c + kStStages - 1;
        if (pc < nch) {
            const int ps = pc % kStStages;
            slow = (slow & ~(1u << ps)) | ((uint32_t)publish(pc, ps) << ps);
            if (pc + 1 < nch) load_meta(pc + 1);
        }
        const int s = c % kStStages;
        if (!mbar_wait(&S.bar[s], (uint32_t)(c / kStStages) & 1u)) {
            report(2100);
            dead = true;
            break;
        }
        __syncwarp();                            // the descriptors and tail bytes other lanes wrote
        const WfStage& st = S.st[s];
        const int nb = min(32, kb - 32 * c);
        if (nb == 32 && !((slow >> s) & 1u))
            wf_st_chunk<true, true, NM>(st, ri, wd, 32 * c, 32, xload4, xa, xb, acc);
        else if (nb == 32)
            wf_st_chunk<false, true, NM>(st, ri, wd, 32 * c, 32, xload4, xa, xb, acc);
        else
            wf_st_chunk<false, false, NM>(st, ri, wd, 32 * c, nb, xload4, xa, xb, acc);
        __syncwarp();                            // stage s is refilled next
    }
    if (dead) {
        // chunks c .. c + stages - 1 were started: give their copies (again a bounded wait)
        // the chance to land before the warp's shared memory goes away
        for (int d = c; d < nch && d < c + kStStages; ++d)
            mbar_wait(&S.bar[d % kStStages], (uint32_t)(d / kStStages) & 1u);
        return;
    }
#pragma unroll
    for (int mi = 0; mi < NM; ++mi) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][mi][e] += acc[1][mi][e];
        // lane (g, t): t even holds the quarter-0/1 sums, t odd the quarter-2/3 sums of the
        // MMA's batch row t >> 1
        const float* a = acc[0][mi];
        float v = (t & 1) ? (g < 4 ? a[2] : a[3]) : (g < 4 ? a[0] : a[1]);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 16);
        const int ob = 2 * mi + (t >> 1);
        if (g < 4 && !(t & 1) && ob < NB && ob < batch && row0 + g < n)
            y[(size_t)ob * n + row0 + g] = (uint16_t)float_to_bf16_bits(v);
    }
}

int grid_cap(int64_t want) {
    const int64_t cap = (int64_t)sm_count() * 8;
    if (want > cap) want = cap;
    return (int)(want < 1 ? 1 : want);
}

}  // namespace

wq_status launch_wf_analyze(const uint16_t* w, int64_t n, int64_t k, double lambda, uint16_t* scale,
                            uint8_t* width, uint32_t* blk_off, double* dist, cudaStream_t s) {
    const int64_t nblk = n * k / 64;
    const int64_t ntiles = (nblk + kScanTile - 1) / kScanTile;
    wf_analyze_kernel<<<grid_cap(ntiles), kThreads, 0, s>>>((const uint4*)w, nblk, 64.0 * lambda, scale,
                                                            width, blk_off, dist);
    wq_status st = check_launch("wf analyze");
    if (st) return st;
    return launch_tile_scan_u8(blk_off, nblk, s);
}

wq_status launch_wf_pack(const uint16_t* w, int64_t n, int64_t k, const uint16_t* scale,
                         const uint8_t* width, const uint32_t* blk_off, uint8_t* packed,
                         int64_t packed_bytes, cudaStream_t s) {
    const int64_t nblk = n * k / 64;
    wf_pack_kernel<<<grid_cap((nblk + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        (const uint4*)w, nblk, scale, width, blk_off, packed, packed_bytes);
    return check_launch("wf pack");
}

wq_status launch_wf_dequant(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                            const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                            uint16_t* out, cudaStream_t s) {
    const int64_t nblk = n * k / 64;
    wf_dequant_kernel<<<grid_cap((nblk * 8 + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        packed, packed_bytes, scale, width, blk_off, nblk, (uint4*)out);
    return check_launch("wf dequant");
}

// Batches of 1 to 4 take the staged kernel, larger ones the 16-row one (8192 x 28672 at
// 4.5 bits per weight: the staged kernel runs batch 1 and 2 in about 97 us, the 16-row one
// batches 3 to 16 in 245-256 us: it reads each block's width, offset and scale at 16
// different rows per warp step, scattered over many cache lines, with no staging).
wq_status launch_wf_gemv(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                         const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                         const uint16_t* x, int batch, uint16_t* y, cudaStream_t s) {
    if (batch <= 4) {
        const unsigned sgrid = (unsigned)((n + 4 * kStWarps - 1) / (4 * kStWarps));
        if (batch == 1)
            wf_gemv_staged_kernel<1><<<sgrid, 32 * kStWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off,
                                                                    (int)n, (int)k, x, batch, y);
        else if (batch == 2)
            wf_gemv_staged_kernel<2><<<sgrid, 32 * kStWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off,
                                                                    (int)n, (int)k, x, batch, y);
        else
            wf_gemv_staged_kernel<4><<<sgrid, 32 * kStWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off,
                                                                    (int)n, (int)k, x, batch, y);
        return check_launch("wf gemv");
    }
    const unsigned grid = (unsigned)((n + 15) / 16);
    if (batch <= 8)
        wf_gemv_kernel<1><<<grid, 32 * kWfWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off, (int)n,
                                                         (int)k, x, batch, y);
    else
        wf_gemv_kernel<2><<<grid, 32 * kWfWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off, (int)n,
                                                         (int)k, x, batch, y);
    return check_launch("wf gemv");
}

wq_status read_wf_error(int32_t* code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_wf_error, sizeof v);
    if (e != cudaSuccess) return fail(WQ_ECUDA, "reading the water-filling error word: %s", cudaGetErrorString(e));
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_wf_error, &zero, sizeof zero);
    }
    *code = v;
    return WQ_OK;
}

}  // namespace wq
