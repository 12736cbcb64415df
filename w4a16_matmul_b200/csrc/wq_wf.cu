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
// block's 128 output bytes leave in one coalesced run), and a GEMV that rebuilds the
// weights the same way and multiplies them in fp32 (the format's decode-side consumer).
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

// bf16((scale / 16) * (idx_5 - 16)) of the 8 codes of b bits in v (code j in bits b j ..),
// as bf16 pairs in column order; sb = the block's bf16 scale bits.
// Each code is brought to bits 5 - b .. 4, where its value is idx_5 = code << (5 - b), by one
// 32-bit funnel shift of the 40 bits (the bits below it hold its neighbour and are masked
// off); a pair of codes is joined into the two halves of one word by a byte permute.
__device__ __forceinline__ void wf_decode8(unsigned long long v, int bw, uint32_t sb, uint32_t (&o)[4]) {
    const uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    const int s5 = 5 - bw;
    const uint32_t mp = (((1u << bw) - 1u) * 0x00010001u) << s5;      // idx_5 fields of a pair
    uint32_t m[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // code 2j starts at bit 2 j b, code 2j + 1 at (2j + 1) b; shifted right by that minus
        // s5 (>= 0 but for code 0, which is shifted left; < 32 but for code 7 at b = 5, bit 35)
        const uint32_t c0 = j == 0 ? lo << s5 : __funnelshift_r(lo, hi, 2 * j * bw - s5);
        const uint32_t c1 = (j == 3 && bw == 5) ? hi >> 3 : __funnelshift_r(lo, hi, (2 * j + 1) * bw - s5);
        m[j] = prmt(c0, c1, 0x5410u) & mp;                               // (idx_5 of 2j, of 2j + 1)
    }
    if ((sb & 0x7FFFu) >= 0x0400u) {
        // scale >= 2^-119: every nonzero (scale / 16) (idx_5 - 16) is a normal bf16.
        // idx_5 | 0x4300 is the bf16 number 128 + idx_5, minus 144 is idx_5 - 16 exactly, and
        // one bf16x2 multiply by scale / 16 (the exponent field minus 4) rounds the product
        // once, as the definition reads.
        const uint32_t s16x2 = prmt(sb - 0x0200u, 0u, 0x1010u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t d = bf16x2_fma(m[j] | 0x43004300u, 0x3F803F80u, 0xC310C310u);   // idx_5 - 16
            o[j] = bf16x2_fma(d, s16x2, 0x80008000u);
        }
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
// Small batches: y[i, r] = sum_c Wdeq[r, c] x[i, c] for NB <= 8 activation
// rows on the CUDA cores, Wdeq rebuilt exactly as wf_dequant_kernel does (bf16), products and sums in fp32.
// One warp per weight row; 8 lanes per 64-weight block (lane t: columns 8t .. 8t + 7, the b
// bytes at the block's offset + b t), 4 blocks per step, 8 steps per chunk of 32 blocks.
// A chunk's widths, offsets and scales are read one block per lane, checked, and handed to
// the decoding lanes by shuffles. Software pipeline: the metadata is read two chunks
// ahead and the packed words one chunk ahead, so that a chunk's loads are in flight while
// the previous chunk is decoded. A block whose width or offset is inconsistent with the
// buffer is reported and contributes nothing.
constexpr int kFmaWarps = 8;

// One chunk's packed words and, per step, the block width (0: nothing) and scale bits.
struct WfChunk {
    unsigned long long v[8];
    uint32_t wpk;                    // width of step j in bits 4j .. 4j + 3
    uint32_t spk[4];                 // scale bits of steps 2i (low half) and 2i + 1 (high half)
};

template <int NB>
__global__ void __launch_bounds__(32 * kFmaWarps)
wf_gemv_fma_kernel(const uint8_t* __restrict__ packed, int64_t packed_bytes, const uint16_t* __restrict__ scale,
               const uint8_t* __restrict__ width, const uint32_t* __restrict__ blk_off, int n, int k,
               const uint16_t* __restrict__ x, uint16_t* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kFmaWarps + (threadIdx.x >> 5);
    if (row >= n) return;                        // the whole warp leaves; no CTA-wide barrier
    const int kb = k >> 6;
    const int nch = (kb + 31) >> 5;
    const int64_t rb = (int64_t)row * kb;
    const int t = lane & 7, sub = lane >> 3;

    // this lane's block of chunk c: width (0 past the row's end), offset, scale bits
    auto meta = [&](int c, int& bw, uint32_t& off, uint32_t& sb) {
        const int bi = 32 * c + lane;
        bw = 0; off = 0; sb = 0;
        if (bi < kb) {
            bw = __ldg(width + rb + bi);
            off = ldg_u32(blk_off + rb + bi);
            sb = ldg_u16(scale + rb + bi);
        }
    };
    // check the lane's block, then issue the chunk's packed loads (the whole warp takes part)
    auto fetch = [&](int c, int bw, uint32_t off, uint32_t sb, WfChunk& ch) {
        if (32 * c + lane < kb && !wf_block_ok(bw, off, packed_bytes)) {
            report(2002);
            bw = 0;
        }
        ch.wpk = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int blk = 4 * j + sub;
            const int b = __shfl_sync(0xFFFFFFFFu, bw, blk);
            const uint32_t o = __shfl_sync(0xFFFFFFFFu, off, blk);
            const uint32_t sj = __shfl_sync(0xFFFFFFFFu, sb, blk);
            ch.wpk |= (uint32_t)b << (4 * j);
            if (j & 1) ch.spk[j >> 1] |= sj << 16; else ch.spk[j >> 1] = sj;
            ch.v[j] = b ? wf_bytes(packed, (int64_t)o + b * t, b) : 0ull;
        }
    };

    float2 acc[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) acc[i] = make_float2(0.f, 0.f);

    WfChunk cur;
    int bw;
    uint32_t off, sb;
    meta(0, bw, off, sb);
    fetch(0, bw, off, sb, cur);
    if (nch > 1) meta(1, bw, off, sb);
    for (int c = 0; c < nch; ++c) {
        WfChunk nxt;
        if (c + 1 < nch) {                       // uniform across the warp
            fetch(c + 1, bw, off, sb, nxt);
            if (c + 2 < nch) meta(c + 2, bw, off, sb);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int b = (int)(cur.wpk >> (4 * j)) & 15;
            if (b == 0) continue;
            const uint32_t sj = (j & 1) ? cur.spk[j >> 1] >> 16 : cur.spk[j >> 1] & 0xFFFFu;
            uint32_t o[4];
            wf_decode8(cur.v[j], b, sj, o);
            const int col = (32 * c + 4 * j + sub) * 64 + 8 * t;
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                // cached in L1: every warp of the SM reads the same activations
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)i * k + col));
                const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 w2 = make_float2(__uint_as_float(o[q] << 16), __uint_as_float(o[q] & 0xFFFF0000u));
                    const float2 x2 = make_float2(__uint_as_float(xs[q] << 16), __uint_as_float(xs[q] & 0xFFFF0000u));
                    acc[i] = __ffma2_rn(w2, x2, acc[i]);
                }
            }
        }
        if (c + 1 < nch) cur = nxt;
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        float r = acc[i].x + acc[i].y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xFFFFFFFFu, r, o);
        if (lane == 0) y[(size_t)i * n + row] = (uint16_t)float_to_bf16_bits(r);
    }
}

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

// Batch 1 takes the CUDA-core kernel, larger batches the tensor-core one (measured on
// 8192 x 28672 at 4.5 bits per weight: 189 us against 245 us at batch 1; from batch 2 the
// tensor-core kernel runs one pass in 245-256 us where the CUDA-core one takes 262 us at
// batch 2, 435 us at 8 and two passes, 896 us, at 16). The tensor-core kernel reads each
// block's width, offset and scale at 16 different rows per warp step, scattered over many
// cache lines, which is what holds it at about 0.65 TB/s.
#ifndef WQ_WF_FMA_MAX
#define WQ_WF_FMA_MAX 1                // largest batch the CUDA-core kernel takes
#endif

wq_status launch_wf_gemv(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                         const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                         const uint16_t* x, int batch, uint16_t* y, cudaStream_t s) {
    if (batch <= WQ_WF_FMA_MAX) {
        const unsigned grid = (unsigned)((n + kFmaWarps - 1) / kFmaWarps);
#define WQ_WF_FMA(NBV)                                                                                    \
    wf_gemv_fma_kernel<NBV><<<grid, 32 * kFmaWarps, 0, s>>>(packed, packed_bytes, scale, width, blk_off, \
                                                            (int)n, (int)k, x, y)
        switch (batch) {
            case 1: WQ_WF_FMA(1); break;
            case 2: WQ_WF_FMA(2); break;
            case 3: WQ_WF_FMA(3); break;
            case 4: WQ_WF_FMA(4); break;
            case 5: WQ_WF_FMA(5); break;
            case 6: WQ_WF_FMA(6); break;
            case 7: WQ_WF_FMA(7); break;
            default: WQ_WF_FMA(8); break;
        }
#undef WQ_WF_FMA
        return check_launch("wf gemv");
    }
    static_assert(WQ_WF_FMA_MAX <= 8, "the CUDA-core kernel takes at most 8 activation rows");
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
