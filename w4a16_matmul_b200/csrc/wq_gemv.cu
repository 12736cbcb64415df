// wq_gemv.cu -- W4A16 GEMV for decode: y[b, r] = sum_c Wdeq[r, c] x[b, c], b < batch <= 16.
//
// Reconstruction follows "MiniCPM5-1B 验证: 6× 压缩…" §2.2/§2.5 (dyadic: bf16(step*(idx-8)))
// and "K-Means量化技术…" §2.2 (LUT16: a 16-entry centroid table per block of 64), fused into
// the product instead of written out as a dense matrix.
//
// Design (HBM-bound: 0.53 B per dyadic weight, 1 B per LUT16 weight):
//   * One CTA owns 8*R rows of one problem and the whole K range; its W warps split K
//     into 256-column steps (warp w takes steps w, w+W, ...). The partial sums meet in
//     shared memory at the end: one launch, no workspace.
//   * Lane (g = lane/4, t = lane%4) streams, per row block, 32 contiguous bytes of row g
//     (64 codes: one dyadic g64 group, two g32 groups, or one LUT16 block) with two
//     128-bit non-allocating loads; a quad of lanes covers 128 contiguous bytes of a row.
//   * The product runs on the warp-level tensor-core path (mma m16n8k16, fp32 accumulate):
//     the reconstructed weights are the B operand (8 rows), the activations the A operand
//     (16 batch rows; rows >= batch are zero). At batch 1..16 this keeps the per-weight
//     instruction count at the nibble-to-bf16 conversion, which CUDA-core FMAs could not.
//   * Dyadic reconstruction is exact: a nibble pair is OR-ed into the mantissa of the bf16
//     value 128 (giving 128 + idx, exact), minus 136 (exact), times step in one bf16 FMA
//     (one rounding, to nearest even) -- the same bits wq_dequant writes.
//   * The k order inside one mma is a permutation of the physical columns (word nibbles
//     pair up as (0,4), (1,5), (2,6), (3,7)); the activation fragment is permuted the same
//     way with byte permutes, so the contraction is unchanged.
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kMaxProblems = WQ_GEMV_MAX_GROUPED;

template <int MAXP>
struct GemvParams {
    int count;
    int batch;
    int tile_start[MAXP + 1];     // prefix sum of row tiles per problem
    GemvProblem prob[MAXP];
};

// bf16 pairs of the 8 codes of one packed word, dyadic: pair j = (code j, code j+4),
// element with the lower code index in the low half.
__device__ __forceinline__ void dyadic_pairs(uint32_t w, uint32_t step2, uint32_t (&p)[4]) {
    const uint32_t kMagic = 0x43004300u;      // bf16 128.0 twice
    const uint32_t kNeg136 = 0xC308C308u;     // bf16 -136.0 twice
    const uint32_t kOne = 0x3F803F80u;        // bf16 1.0 twice
    const uint32_t kNegZero = 0x80008000u;    // -0.0: keeps bf16(0 * -8) = -0.0
    p[0] = (w & 0x000F000Fu) | kMagic;
    p[1] = ((w >> 4) & 0x000F000Fu) | kMagic;
    p[2] = ((w >> 8) & 0x000F000Fu) | kMagic;
    p[3] = ((w >> 12) & 0x000F000Fu) | kMagic;
#pragma unroll
    for (int j = 0; j < 4; ++j) p[j] = bf16x2_fma(bf16x2_fma(p[j], kOne, kNeg136), step2, kNegZero);
}

// Same pairs computed in fp32 for tiny scales (step would lose bits as a bf16).
__device__ __forceinline__ void dyadic_pairs_tiny(uint32_t w, float step, uint32_t (&p)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = step * (float)((int)((w >> (4 * j)) & 15) - 8);
        const float hi = step * (float)((int)((w >> (4 * j + 16)) & 15) - 8);
        p[j] = pack_bf16x2(lo, hi);
    }
}

// step = scale / 8 as a bf16 pair (exact for scale >= 2^-123).
__device__ __forceinline__ uint32_t step_pair(uint32_t scale_bits) {
    return bf16x2_fma(scale_bits | (scale_bits << 16), 0x3E003E00u, 0x80008000u);
}

// LUT16 lookup of 4 codes (nibbles of the low 16 bits of s) in a 16-entry fp16 table held
// as byte planes: lo[q] / hi[q] hold the low / high bytes of entries 4q..4q+3. Returns the
// fp16 pairs (code0, code1) and (code2, code3).
__device__ __forceinline__ void lut16_lookup4(uint32_t s, const uint32_t (&lo)[4],
                                              const uint32_t (&hi)[4], uint32_t& p01,
                                              uint32_t& p23) {
    const uint32_t s7 = s & 0x7777u;                                  // index within 8 entries
    const uint32_t m = prmt(0x00000000u, 0xFFFFFFFFu, (s >> 1) & 0x4444u);   // byte mask: code >= 8
    const uint32_t l = (prmt(lo[0], lo[1], s7) & ~m) | (prmt(lo[2], lo[3], s7) & m);
    const uint32_t h = (prmt(hi[0], hi[1], s7) & ~m) | (prmt(hi[2], hi[3], s7) & m);
    p01 = prmt(l, h, 0x5140u);
    p23 = prmt(l, h, 0x7362u);
}

// bf16x2 -> fp16x2 (round to nearest even; exact for |x| in [2^-14, 65504]).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
    const float lo = __uint_as_float(v << 16), hi = __uint_as_float(v & 0xFFFF0000u);
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

enum Kind { kDyadic64 = 0, kDyadic32 = 1, kLut16 = 2 };

template <int KIND, bool BIG, int R, int W, int MAXP>
__global__ void __launch_bounds__(W * 32)
gemv_kernel(const __grid_constant__ GemvParams<MAXP> prm) {
    // ---- which problem / row tile ------------------------------------------------------
    int p = 0;
    if (MAXP > 1) {
        int lo = 0, hi = prm.count - 1;
        while (lo < hi) {                      // last p with tile_start[p] <= blockIdx.x
            const int mid = (lo + hi + 1) >> 1;
            if (prm.tile_start[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
        }
        p = lo;
    }
    const GemvProblem& pb = prm.prob[p];
    const int N = pb.n, K = pb.k, B = prm.batch;
    const int row0 = ((int)blockIdx.x - prm.tile_start[p]) * (8 * R);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int steps = (K + 255) >> 8;
    const size_t row_bytes = (size_t)K / 2;

    float acc[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r][0] = acc[r][1] = acc[r][2] = acc[r][3] = 0.f;

    const uint16_t* xg = pb.x + (size_t)g * K;
    const uint16_t* xg8 = pb.x + (size_t)(g + 8) * K;
    const bool xa_live = g < B, xb_live = BIG && (g + 8 < B);

    for (int s = warp; s < steps; s += W) {
        const int kk = s * 256 + t * 64;                 // first column of this lane's chunk
        const bool h0 = kk < K, h1 = kk + 32 < K;        // the two 32-column halves
        // ---- weights and per-group parameters of R rows -----------------------------
        uint32_t wv[R][8];
        uint32_t aux[R][8];                              // dyadic: steps; LUT16: byte planes
        bool tiny[R];
        float tiny_step[R][2];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int row = row0 + 8 * r + g;
            const bool rl = row < N;
            const uint8_t* wp = pb.packed + (size_t)row * row_bytes + kk / 2;
            uint4 a = (rl && h0) ? ldg_nc_v4(wp) : make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
            uint4 b = (rl && h1) ? ldg_nc_v4(wp + 16) : make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
            wv[r][0] = a.x; wv[r][1] = a.y; wv[r][2] = a.z; wv[r][3] = a.w;
            wv[r][4] = b.x; wv[r][5] = b.y; wv[r][6] = b.z; wv[r][7] = b.w;
            tiny[r] = false;
            if (KIND == kLut16) {
                uint4 la = make_uint4(0, 0, 0, 0), lb = la;
                if (rl && h0) {
                    const uint4* lp = (const uint4*)((const uint16_t*)pb.aux + ((size_t)row * (K / 64) + kk / 64) * 16);
                    la = ldg_nc_v4(lp);
                    lb = ldg_nc_v4(lp + 1);
                }
                // byte planes: entries 4q..4q+3 live in words 2q (entries 4q, 4q+1) and 2q+1
                aux[r][0] = prmt(la.x, la.y, 0x6420u); aux[r][4] = prmt(la.x, la.y, 0x7531u);
                aux[r][1] = prmt(la.z, la.w, 0x6420u); aux[r][5] = prmt(la.z, la.w, 0x7531u);
                aux[r][2] = prmt(lb.x, lb.y, 0x6420u); aux[r][6] = prmt(lb.x, lb.y, 0x7531u);
                aux[r][3] = prmt(lb.z, lb.w, 0x6420u); aux[r][7] = prmt(lb.z, lb.w, 0x7531u);
            } else {
                const uint16_t* sp = (const uint16_t*)pb.aux;
                uint32_t s0 = 0, s1 = 0;
                if (KIND == kDyadic64) {
                    if (rl && h0) s0 = ldg_u16(sp + (size_t)row * (K / 64) + kk / 64);
                    s1 = s0;
                } else {
                    if (rl && h0) s0 = ldg_u16(sp + (size_t)row * (K / 32) + kk / 32);
                    if (rl && h1) s1 = ldg_u16(sp + (size_t)row * (K / 32) + kk / 32 + 1);
                }
                const float f0 = bf16_bits_to_float(s0), f1 = bf16_bits_to_float(s1);
                tiny[r] = (f0 != 0.f && f0 < 0x1p-100f) || (f1 != 0.f && f1 < 0x1p-100f);
                tiny_step[r][0] = f0 * 0.125f;
                tiny_step[r][1] = f1 * 0.125f;
                aux[r][0] = step_pair(s0);
                aux[r][1] = step_pair(s1);
            }
        }
        // ---- the 8 words of the chunk: 2 mma per word per row block ---------------------
#pragma unroll
        for (int sub = 0; sub < 8; ++sub) {
            const int kx = kk + 8 * sub;
            const bool xv = (sub < 4) ? h0 : h1;
            uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
            if (xa_live && xv) xa = ldg_v4(xg + kx);
            if (BIG && xb_live && xv) xb = ldg_v4(xg8 + kx);
            uint32_t a0, a1, a2, a3, a4, a5, a6, a7;     // A fragments of the two mma
            if (KIND == kLut16) {
                // natural pairs (k0,k1), (k2,k3) | (k4,k5), (k6,k7), converted to fp16
                a0 = bf16x2_to_f16x2(xa.x); a2 = bf16x2_to_f16x2(xa.y);
                a4 = bf16x2_to_f16x2(xa.z); a6 = bf16x2_to_f16x2(xa.w);
                if (BIG) {
                    a1 = bf16x2_to_f16x2(xb.x); a3 = bf16x2_to_f16x2(xb.y);
                    a5 = bf16x2_to_f16x2(xb.z); a7 = bf16x2_to_f16x2(xb.w);
                } else {
                    a1 = a3 = a5 = a7 = 0;
                }
            } else {
                // pairs (k0,k4), (k1,k5) | (k2,k6), (k3,k7)
                a0 = prmt(xa.x, xa.z, 0x5410u); a2 = prmt(xa.x, xa.z, 0x7632u);
                a4 = prmt(xa.y, xa.w, 0x5410u); a6 = prmt(xa.y, xa.w, 0x7632u);
                if (BIG) {
                    a1 = prmt(xb.x, xb.z, 0x5410u); a3 = prmt(xb.x, xb.z, 0x7632u);
                    a5 = prmt(xb.y, xb.w, 0x5410u); a7 = prmt(xb.y, xb.w, 0x7632u);
                } else {
                    a1 = a3 = a5 = a7 = 0;
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                uint32_t q[4];
                if (KIND == kLut16) {
                    const uint32_t lo[4] = {aux[r][0], aux[r][1], aux[r][2], aux[r][3]};
                    const uint32_t hi[4] = {aux[r][4], aux[r][5], aux[r][6], aux[r][7]};
                    lut16_lookup4(wv[r][sub], lo, hi, q[0], q[1]);
                    lut16_lookup4(wv[r][sub] >> 16, lo, hi, q[2], q[3]);
                    mma_f16_16816(acc[r], a0, a1, a2, a3, q[0], q[1]);
                    mma_f16_16816(acc[r], a4, a5, a6, a7, q[2], q[3]);
                } else {
                    const int hsel = (KIND == kDyadic32 && sub >= 4) ? 1 : 0;
                    if (__builtin_expect(tiny[r], 0))
                        dyadic_pairs_tiny(wv[r][sub], tiny_step[r][hsel], q);
                    else
                        dyadic_pairs(wv[r][sub], aux[r][hsel], q);
                    mma_bf16_16816(acc[r], a0, a1, a2, a3, q[0], q[1]);
                    mma_bf16_16816(acc[r], a4, a5, a6, a7, q[2], q[3]);
                }
            }
        }
    }

    // ---- reduce the W warps' partial sums, write bf16 ----------------------------------
    __shared__ float red[W][R][4][32];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp][r][j][lane] = acc[r][j];
    __syncthreads();
    for (int e = threadIdx.x; e < R * 4 * 32; e += W * 32) {
        const int r = e / 128, j = (e / 32) % 4, ln = e % 32;
        float v = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < W; ++w2) v += red[w2][r][j][ln];
        // fragment (lane ln, element j): batch = ln/4 (+8 for j >= 2), row = 2*(ln%4) + (j&1)
        const int b = (ln >> 2) + ((j >> 1) << 3);
        const int row = row0 + 8 * r + 2 * (ln & 3) + (j & 1);
        if (b < B && row < N) pb.y[(size_t)b * N + row] = (uint16_t)float_to_bf16_bits(v);
    }
}

template <int KIND, bool BIG, int R, int W, int MAXP>
wq_status run(const GemvParams<MAXP>& prm, int tiles, cudaStream_t s) {
    gemv_kernel<KIND, BIG, R, W, MAXP><<<tiles, W * 32, 0, s>>>(prm);
    return check_launch("gemv");
}

template <int KIND, int MAXP>
wq_status dispatch(const GemvParams<MAXP>& prm, int tiles_r1, int tiles_r2, bool big, bool use_r2,
                   cudaStream_t s) {
    if (big) {
        if (use_r2) return run<KIND, true, 2, 8, MAXP>(prm, tiles_r2, s);
        return run<KIND, true, 1, 8, MAXP>(prm, tiles_r1, s);
    }
    if (use_r2) return run<KIND, false, 2, 8, MAXP>(prm, tiles_r2, s);
    return run<KIND, false, 1, 8, MAXP>(prm, tiles_r1, s);
}

template <int MAXP>
wq_status launch_impl(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    // Row tile: 8 rows per CTA while that still gives at least two CTAs per SM over the
    // whole launch, 16 rows otherwise (fewer, longer CTAs; activations reused twice).
    GemvParams<MAXP> local;
    local.count = count;
    local.batch = batch;
    int64_t rows_total = 0;
    for (int i = 0; i < count; ++i) { local.prob[i] = probs[i]; rows_total += probs[i].n; }
    const bool use_r2 = rows_total / 8 > 4LL * sm_count();
    const int rt = use_r2 ? 16 : 8;
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        local.tile_start[i] = tiles;
        tiles += (probs[i].n + rt - 1) / rt;
    }
    local.tile_start[count] = tiles;
    const bool big = batch > 8;
    const int kind = (fmt == WQ_FMT_LUT16) ? kLut16 : (group == 64 ? kDyadic64 : kDyadic32);
    if (kind == kLut16) return dispatch<kLut16, MAXP>(local, tiles, tiles, big, use_r2, s);
    if (kind == kDyadic64) return dispatch<kDyadic64, MAXP>(local, tiles, tiles, big, use_r2, s);
    return dispatch<kDyadic32, MAXP>(local, tiles, tiles, big, use_r2, s);
}

}  // namespace

wq_status launch_gemv(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    if (count == 1) return launch_impl<1>(fmt, group, probs, count, batch, s);
    return launch_impl<kMaxProblems>(fmt, group, probs, count, batch, s);
}

}  // namespace wq
