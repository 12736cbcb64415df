// wq_gemv.cu -- W4A16 GEMV for decode: y[b, r] = sum_c Wdeq[r, c] x[b, c], b < batch <= 16.
//
// Reconstruction follows "MiniCPM5-1B 验证: 6× 压缩…" §2.2/§2.5 (dyadic: bf16(step*(idx-8)))
// and "K-Means量化技术…" §2.2 (LUT16: a 16-entry centroid table per block of 64), fused into
// the product instead of written out as a dense matrix.
//
// Design (HBM-bound: 0.53 B per dyadic weight, 1 B per LUT16 weight; the limit to beat is
// the instruction issue rate of the in-register reconstruction):
//   * A warp owns 16*R rows of one problem. Lane (g = lane/4, t = lane%4) streams rows g
//     and g+8 of every 16-row block: per 256-column step, 32 contiguous bytes of each
//     (64 codes: one dyadic g64 group, two g32 groups, or one LUT16 block) with two
//     128-bit non-allocating loads; a quad of lanes covers 128 contiguous bytes of a row.
//     The next step's bytes are loaded while the current step computes.
//   * The product runs on the warp-level tensor-core path (mma m16n8k16, fp32
//     accumulate): the reconstructed weights are the A operand (16 rows x 16 columns, no
//     padding), the activations the B operand (batch columns 0..7, and 8..15 in a second
//     mma when batch > 8). Issuing one mma per 256 weights keeps the per-weight cost at
//     the nibble-to-bf16 conversion, which CUDA-core FMAs could not match at batch > 1.
//   * Dyadic reconstruction is exact: a nibble pair is OR-ed into the mantissa of the bf16
//     value 128 (giving 128 + idx, exact), minus 136 (exact), times step in one bf16 FMA
//     (one rounding, to nearest even) -- the same bits wq_dequant writes. Groups whose
//     scale is below 2^-100 (step not representable as a normal bf16) take an fp32 path.
//   * The k order inside one mma is a permutation of the physical columns (word nibbles
//     pair up as (0,4), (1,5), (2,6), (3,7)); the activation fragment is permuted the same
//     way with byte permutes, so the contraction is unchanged.
//   * When a launch has too few rows to fill the GPU, WK warps of a CTA split K and meet
//     in shared memory at the end; otherwise every warp covers the full K and no
//     reduction exists. One launch, no workspace, either way.
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

// bf16 pairs of the 8 codes of one packed word, dyadic: pair j = (code j, code j+4), the
// lower code index in the low half, each bf16(step * (idx - 8)) rounded once.
//
// A bf16 bit pattern below 0x0100 is worth exactly (pattern) * 2^-133: the subnormals and
// the first normal binade share that spacing. So (w & 0x000F000F) is the pair (idx0, idx4)
// times 2^-133 and (w & 0x00F000F0) is (idx1, idx5) times 2^-129, with no shift; w >> 8 gives
// the other two pairs the same way. One FMA by 2^126 (resp. 2^122) brings them to idx * 2^-7
// exactly, and fma(idx * 2^-7, 16 * scale, -scale) = scale * (idx - 8) / 8 is formed exactly
// and rounded once. cs = (16 * scale) pair, cn = (-scale) pair.
__device__ __forceinline__ void dyadic_pairs(uint32_t w, uint32_t cs, uint32_t cn, uint32_t (&p)[4]) {
    const uint32_t kP126 = 0x7E807E80u;       // bf16 2^126 twice
    const uint32_t kP122 = 0x7C807C80u;       // bf16 2^122 twice
    const uint32_t kNegZero = 0x80008000u;
    const uint32_t t = w >> 8;
    p[0] = bf16x2_fma(bf16x2_fma(w & 0x000F000Fu, kP126, kNegZero), cs, cn);
    p[1] = bf16x2_fma(bf16x2_fma(w & 0x00F000F0u, kP122, kNegZero), cs, cn);
    p[2] = bf16x2_fma(bf16x2_fma(t & 0x000F000Fu, kP126, kNegZero), cs, cn);
    p[3] = bf16x2_fma(bf16x2_fma(t & 0x00F000F0u, kP122, kNegZero), cs, cn);
}

// Same pairs computed in fp32 (for scales whose 16x overflows bf16).
__device__ __forceinline__ void dyadic_pairs_f32(uint32_t w, float step, uint32_t (&p)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = step * (float)((int)((w >> (4 * j)) & 15) - 8);
        const float hi = step * (float)((int)((w >> (4 * j + 16)) & 15) - 8);
        p[j] = pack_bf16x2(lo, hi);
    }
}

// (16 * scale, -scale) as bf16 pairs (exact for every finite scale below 2^124).
__device__ __forceinline__ void scale_pairs(uint32_t scale_bits, uint32_t& cs, uint32_t& cn) {
    const uint32_t s2 = prmt(scale_bits, 0, 0x1010u);
    cs = bf16x2_fma(s2, 0x41804180u, 0x80008000u);     // x 16.0
    cn = s2 ^ 0x80008000u;
}

// LUT16 lookup of 4 codes (nibbles of the low 16 bits of s) in a 16-entry fp16 table held
// as byte planes: lo[q] / hi[q] hold the low / high bytes of entries 4q..4q+3. Returns the
// fp16 pairs (code0, code1) and (code2, code3).
__device__ __forceinline__ void lut16_lookup4(uint32_t s, const uint32_t* lo, const uint32_t* hi,
                                              uint32_t& p01, uint32_t& p23) {
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

// Per-lane state of one 256-column step for R 16-row blocks: the 32 bytes of rows g and
// g+8 of each block, and their per-group parameters.
template <int KIND, int R>
struct Step {
    uint32_t w[R][2][8];
    uint32_t aux[R][2][KIND == kLut16 ? 8 : 2];   // dyadic: bf16 scales; LUT16: table words
};

template <int KIND, int R, bool FULL>
__device__ __forceinline__ void load_step(Step<KIND, R>& st, const GemvProblem& pb, int row0, int g,
                                          int kk, int N, int K) {
    const bool h0 = FULL || kk < K, h1 = FULL || kk + 32 < K;
    const size_t row_bytes = (size_t)K / 2;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = row0 + 16 * r + 8 * h + g;
            const bool rl = FULL || row < N;
            const uint8_t* wp = pb.packed + (size_t)row * row_bytes + kk / 2;
            const uint4 fill = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u);
            const uint4 a = (rl && h0) ? ldg_nc_v4(wp) : fill;
            const uint4 b = (rl && h1) ? ldg_nc_v4(wp + 16) : fill;
            st.w[r][h][0] = a.x; st.w[r][h][1] = a.y; st.w[r][h][2] = a.z; st.w[r][h][3] = a.w;
            st.w[r][h][4] = b.x; st.w[r][h][5] = b.y; st.w[r][h][6] = b.z; st.w[r][h][7] = b.w;
            if (KIND == kLut16) {
                uint4 la = make_uint4(0, 0, 0, 0), lb = la;
                if (rl && h0) {
                    const uint4* lp = (const uint4*)((const uint16_t*)pb.aux + ((size_t)row * (K / 64) + kk / 64) * 16);
                    la = ldg_nc_v4(lp);
                    lb = ldg_nc_v4(lp + 1);
                }
                // raw table words; split into byte planes at use
                st.aux[r][h][0] = la.x; st.aux[r][h][1] = la.y; st.aux[r][h][2] = la.z; st.aux[r][h][3] = la.w;
                st.aux[r][h][4] = lb.x; st.aux[r][h][5] = lb.y; st.aux[r][h][6] = lb.z; st.aux[r][h][7] = lb.w;
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
                st.aux[r][h][0] = s0;
                st.aux[r][h][1] = s1;
            }
        }
}

// One 256-column step: 8 words per row, 2 (or 4) mma per word pair. FULL: the step lies
// inside K, so every activation load is in range; lanes whose batch column is unused load
// some valid row (those output columns are computed but never stored).
template <int KIND, int NB, int R, bool SLOW, bool FULL>
__device__ __forceinline__ void compute_step(const Step<KIND, R>& st, float (&acc)[R][NB][4],
                                             const uint16_t* xg, const uint16_t* xg8, bool xa_live,
                                             bool xb_live, int kk, int K, uint4 (&xr)[2]) {
    const bool h0 = kk < K, h1 = kk + 32 < K;
    uint32_t cs[R][2][2], cn[R][2][2];
    float fst[R][2][2];
    uint32_t plo[R][2][4], phi[R][2][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (KIND == kLut16) {
                const uint32_t* L = st.aux[r][h];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    plo[r][h][q] = prmt(L[2 * q], L[2 * q + 1], 0x6420u);
                    phi[r][h][q] = prmt(L[2 * q], L[2 * q + 1], 0x7531u);
                }
            } else {
#pragma unroll
                for (int j = 0; j < (KIND == kDyadic32 ? 2 : 1); ++j) {
                    if (SLOW) fst[r][h][j] = bf16_bits_to_float(st.aux[r][h][j]) * 0.125f;
                    else scale_pairs(st.aux[r][h][j], cs[r][h][j], cn[r][h][j]);
                }
            }
        }
#pragma unroll
    for (int sub = 0; sub < 8; ++sub) {
        const int kx = kk + 8 * sub;
        uint4 xa, xb;
        if (FULL) {
            // lanes of unused batch columns keep stale registers: their columns are never stored
            ldg_v4_if(xr[0], xg + kx, xa_live);
            xa = xr[0];
            if (NB == 2) {
                ldg_v4_if(xr[1], xg8 + kx, xb_live);
                xb = xr[1];
            }
        } else {
            const bool xv = (sub < 4) ? h0 : h1;
            xa = make_uint4(0, 0, 0, 0);
            xb = xa;
            if (xa_live && xv) xa = ldg_v4(xg + kx);
            if (NB == 2 && xb_live && xv) xb = ldg_v4(xg8 + kx);
        }
        uint32_t b[NB][4];                              // B fragments of the two mma
        if (KIND == kLut16) {
            b[0][0] = bf16x2_to_f16x2(xa.x); b[0][1] = bf16x2_to_f16x2(xa.y);
            b[0][2] = bf16x2_to_f16x2(xa.z); b[0][3] = bf16x2_to_f16x2(xa.w);
            if (NB == 2) {
                b[NB - 1][0] = bf16x2_to_f16x2(xb.x); b[NB - 1][1] = bf16x2_to_f16x2(xb.y);
                b[NB - 1][2] = bf16x2_to_f16x2(xb.z); b[NB - 1][3] = bf16x2_to_f16x2(xb.w);
            }
        } else {
            b[0][0] = prmt(xa.x, xa.z, 0x5410u); b[0][1] = prmt(xa.x, xa.z, 0x7632u);
            b[0][2] = prmt(xa.y, xa.w, 0x5410u); b[0][3] = prmt(xa.y, xa.w, 0x7632u);
            if (NB == 2) {
                b[NB - 1][0] = prmt(xb.x, xb.z, 0x5410u); b[NB - 1][1] = prmt(xb.x, xb.z, 0x7632u);
                b[NB - 1][2] = prmt(xb.y, xb.w, 0x5410u); b[NB - 1][3] = prmt(xb.y, xb.w, 0x7632u);
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            uint32_t q0[4], q1[4];                      // rows g and g+8
            if (KIND == kLut16) {
                lut16_lookup4(st.w[r][0][sub], plo[r][0], phi[r][0], q0[0], q0[1]);
                lut16_lookup4(st.w[r][0][sub] >> 16, plo[r][0], phi[r][0], q0[2], q0[3]);
                lut16_lookup4(st.w[r][1][sub], plo[r][1], phi[r][1], q1[0], q1[1]);
                lut16_lookup4(st.w[r][1][sub] >> 16, plo[r][1], phi[r][1], q1[2], q1[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_f16_16816(acc[r][nb], q0[0], q1[0], q0[1], q1[1], b[nb][0], b[nb][1]);
                    mma_f16_16816(acc[r][nb], q0[2], q1[2], q0[3], q1[3], b[nb][2], b[nb][3]);
                }
            } else {
                const int hs = (KIND == kDyadic32 && sub >= 4) ? 1 : 0;
                if (SLOW) {
                    dyadic_pairs_f32(st.w[r][0][sub], fst[r][0][hs], q0);
                    dyadic_pairs_f32(st.w[r][1][sub], fst[r][1][hs], q1);
                } else {
                    dyadic_pairs(st.w[r][0][sub], cs[r][0][hs], cn[r][0][hs], q0);
                    dyadic_pairs(st.w[r][1][sub], cs[r][1][hs], cn[r][1][hs], q1);
                }
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_bf16_16816(acc[r][nb], q0[0], q1[0], q0[1], q1[1], b[nb][0], b[nb][1]);
                    mma_bf16_16816(acc[r][nb], q0[2], q1[2], q0[3], q1[3], b[nb][2], b[nb][3]);
                }
            }
        }
    }
}

// A step needs the fp32 path when 16 * scale would overflow bf16 (scale >= 2^124).
template <int KIND, int R>
__device__ __forceinline__ bool step_needs_slow(const Step<KIND, R>& st) {
    if (KIND == kLut16) return false;
    uint32_t m = 0;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 2; ++j) m = max(m, st.aux[r][h][j] & 0x7FFFu);
    return m >= 0x7D80u;
}

template <int KIND, int NB, int R, int WK, int MAXP>
__global__ void __launch_bounds__(128)
gemv_kernel(const __grid_constant__ GemvParams<MAXP> prm) {
    constexpr int WR = 4 / WK;                       // warps with distinct rows per CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wr = warp % WR, wk = warp / WR;
    // ---- which problem / row tile (a tile = the 16*R*WR rows of one CTA) -----------------
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
    const int row0 = ((int)blockIdx.x - prm.tile_start[p]) * (16 * R * WR) + wr * 16 * R;
    const int g = lane >> 2, t = lane & 3;
    const int steps = (K + 255) >> 8;

    float acc[R][NB][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[r][nb][0] = acc[r][nb][1] = acc[r][nb][2] = acc[r][nb][3] = 0.f;

    const bool xa_live = g < B, xb_live = NB == 2 && (g + 8 < B);
    // lanes whose batch column is unused read row 0 (their outputs are never stored)
    const uint16_t* xg = pb.x + (size_t)(xa_live ? g : 0) * K;
    const uint16_t* xg8 = pb.x + (size_t)(xb_live ? g + 8 : 0) * K;

    if (row0 < N && wk == 0 && lane == 0) {
        // The warp's rows are contiguous in memory: ask the L2 for all of them now, so the
        // register loads below see L2 latency rather than DRAM latency.
        const int rows = min(16 * R, N - row0);
        const size_t row_bytes = (size_t)K / 2;
        prefetch_l2_bulk(pb.packed + (size_t)row0 * row_bytes, (uint32_t)(rows * row_bytes));
        if (KIND == kLut16) {
            const size_t lb = (size_t)(K / 64) * 32;                  // fp16 [16] per block
            prefetch_l2_bulk((const uint8_t*)pb.aux + (size_t)row0 * lb, (uint32_t)(rows * lb));
        } else {
            // scales: the 16-byte-aligned interior of this warp's rows
            const size_t sb = (size_t)(K / (KIND == kDyadic64 ? 64 : 32)) * 2;
            const uintptr_t a0 = (uintptr_t)pb.aux + (size_t)row0 * sb;
            const uintptr_t a1 = a0 + (size_t)rows * sb;
            const uintptr_t b0 = (a0 + 15) & ~(uintptr_t)15, b1 = a1 & ~(uintptr_t)15;
            if (b1 > b0) prefetch_l2_bulk((const void*)b0, (uint32_t)(b1 - b0));
        }
    }
    if (row0 < N) {
        // FULL steps (all rows of the warp and all 256 columns in range) run without
        // predicates; only a ragged last step or a ragged last row block take the checks
        const bool rows_full = row0 + 16 * R <= N;
        const int full_steps = rows_full ? (K >> 8) : 0;
        auto load = [&](Step<KIND, R>& st, int s) {
            if (s < full_steps) load_step<KIND, R, true>(st, pb, row0, g, s * 256 + t * 64, N, K);
            else load_step<KIND, R, false>(st, pb, row0, g, s * 256 + t * 64, N, K);
        };
        uint4 xr[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        auto run_step = [&](const Step<KIND, R>& st, int s) {
            const int kk = s * 256 + t * 64;
            if (__builtin_expect(__any_sync(0xFFFFFFFFu, step_needs_slow<KIND, R>(st)), 0))
                compute_step<KIND, NB, R, true, false>(st, acc, xg, xg8, xa_live, xb_live, kk, K, xr);
            else if (s < (K >> 8))
                compute_step<KIND, NB, R, false, true>(st, acc, xg, xg8, xa_live, xb_live, kk, K, xr);
            else
                compute_step<KIND, NB, R, false, false>(st, acc, xg, xg8, xa_live, xb_live, kk, K, xr);
        };
        // two register buffers in ping-pong: the next step's bytes load while this one computes
        Step<KIND, R> b0, b1;
        if (wk < steps) load(b0, wk);
        for (int s = wk; s < steps; s += 2 * WK) {
            if (s + WK < steps) load(b1, s + WK);
            run_step(b0, s);
            if (s + WK >= steps) break;
            if (s + 2 * WK < steps) load(b0, s + 2 * WK);
            run_step(b1, s + WK);
        }
    }

    // ---- output: fragment (lane, nb, j): row = g + 8*(j>>1), batch = 8*nb + 2t + (j&1) ----
    if (WK > 1) {
        __shared__ float red[WK > 1 ? WK : 1][WR][R][NB][4][32];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int j = 0; j < 4; ++j) red[wk][wr][r][nb][j][lane] = acc[r][nb][j];
        __syncthreads();
        if (wk != 0) return;
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float v = 0.f;
#pragma unroll
                    for (int w2 = 0; w2 < WK; ++w2) v += red[w2][wr][r][nb][j][lane];
                    acc[r][nb][j] = v;
                }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int row = row0 + 16 * r + g + 8 * (j >> 1);
                const int b = 8 * nb + 2 * t + (j & 1);
                if (b < B && row < N) pb.y[(size_t)b * N + row] = (uint16_t)float_to_bf16_bits(acc[r][nb][j]);
            }
}

template <int KIND, int NB, int R, int WK, int MAXP>
wq_status run(const GemvParams<MAXP>& prm, int tiles, cudaStream_t s) {
    gemv_kernel<KIND, NB, R, WK, MAXP><<<tiles, 128, 0, s>>>(prm);
    return check_launch("gemv");
}

template <int KIND, int NB, int MAXP>
wq_status pick_split(GemvParams<MAXP>& prm, const GemvProblem* probs, int count, int64_t rows16,
                     int batch, cudaStream_t s) {
    // Full-K warps (no reduction) when the launch has at least ~6 warps of 32 rows per SM;
    // otherwise 16-row warps, and K split over 2 or 4 warps of a CTA for small launches.
    const int64_t sms = sm_count();
    auto tiles_for = [&](int rows_per_cta) {
        int tiles = 0;
        for (int i = 0; i < count; ++i) {
            prm.tile_start[i] = tiles;
            tiles += (probs[i].n + rows_per_cta - 1) / rows_per_cta;
        }
        prm.tile_start[count] = tiles;
        return tiles;
    };
    // 32-row warps pay off once the activation fragment is shared by more batch rows
    // (measured: 16-row warps win at batch <= 4, 32-row warps at batch 5..16)
    constexpr int BIGR = (KIND == kLut16) ? 1 : 2;
    if (BIGR == 2 && batch > 4 && rows16 >= 12 * sms * 2)
        return run<KIND, NB, BIGR, 1, MAXP>(prm, tiles_for(64 * BIGR), s);
    if (rows16 >= 8 * sms) return run<KIND, NB, 1, 1, MAXP>(prm, tiles_for(64), s);
    if (rows16 >= 2 * sms) return run<KIND, NB, 1, 2, MAXP>(prm, tiles_for(32), s);
    return run<KIND, NB, 1, 4, MAXP>(prm, tiles_for(16), s);
}

template <int MAXP>
wq_status launch_impl(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    GemvParams<MAXP> prm;
    prm.count = count;
    prm.batch = batch;
    int64_t rows16 = 0;
    for (int i = 0; i < count; ++i) { prm.prob[i] = probs[i]; rows16 += (probs[i].n + 15) / 16; }
    const bool two = batch > 8;
    const int kind = (fmt == WQ_FMT_LUT16) ? kLut16 : (group == 64 ? kDyadic64 : kDyadic32);
    if (kind == kLut16)
        return two ? pick_split<kLut16, 2, MAXP>(prm, probs, count, rows16, batch, s)
                   : pick_split<kLut16, 1, MAXP>(prm, probs, count, rows16, batch, s);
    if (kind == kDyadic64)
        return two ? pick_split<kDyadic64, 2, MAXP>(prm, probs, count, rows16, batch, s)
                   : pick_split<kDyadic64, 1, MAXP>(prm, probs, count, rows16, batch, s);
    return two ? pick_split<kDyadic32, 2, MAXP>(prm, probs, count, rows16, batch, s)
               : pick_split<kDyadic32, 1, MAXP>(prm, probs, count, rows16, batch, s);
}

}  // namespace

wq_status launch_gemv(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    if (count == 1) return launch_impl<1>(fmt, group, probs, count, batch, s);
    return launch_impl<kMaxProblems>(fmt, group, probs, count, batch, s);
}

}  // namespace wq
