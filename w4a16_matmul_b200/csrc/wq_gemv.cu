// wq_gemv.cu -- W4A16 GEMV for decode: y[b, r] = sum_c Wdeq[r, c] x[b, c], b < batch <= 16.
//
// Reconstruction follows "MiniCPM5-1B 验证: 6× 压缩…" §2.2/§2.5 (dyadic: bf16(step*(idx-8)))
// "K-Means量化技术…" §2.2 (LUT16: a 16-entry centroid table per block of 64) and
// "int4-g32+warm 裸量化…" §5.2 (LLOYD8S: bf16(±level) from a group's 8 levels, the codebook
// held in registers), fused into the product instead of written out as a dense matrix.
//
// Design (HBM-bound: 0.53 B per dyadic weight, 1 B per LUT16 weight; what stands between
// the kernel and the memory roof is the instruction count and latency of the in-register
// reconstruction):
//   * A warp owns 16*R rows of one problem. Lane (g = lane/4, t = lane%4) streams rows g
//     and g+8 of every 16-row block: per 256-column step, 32 contiguous bytes of each
//     (64 codes: one dyadic g64 group, two g32 groups, or one LUT16 block) with two
//     128-bit non-allocating loads; a quad of lanes covers 128 contiguous bytes of a row.
//     The next step's bytes are loaded while the current step computes.
//   * The CTA stages its activations once per K chunk into shared memory, already in the
//     order of the mma B fragment, so one 128-bit shared load per 8 columns replaces the
//     global load and the byte permutes of every warp (the activations are read from L2
//     once per CTA instead of once per warp).
//   * The product runs on the warp-level tensor-core path (mma m16n8k16, fp32
//     accumulate): the reconstructed weights are the A operand (16 rows x 16 columns, no
//     padding), the activations the B operand (batch columns 0..7, and 8..15 in a second
//     mma when batch > 8).
//   * Dyadic reconstruction is exact and costs one bf16x2 FMA per weight pair. The nibble
//     pairs are masked straight out of the packed word, which makes them bf16 numbers
//     idx * 2^-133 (or idx * 2^-129); one FMA with (scale * 2^66, -scale * 2^-64) forms
//     2^-64 * step * (idx - 8) and rounds it once, i.e. 2^-64 times the bf16 weight that
//     wq_dequant writes. The staged activations carry the compensating 2^64, so every
//     product, and hence the fp32 sum, is the one of the unscaled operands. Steps whose
//     scales fall outside [2^-59, 2^62), or chunks whose activations reach 2^64, take an
//     exact fp32 path with unscaled activations.
//   * The k order inside one mma is a permutation of the physical columns (word nibbles
//     pair up as (0,4), (1,5), (2,6), (3,7)); the staged activations follow it, so the
//     contraction is unchanged.
//   * When a launch has too few rows to fill the GPU, WK warps of a CTA split K and meet
//     in shared memory at the end; otherwise every warp covers the full K and no
//     reduction exists. One launch, no workspace, either way.
#include <cooperative_groups.h>
#include <new>

#include "wq_internal.cuh"

namespace wq {

WQ_DEBUG_WORD(gemv)
namespace {

constexpr int kMaxProblems = WQ_GEMV_MAX_GROUPED;
#ifndef WQ_GEMV_DEPTH
#define WQ_GEMV_DEPTH 2
#endif
#ifndef WQ_GEMV_MIN_CTAS_NB1
#define WQ_GEMV_MIN_CTAS_NB1 (WQ_GEMV_DEPTH >= 4 ? 4 : 5)
#endif
#ifndef WQ_GEMV_MIN_CTAS_NB2
#define WQ_GEMV_MIN_CTAS_NB2 4
#endif
#ifndef WQ_GEMV_L2HINT
#define WQ_GEMV_L2HINT 2             // weight loads: 0 plain, 1 L2::128B, 2 L2::256B sector prefetch
#endif
#ifndef WQ_GEMV_R2_MIN_BATCH
#define WQ_GEMV_R2_MIN_BATCH 8       // 32-row warps above this batch (large launches)
#endif

template <int MAXP>
struct GemvParams {
    int count;
    int batch;
    int chunk_steps;              // 256-column steps per staged activation chunk
    int tile_start[MAXP + 1];     // prefix sum of row tiles per problem
    GemvProblem prob[MAXP];
};

// bf16 pairs of the 8 codes of one packed word, dyadic, computed in fp32 (exact for every
// scale) and rounded once: pair j = (code j, code j+4), the lower code index in the low half.
__device__ __forceinline__ void dyadic_pairs_f32(uint32_t w, float step, uint32_t (&p)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float lo = step * (float)((int)((w >> (4 * j)) & 15) - 8);
        const float hi = step * (float)((int)((w >> (4 * j + 16)) & 15) - 8);
        p[j] = pack_bf16x2(lo, hi);
    }
}

// Staged-activation scale and the range of scales the one-FMA reconstruction covers.
// With e = 64: the weights come out times 2^-64 and stay normal for scale >= 2^-59 (biased
// exponent 68); scale * 2^66 stays finite for scale < 2^62 (biased exponent <= 188);
// activations times 2^64 stay finite for |x| < 2^64 (bf16 magnitude bits < 0x5F80).
constexpr uint32_t kXScalePair = 0x5F805F80u;    // bf16 2^64 twice
constexpr uint32_t kScaleExpLo = 68, kScaleExpHi = 188;

// (scale * 2^66, scale * 2^62, -scale * 2^-64) as bf16 pairs, by adding to the exponent
// field (exact: the range check keeps every result a normal number).
__device__ __forceinline__ void scaled_consts(uint32_t scale_bits, uint32_t& c1, uint32_t& c2,
                                              uint32_t& d) {
    const uint32_t s2 = prmt(scale_bits, 0, 0x1010u);
    c1 = s2 + 0x21002100u;
    c2 = s2 + 0x1F001F00u;
    d = (s2 - 0x20002000u) ^ 0x80008000u;
}

// Pairs of 2^-64 * bf16(step * (idx - 8)): (w & 0x000F000F) is (idx0, idx4) * 2^-133 and
// (w & 0x00F000F0) is (idx1, idx5) * 2^-129 as bf16 numbers; times scale * 2^66 (resp.
// 2^62) they are exactly idx * step * 2^-64, and adding -8 * step * 2^-64 in the same FMA
// rounds once.
__device__ __forceinline__ void dyadic_pairs_scaled(uint32_t w, uint32_t c1, uint32_t c2,
                                                    uint32_t d, uint32_t (&p)[4]) {
    const uint32_t t = w >> 8;
    p[0] = bf16x2_fma(w & 0x000F000Fu, c1, d);
    p[1] = bf16x2_fma(w & 0x00F000F0u, c2, d);
    p[2] = bf16x2_fma(t & 0x000F000Fu, c1, d);
    p[3] = bf16x2_fma(t & 0x00F000F0u, c2, d);
}

enum Kind { kDyadic64 = 0, kDyadic32 = 1, kLut16 = 2, kLloyd8 = 3 };

// Per-lane state of one 256-column step for R 16-row blocks: the 32 bytes of rows g and
// g+8 of each block, and their per-group parameters.
template <int KIND, int R>
struct Step {
    uint32_t w[R][2][8];
    // dyadic: bf16 scales; LUT16: table words; LLOYD8S: the fp32 levels of two groups
    uint32_t aux[R][2][KIND == kLut16 ? 8 : KIND == kLloyd8 ? 16 : 2];
};

// A 128-bit weight load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_w(const void* p) {
    uint4 v;
#if WQ_GEMV_L2HINT == 2
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
#elif WQ_GEMV_L2HINT == 1
    asm volatile("ld.global.nc.L1::no_allocate.L2::128B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
#else
    v = ldg_nc_v4(p);
#endif
    return v;
}

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
            const uint4 a = (rl && h0) ? ldg_w(wp) : fill;
            const uint4 b = (rl && h1) ? ldg_w(wp + 16) : fill;
            st.w[r][h][0] = a.x; st.w[r][h][1] = a.y; st.w[r][h][2] = a.z; st.w[r][h][3] = a.w;
            st.w[r][h][4] = b.x; st.w[r][h][5] = b.y; st.w[r][h][6] = b.z; st.w[r][h][7] = b.w;
            if (KIND == kLloyd8) {
                // the 8 fp32 levels of groups kk/32 and kk/32 + 1 (64 contiguous bytes)
                const uint4* lp = (const uint4*)((const float*)pb.aux + ((size_t)row * (K / 32) + kk / 32) * 8);
                uint4 l[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) l[q] = make_uint4(0, 0, 0, 0);
                if (rl && h0) { l[0] = ldg_nc_v4(lp); l[1] = ldg_nc_v4(lp + 1); }
                if (rl && h1) { l[2] = ldg_nc_v4(lp + 2); l[3] = ldg_nc_v4(lp + 3); }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    st.aux[r][h][4 * q] = l[q].x; st.aux[r][h][4 * q + 1] = l[q].y;
                    st.aux[r][h][4 * q + 2] = l[q].z; st.aux[r][h][4 * q + 3] = l[q].w;
                }
            } else if (KIND == kLut16) {
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
                // rows or groups outside the matrix get scale 1.0 (their codes are 8, so their
                // weights are 0) which keeps the step on the one-FMA path
                const uint16_t* sp = (const uint16_t*)pb.aux;
                uint32_t s0 = 0x3F80u, s1 = 0x3F80u;
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

// This lane's weight and scale pointers at step 0, for the rows g and g + 8 of each 16-row
// block (computed once per warp; a FULL dyadic step only adds its offset).
template <int KIND, int R>
struct LaneRows {
    const uint8_t* w[R][2];
    const uint16_t* sc[R][2];
};

template <int KIND, int R>
__device__ __forceinline__ LaneRows<KIND, R> lane_rows(const GemvProblem& pb, int row0, int g, int t,
                                                       int N, int K) {
    LaneRows<KIND, R> lr;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = min(row0 + 16 * r + 8 * h + g, N - 1);   // only FULL steps use these
            lr.w[r][h] = pb.packed + (size_t)row * (K / 2) + 32 * t;
            lr.sc[r][h] = (const uint16_t*)pb.aux + (KIND == kDyadic32 ? (size_t)row * (K / 32) + 2 * t
                                                                      : (size_t)row * (K / 64) + t);
        }
    return lr;
}

// A FULL dyadic step (every row and column in range) from the precomputed pointers.
template <int KIND, int R>
__device__ __forceinline__ void load_step_full(Step<KIND, R>& st, const LaneRows<KIND, R>& lr, int s) {
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint8_t* wp = lr.w[r][h] + 128 * s;
            const uint4 a = ldg_w(wp), b = ldg_w(wp + 16);
            st.w[r][h][0] = a.x; st.w[r][h][1] = a.y; st.w[r][h][2] = a.z; st.w[r][h][3] = a.w;
            st.w[r][h][4] = b.x; st.w[r][h][5] = b.y; st.w[r][h][6] = b.z; st.w[r][h][7] = b.w;
            if (KIND == kDyadic64) {
                st.aux[r][h][0] = ldg_u16(lr.sc[r][h] + 4 * s);
                st.aux[r][h][1] = st.aux[r][h][0];
            } else {
                st.aux[r][h][0] = ldg_u16(lr.sc[r][h] + 8 * s);
                st.aux[r][h][1] = ldg_u16(lr.sc[r][h] + 8 * s + 1);
            }
        }
}

// One 256-column step from the staged activations: 8 words per row, 2 (or 4) mma per word
// pair. xs0 / xs1: this lane's 16-byte slot of the step in the staged rows of batch
// columns g and g + 8 (lanes of unused batch columns read some staged row; their outputs
// are never stored).
template <int KIND, int NB, int R>
__device__ __forceinline__ void compute_step_staged(const Step<KIND, R>& st, float (&acc)[R][NB][4],
                                                    const uint8_t* xs0, const uint8_t* xs1) {
    constexpr int J = (KIND == kDyadic32) ? 2 : 1;
    uint32_t c1[R][2][J], c2[R][2][J], dd[R][2][J];
    uint32_t plo[R][2][4], phi[R][2][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (KIND == kLloyd8) {
                // bf16(level) of both groups, split into byte planes: plo/phi[2j..2j+1] for
                // group j (one rounding per level, to nearest even)
                const uint32_t* L = st.aux[r][h];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t b01 = pack_bf16x2(__uint_as_float(L[8 * j]), __uint_as_float(L[8 * j + 1]));
                    const uint32_t b23 = pack_bf16x2(__uint_as_float(L[8 * j + 2]), __uint_as_float(L[8 * j + 3]));
                    const uint32_t b45 = pack_bf16x2(__uint_as_float(L[8 * j + 4]), __uint_as_float(L[8 * j + 5]));
                    const uint32_t b67 = pack_bf16x2(__uint_as_float(L[8 * j + 6]), __uint_as_float(L[8 * j + 7]));
                    plo[r][h][2 * j] = prmt(b01, b23, 0x6420u);
                    plo[r][h][2 * j + 1] = prmt(b45, b67, 0x6420u);
                    phi[r][h][2 * j] = prmt(b01, b23, 0x7531u);
                    phi[r][h][2 * j + 1] = prmt(b45, b67, 0x7531u);
                }
            } else if (KIND == kLut16) {
                const uint32_t* L = st.aux[r][h];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    plo[r][h][q] = prmt(L[2 * q], L[2 * q + 1], 0x6420u);
                    phi[r][h][q] = prmt(L[2 * q], L[2 * q + 1], 0x7531u);
                }
            } else {
#pragma unroll
                for (int j = 0; j < J; ++j) scaled_consts(st.aux[r][h][j], c1[r][h][j], c2[r][h][j], dd[r][h][j]);
            }
        }
#pragma unroll
    for (int sub = 0; sub < 8; ++sub) {
        uint32_t b[NB][4];
        {
            const uint4 xa = *reinterpret_cast<const uint4*>(xs0 + 64 * sub);
            b[0][0] = xa.x; b[0][1] = xa.y; b[0][2] = xa.z; b[0][3] = xa.w;
            if (NB == 2) {
                const uint4 xb = *reinterpret_cast<const uint4*>(xs1 + 64 * sub);
                b[NB - 1][0] = xb.x; b[NB - 1][1] = xb.y; b[NB - 1][2] = xb.z; b[NB - 1][3] = xb.w;
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            uint32_t q0[4], q1[4];                      // rows g and g+8
            if (KIND == kLloyd8) {
                const int j = sub < 4 ? 0 : 2;          // words 0-3: first group, 4-7: second
                lloyd8_lookup4(st.w[r][0][sub], plo[r][0] + j, phi[r][0] + j, q0[0], q0[1]);
                lloyd8_lookup4(st.w[r][0][sub] >> 16, plo[r][0] + j, phi[r][0] + j, q0[2], q0[3]);
                lloyd8_lookup4(st.w[r][1][sub], plo[r][1] + j, phi[r][1] + j, q1[0], q1[1]);
                lloyd8_lookup4(st.w[r][1][sub] >> 16, plo[r][1] + j, phi[r][1] + j, q1[2], q1[3]);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_bf16_16816(acc[r][nb], q0[0], q1[0], q0[1], q1[1], b[nb][0], b[nb][1]);
                    mma_bf16_16816(acc[r][nb], q0[2], q1[2], q0[3], q1[3], b[nb][2], b[nb][3]);
                }
            } else if (KIND == kLut16) {
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
                const int hs = (J == 2 && sub >= 4) ? 1 : 0;
                dyadic_pairs_scaled(st.w[r][0][sub], c1[r][0][hs], c2[r][0][hs], dd[r][0][hs], q0);
                dyadic_pairs_scaled(st.w[r][1][sub], c1[r][1][hs], c2[r][1][hs], dd[r][1][hs], q1);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    mma_bf16_16816(acc[r][nb], q0[0], q1[0], q0[1], q1[1], b[nb][0], b[nb][1]);
                    mma_bf16_16816(acc[r][nb], q0[2], q1[2], q0[3], q1[3], b[nb][2], b[nb][3]);
                }
            }
        }
    }
}

// The exact fallback for a dyadic step the one-FMA form does not cover (a scale outside
// [2^-59, 2^62) or staged activations that would overflow): weights formed in fp32 (exact
// for every finite scale) and rounded once, activations read unscaled from global memory.
// It reloads the step's bytes itself, one word per row and sub-step, so that it needs few
// registers beyond those the hot loop holds.
template <int KIND, int NB, int R>
__device__ __forceinline__ void compute_step_exact(const GemvProblem& pb, int row0, int g, int kk, int N,
                                                   int K, int B, float (&acc)[R][NB][4]) {
    const int group = (KIND == kDyadic32) ? 32 : 64;
    const bool xa_live = g < B, xb_live = NB == 2 && (g + 8 < B);
    const uint16_t* xg = pb.x + (size_t)(xa_live ? g : 0) * K;
    const uint16_t* xg8 = pb.x + (size_t)(xb_live ? g + 8 : 0) * K;
    const size_t row_bytes = (size_t)K / 2;
    const uint16_t* sp = (const uint16_t*)pb.aux;
#pragma unroll 1
    for (int sub = 0; sub < 8; ++sub) {
        const int kx = kk + 8 * sub;
        const bool xv = kx < K;
        uint4 xa = make_uint4(0, 0, 0, 0), xb = xa;
        if (xa_live && xv) xa = ldg_v4(xg + kx);
        if (NB == 2 && xb_live && xv) xb = ldg_v4(xg8 + kx);
        uint32_t b[NB][4];
        b[0][0] = prmt(xa.x, xa.z, 0x5410u); b[0][1] = prmt(xa.x, xa.z, 0x7632u);
        b[0][2] = prmt(xa.y, xa.w, 0x5410u); b[0][3] = prmt(xa.y, xa.w, 0x7632u);
        if (NB == 2) {
            b[NB - 1][0] = prmt(xb.x, xb.z, 0x5410u); b[NB - 1][1] = prmt(xb.x, xb.z, 0x7632u);
            b[NB - 1][2] = prmt(xb.y, xb.w, 0x5410u); b[NB - 1][3] = prmt(xb.y, xb.w, 0x7632u);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            uint32_t q[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = row0 + 16 * r + 8 * h + g;
                uint32_t w = 0x88888888u, sc = 0;
                if (row < N && xv) {
                    w = ldg_u32(pb.packed + (size_t)row * row_bytes + kx / 2);
                    sc = ldg_u16(sp + (size_t)row * (K / group) + kx / group);
                }
                dyadic_pairs_f32(w, bf16_bits_to_float(sc) * 0.125f, q[h]);
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                mma_bf16_16816(acc[r][nb], q[0][0], q[1][0], q[0][1], q[1][1], b[nb][0], b[nb][1]);
                mma_bf16_16816(acc[r][nb], q[0][2], q[1][2], q[0][3], q[1][3], b[nb][2], b[nb][3]);
            }
        }
    }
}

// True when every scale of the step lies in [2^-59, 2^62) (biased exponent 68..188), the
// range the one-FMA reconstruction covers.
template <int KIND, int R>
__device__ __forceinline__ bool step_scales_in_range(const Step<KIND, R>& st) {
    if (KIND == kLut16 || KIND == kLloyd8) return true;
    bool ok = true;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < (KIND == kDyadic32 ? 2 : 1); ++j) {
                const uint32_t e = (st.aux[r][h][j] >> 7) & 0xFFu;
                ok = ok && (e - kScaleExpLo <= kScaleExpHi - kScaleExpLo);
            }
    return ok;
}

// Staged activations: batch row b at byte b * rs (rs = 512 * chunk_steps + 64, so the
// eight rows one 128-bit shared load phase touches start on distinct banks); inside a row,
// step s of the chunk at 512 * s, sub-step u at 64 * u, quad position t at 16 * t: the
// 8 columns 256 * s + 64 * t + 8 * u .. +7 in B-fragment order. Dyadic: bf16 times 2^64,
// columns paired (0,4), (1,5), (2,6), (3,7); LUT16: fp16 in natural order, each batch row's
// 256 columns of a step times the power of two 2^e that puts their largest magnitude in
// [2^15, 2^16) (lut_x_exponent), with 2^-e in xf[b * ns + step] for the step's sums (a warp
// stages exactly one row's step: its 32 consecutive 8-column blocks); LLOYD8S: bf16 in
// natural order. Columns at or beyond K are zero. Stages steps [c0, c0 + ns) of all B rows
// with the whole CTA; returns (dyadic) whether some staged |x| reaches 2^64 or is not finite.
template <int KIND, int THREADS>
__device__ __forceinline__ bool stage_x(uint8_t* xs, const uint16_t* x, int B, int K, int c0,
                                        int ns, int rs, float* xf) {
    const int per_row = ns * 32;                 // 16-byte blocks of 8 columns
    const int total = B * per_row;
    uint32_t bad = 0;
    constexpr int U = 4;                         // loads in flight per thread
    for (int base = threadIdx.x; base < total; base += THREADS * U) {
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + THREADS * u;
            v[u] = make_uint4(0, 0, 0, 0);
            if (i < total) {
                const int b = i / per_row, j = i - b * per_row;
                const int col = c0 * 256 + 8 * j;
                if (col < K) v[u] = ldg_v4(x + (size_t)b * K + col);
                WQ_DCHECK(b < B && bf16x8_finite(v[u]), kDbgNonFiniteActivation + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + THREADS * u;
            if (i >= total) break;
            const int b = i / per_row, j = i - b * per_row;
            uint4 f;
            if (KIND == kLut16) {
                // the warp's 32 blocks are row b's step j >> 5 (a row is ns * 32 blocks)
                const int e = lut_x_exponent(__reduce_max_sync(0xFFFFFFFFu, bf16x8_max_mag(v[u])));
                if ((threadIdx.x & 31) == 0) xf[b * ns + (j >> 5)] = pow2_f32(-e);
                if (e <= 127) {                         // (warp-uniform) 2^e is a bf16 number
                    const uint32_t p2 = bf16_pow2_bits(e) * 0x10001u;
                    f.x = bf16x2_to_f16x2_pow2(v[u].x, p2); f.y = bf16x2_to_f16x2_pow2(v[u].y, p2);
                    f.z = bf16x2_to_f16x2_pow2(v[u].z, p2); f.w = bf16x2_to_f16x2_pow2(v[u].w, p2);
                } else {                                // a step whose largest |x| is below 2^-112
                    const float s1 = pow2_f32(e >> 1), s2 = pow2_f32(e - (e >> 1));
                    f.x = bf16x2_to_f16x2_scaled(v[u].x, s1, s2); f.y = bf16x2_to_f16x2_scaled(v[u].y, s1, s2);
                    f.z = bf16x2_to_f16x2_scaled(v[u].z, s1, s2); f.w = bf16x2_to_f16x2_scaled(v[u].w, s1, s2);
                }
            } else if (KIND == kLloyd8) {
                f = v[u];                               // bf16 in natural order
            } else {
                // a half of magnitude bits m >= 0x5F80 (|x| >= 2^64, inf, NaN) carries into
                // bit 15 of that half when 0x2080 is added
                const uint32_t m = ((v[u].x & 0x7FFF7FFFu) + 0x20802080u) | ((v[u].y & 0x7FFF7FFFu) + 0x20802080u) |
                                   ((v[u].z & 0x7FFF7FFFu) + 0x20802080u) | ((v[u].w & 0x7FFF7FFFu) + 0x20802080u);
                bad |= m & 0x80008000u;
                const uint32_t kNegZero = 0x80008000u;
                f.x = bf16x2_fma(prmt(v[u].x, v[u].z, 0x5410u), kXScalePair, kNegZero);
                f.y = bf16x2_fma(prmt(v[u].x, v[u].z, 0x7632u), kXScalePair, kNegZero);
                f.z = bf16x2_fma(prmt(v[u].y, v[u].w, 0x5410u), kXScalePair, kNegZero);
                f.w = bf16x2_fma(prmt(v[u].y, v[u].w, 0x7632u), kXScalePair, kNegZero);
            }
            *reinterpret_cast<uint4*>(xs + b * rs + (j >> 5) * 512 + (j & 7) * 64 + ((j >> 3) & 3) * 16) = f;
        }
    }
    return bad != 0;
}

// Steps of weight bytes held in registers per warp (D - 1 of them in flight): the bytes in
// flight per SM, warps x (D - 1) x 2 KB, set the bandwidth a latency-bound stream reaches,
// and deeper buffers buy them at fewer registers than more warps would.
constexpr int depth(int kind, int nb, int r) {
    return (kind < kLut16 && nb == 1 && r == 1) ? WQ_GEMV_DEPTH : 2;
}

#ifndef WQ_GEMV_CL_WARPS
#define WQ_GEMV_CL_WARPS 24           // resident warps per SM the cluster split of small launches aims at
#endif
#ifndef WQ_GEMV_CLUSTER
#define WQ_GEMV_CLUSTER 1             // small launches split K across a thread-block cluster
#endif
#ifndef WQ_GEMV_WARPS_BATCHED
#define WQ_GEMV_WARPS_BATCHED 8
#endif
// Warps per CTA: full-K kernels (WK = 1) take FW row warps (a CTA stages its activations
// once for all of them, so more warps per CTA pay once the staged batch is larger);
// split-K kernels have 4 warps in total.
constexpr int cta_warps(int wk, int fw) { return wk == 1 ? fw : 4; }

// Resident warps per SM the register budget aims at. The dyadic 16-row kernels: 4-warp
// CTAs (batch 1) at WQ_GEMV_MIN_CTAS_NB1 CTAs (measured on the decode sweep: 5 CTAs of
// 96 registers beat 6 of 80 by 2-3 %, the fatter budget saving more instructions than the
// lost warps cost), 8-warp CTAs (batch 2..8) at 24 warps; the other variants take what
// they need.
#ifndef WQ_GEMV_R2_CAP
#define WQ_GEMV_R2_CAP 4
#endif
// LUT16: 4 CTAs per SM (at most 128 registers, no spills; measured on the 8192 x 28672
// LUT16 GEMV: 84 -> 78 / 110 -> 96 / 141 -> 118 us at batch 1 / 8 / 16 against 3 CTAs);
// LLOYD8S keeps its full register budget (it spills at 128).
#ifndef WQ_GEMV_LUT_CAP
#define WQ_GEMV_LUT_CAP 4
#endif
#ifndef WQ_GEMV_LUT_FW
#define WQ_GEMV_LUT_FW 8
#endif
#ifndef WQ_GEMV_CL_FW
#define WQ_GEMV_CL_FW 8               // warps per CTA in the cluster split, other formats, batch >= 4
#endif
#ifndef WQ_GEMV_LLOYD_CAP
#define WQ_GEMV_LLOYD_CAP 1
#endif
constexpr int min_warps(int kind, int nb, int r, int warps_per_cta) {
    return kind == kLloyd8 ? 4 * WQ_GEMV_LLOYD_CAP
         : kind == kLut16 ? 4 * WQ_GEMV_LUT_CAP
         : r != 1 ? 4 * WQ_GEMV_R2_CAP
         : nb != 1 ? 4 * WQ_GEMV_MIN_CTAS_NB2
         : warps_per_cta == 4 ? 4 * WQ_GEMV_MIN_CTAS_NB1 : 24;
}
constexpr int min_blocks(int kind, int nb, int r, int warps_per_cta) {
    return min_warps(kind, nb, r, warps_per_cta) / warps_per_cta > 0
               ? min_warps(kind, nb, r, warps_per_cta) / warps_per_cta : 1;
}

// CL > 1: a thread-block cluster of CL CTAs shares each row tile, CTA rank c taking a
// contiguous slice of the K steps; the partial sums meet in rank 0's shared memory over the
// cluster (distributed shared memory), between two cluster barriers.
template <int KIND, int NB, int R, int WK, int FW, int MAXP, int CL>
__global__ void __launch_bounds__(32 * cta_warps(WK, FW), min_blocks(KIND, NB, R, cta_warps(WK, FW)))
gemv_kernel(const __grid_constant__ GemvParams<MAXP> prm) {
    static_assert(CL == 1 || WK == 1, "a cluster splits K across CTAs, not within one");
    constexpr int THREADS = 32 * cta_warps(WK, FW);
    constexpr int WR = cta_warps(WK, FW) / WK;       // warps with distinct rows per CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wr = warp % WR, wk = warp / WR;
    const int tb = (int)blockIdx.x / CL;             // row tile (clusters are CL consecutive CTAs)
    const int crank = (int)blockIdx.x % CL;
    // A launch made with programmatic stream serialization (a plan with overlap enabled) may
    // start while the kernel before it finishes: let the next launch do the same with this
    // one as soon as all of this grid's CTAs are running. (No effect on other launches.)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // ---- which problem / row tile (a tile = the 16*R*WR rows of one CTA) -----------------
    int p = 0;
    if (MAXP > 1) {
        int lo = 0, hi = prm.count - 1;
        while (lo < hi) {                      // last p with tile_start[p] <= tb
            const int mid = (lo + hi + 1) >> 1;
            if (prm.tile_start[mid] <= tb) lo = mid; else hi = mid - 1;
        }
        p = lo;
    }
    WQ_DCHECK(p >= 0 && p < prm.count && tb >= prm.tile_start[p] && tb < prm.tile_start[p + 1], kDbgIndex + 10);
    const GemvProblem& pb = prm.prob[p];
    const int N = pb.n, K = pb.k, B = prm.batch;
    const int row0 = (tb - prm.tile_start[p]) * (16 * R * WR) + wr * 16 * R;
    const int g = lane >> 2, t = lane & 3;
    const int all_steps = (K + 255) >> 8;
    // this CTA's steps: [s_lo, steps)
    const int per = (all_steps + CL - 1) / CL;
    const int s_lo = min(all_steps, crank * per);
    const int steps = min(all_steps, s_lo + per);

    float acc[R][NB][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[r][nb][0] = acc[r][nb][1] = acc[r][nb][2] = acc[r][nb][3] = 0.f;

    extern __shared__ __align__(16) uint8_t xs[];
    const int cs = prm.chunk_steps, rs = 512 * cs + 64;
    const uint8_t* xs0 = xs + min(g, B - 1) * rs + 16 * t;
    const uint8_t* xs1 = xs + min(g + 8, B - 1) * rs + 16 * t;
    const bool live = row0 < N;
    // FULL loads (all rows of the warp and all 256 columns in range) run without
    // predicates; only a ragged last step or a ragged last row block take the checks
    const int full_steps = (row0 + 16 * R <= N) ? (K >> 8) : 0;
    // (16-row warps only: the pointers cost the 32-row kernel registers it does not have)
    constexpr bool kFastLoad = KIND == kDyadic64 && R == 1;
    const LaneRows<KIND, R> lr = lane_rows<KIND, R>(pb, row0, g, t, N, K);
    auto load = [&](Step<KIND, R>& st, int s) {
        if (kFastLoad && s < full_steps) load_step_full<KIND, R>(st, lr, s);
        else if (s < full_steps) load_step<KIND, R, true>(st, pb, row0, g, s * 256 + t * 64, N, K);
        else load_step<KIND, R, false>(st, pb, row0, g, s * 256 + t * 64, N, K);
    };
    // LUT16: each step's staged activations carry their own power of two (stage_x), so a
    // step's products are summed apart and added to acc times the step's 2^-e per batch row
    // (exact); the sums below then hold plain values
    float* xf = reinterpret_cast<float*>(xs + (size_t)B * rs);
    auto run_step = [&](const Step<KIND, R>& st, int s, int c0, bool xbad) {
        if constexpr (KIND == kLut16) {
            float sacc[R][NB][4];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) sacc[r][nb][0] = sacc[r][nb][1] = sacc[r][nb][2] = sacc[r][nb][3] = 0.f;
            compute_step_staged<KIND, NB, R>(st, sacc, xs0 + 512 * (s - c0), xs1 + 512 * (s - c0));
            const int ns = min(cs, steps - c0);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float f = xf[min(8 * nb + 2 * t + h, B - 1) * ns + (s - c0)];
#pragma unroll
                    for (int r = 0; r < R; ++r)
#pragma unroll
                        for (int j = h; j < 4; j += 2) acc[r][nb][j] = fmaf(sacc[r][nb][j], f, acc[r][nb][j]);
                }
        } else if (KIND == kLloyd8 || (!xbad && __all_sync(0xFFFFFFFFu, step_scales_in_range<KIND, R>(st)))) {
            compute_step_staged<KIND, NB, R>(st, acc, xs0 + 512 * (s - c0), xs1 + 512 * (s - c0));
        } else {
            compute_step_exact<KIND, NB, R>(pb, row0, g, s * 256 + t * 64, N, K, B, acc);
        }
    };
    // D register buffers in rotation: the bytes of D - 1 steps are in flight while one step
    // computes, and the first D - 1 steps' loads are issued before the activations are
    // staged. A chunk holds a whole multiple of D * WK steps, so every chunk starts at
    // buffer 0 (step j of this warp lives in buffer j % D).
    constexpr int D = depth(KIND, NB, R);
    Step<KIND, R> buf[D];
    if (live) {
#pragma unroll
        for (int i = 0; i < D - 1; ++i)
            if (s_lo + wk + i * WK < steps) load(buf[i], s_lo + wk + i * WK);
    }
    // Activations are read, and outputs written, only once the kernel before this launch has
    // completed and its writes are visible (immediate without programmatic serialization);
    // the weight loads above may run beside that kernel's tail.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int c0 = s_lo; c0 < steps; c0 += cs) {
        if (c0 > s_lo) __syncthreads();            // every warp is done with the last chunk
        const int ns = min(cs, steps - c0);
        WQ_DCHECK(ns >= 1 && ns <= cs && c0 + ns <= all_steps, kDbgIndex + 11);
        const bool xbad = __syncthreads_or(stage_x<KIND, THREADS>(xs, pb.x, B, K, c0, ns, rs, xf)) != 0;
        if (!live) continue;
        const int cend = c0 + ns;
        for (int s0 = c0 + wk; s0 < cend; s0 += D * WK) {
#pragma unroll
            for (int i = 0; i < D; ++i) {
                const int s = s0 + i * WK;
                if (s >= cend) break;
                if (s + (D - 1) * WK < steps) load(buf[(i + D - 1) % D], s + (D - 1) * WK);
                run_step(buf[i], s, c0, xbad);
            }
        }
    }

    // ---- output: fragment (lane, nb, j): row = g + 8*(j>>1), batch = 8*nb + 2t + (j&1) ----
    if constexpr (CL > 1) {
        __shared__ float cred[WR][R][NB][4][32];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int j = 0; j < 4; ++j) cred[wr][r][nb][j][lane] = acc[r][nb][j];
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();                          // every rank's partial sums are in place
        if (crank == 0) {
#pragma unroll 1
            for (int q = 1; q < CL; ++q) {
                const float* rem = cluster.map_shared_rank(&cred[0][0][0][0][0], q);
#pragma unroll
                for (int r = 0; r < R; ++r)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            acc[r][nb][j] += rem[(((wr * R + r) * NB + nb) * 4 + j) * 32 + lane];
            }
        }
        cluster.sync();                          // rank 0 is done reading the others
        if (crank != 0) return;
    }
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

// Staged activations per CTA: at most this many bytes (a chunk of 256-column steps of all
// batch rows); K is walked in chunks when batch * K does not fit.
constexpr int kXStageBudget = 32 * 1024;

// A launch chosen and parameterised once: the kernel variant, its grid and shared memory.
template <int MAXP>
struct Prepared {
    void (*kern)(GemvParams<MAXP>);
    GemvParams<MAXP> prm;
    int tiles;                   // row tiles; the grid has tiles * cl CTAs
    int cl;                      // cluster size (CTAs splitting one tile's K)
    int threads;
    size_t smem;
    bool overlap = false;        // launch with programmatic stream serialization
};

template <int KIND, int NB, int R, int WK, int FW, int MAXP, int CL = 1>
wq_status prepare_variant(Prepared<MAXP>& pr, const GemvProblem* probs, int tiles) {
    constexpr int unit = depth(KIND, NB, R) * WK;   // chunks are whole multiples of this
    GemvParams<MAXP>& prm = pr.prm;
    int max_steps = 1;
    for (int i = 0; i < prm.count; ++i) max_steps = max(max_steps, (probs[i].k + 255) / 256);
    int cs = max(1, (kXStageBudget / prm.batch - 64) / 512);
    cs = max(unit, cs - cs % unit);
    prm.chunk_steps = min(cs, max_steps);
    pr.smem = (size_t)prm.batch * (512 * prm.chunk_steps + 64);
    if (KIND == kLut16) pr.smem += (size_t)prm.batch * prm.chunk_steps * sizeof(float);   // step factors
    pr.kern = gemv_kernel<KIND, NB, R, WK, FW, MAXP, CL>;
    pr.tiles = tiles;
    pr.cl = CL;
    pr.threads = 32 * cta_warps(WK, FW);
    if (pr.smem > 48 * 1024) {
        // small launches with many batch rows: a chunk of D * WK steps may pass 48 KB
        if (cudaFuncSetAttribute(pr.kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024) !=
            cudaSuccess)
            return check_launch("gemv shared memory");
    }
    return WQ_OK;
}

template <int KIND, int NB, int MAXP>
wq_status pick_split(Prepared<MAXP>& pr, const GemvProblem* probs, int count, int64_t rows16,
                     int batch) {
    // Full-K warps (no reduction) when the launch has at least ~8 warps of rows per SM;
    // otherwise K split over 2 or 4 warps of a CTA for small launches.
    const int64_t sms = sm_count();
    GemvParams<MAXP>& prm = pr.prm;
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
    // (measured on the decode sweep: 16-row warps win up to batch 8, 32-row warps at 9..16)
    constexpr int BIGR = (KIND >= kLut16) ? 1 : 2;
    // warps (of 16 rows) per CTA where a CTA stages its whole K range at batch 1 and in the
    // cluster split: LUT16 takes 8 (each staged activation chunk, converted to fp16 with its
    // scale, then serves 128 weight rows; the CTAs per SM halve at the same 128 registers)
    constexpr int FWL = (KIND == kLut16) ? WQ_GEMV_LUT_FW : 4;
    // the cluster split: 8 warps (128 rows) per CTA for LUT16, and for the other formats
    // from batch 4 on, where staging the activations is a large share of a CTA's work
    // (measured on 4096 x 11008 and 11008 x 4096 at m = 8 / 12 / 16: 12.5 -> 12.0 / 19.7 ->
    // 17.9 / 22.9 -> 19.9 us and 14.5 -> 13.3 / 18.7 -> 16.6 / 21.4 -> 17.9 us; at batch 1
    // it was up to 0.9 us slower)
    constexpr int FWC = (KIND == kLut16) ? WQ_GEMV_LUT_FW : WQ_GEMV_CL_FW;
    // full-K CTAs: 4 row warps at batch 1, WQ_GEMV_WARPS_BATCHED above (measured on the
    // decode sweep: 8 warps +9 / +13 / +14 % at batch 4 / 8 / 16, neutral at batch 1)
    if (BIGR == 2 && batch > WQ_GEMV_R2_MIN_BATCH && rows16 >= 12 * sms * 2) {
        constexpr int FWB = WQ_GEMV_WARPS_BATCHED;
        return prepare_variant<KIND, NB, BIGR, 1, FWB, MAXP>(pr, probs, tiles_for(16 * FWB * BIGR));
    }
    if (rows16 >= 8 * sms) {
        if (batch == 1) return prepare_variant<KIND, NB, 1, 1, FWL, MAXP>(pr, probs, tiles_for(16 * FWL));
        constexpr int FWB = WQ_GEMV_WARPS_BATCHED;
        return prepare_variant<KIND, NB, 1, 1, FWB, MAXP>(pr, probs, tiles_for(16 * FWB));
    }
#if WQ_GEMV_CLUSTER
    {
        // too few rows to fill the GPU: a cluster of CL CTAs per 64-row tile splits K (each
        // CTA at least 2 steps), sized for about 24 resident warps per SM
        // (only for launches of >= 16 M weights: below that the cluster launch costs more
        // than it saves; measured 5.0 -> 6.3 us on a 2048 x 2048 matrix)
        int max_steps = 1;
        int64_t weights = 0;
        for (int i = 0; i < count; ++i) {
            max_steps = max(max_steps, (probs[i].k + 255) / 256);
            weights += (int64_t)probs[i].n * probs[i].k;
        }
        const int64_t tiles64 = (rows16 + 3) / 4;
        int64_t want = (WQ_GEMV_CL_WARPS * sms + 4 * tiles64 - 1) / (4 * tiles64);
        int cl = weights < ((int64_t)1 << 24) ? 1 : want >= 8 ? 8 : want >= 4 ? 4 : want >= 2 ? 2 : 1;
        while (cl > 1 && max_steps / cl < 2) cl >>= 1;
        if (cl == 8) return batch >= 4 || KIND == kLut16
                                  ? prepare_variant<KIND, NB, 1, 1, FWC, MAXP, 8>(pr, probs, tiles_for(16 * FWC))
                                  : prepare_variant<KIND, NB, 1, 1, 4, MAXP, 8>(pr, probs, tiles_for(64));
        if (cl == 4) return batch >= 4 || KIND == kLut16
                                  ? prepare_variant<KIND, NB, 1, 1, FWC, MAXP, 4>(pr, probs, tiles_for(16 * FWC))
                                  : prepare_variant<KIND, NB, 1, 1, 4, MAXP, 4>(pr, probs, tiles_for(64));
        if (cl == 2) return batch >= 4 || KIND == kLut16
                                  ? prepare_variant<KIND, NB, 1, 1, FWC, MAXP, 2>(pr, probs, tiles_for(16 * FWC))
                                  : prepare_variant<KIND, NB, 1, 1, 4, MAXP, 2>(pr, probs, tiles_for(64));
    }
#endif
    if (rows16 >= 2 * sms) return prepare_variant<KIND, NB, 1, 2, 4, MAXP>(pr, probs, tiles_for(32));
    return prepare_variant<KIND, NB, 1, 4, 4, MAXP>(pr, probs, tiles_for(16));
}

template <int MAXP>
wq_status prepare(int fmt, int group, const GemvProblem* probs, int count, int batch,
                  Prepared<MAXP>& pr) {
    if (count < 1 || count > MAXP) return fail(WQ_EINVAL, "count=%d outside 1..%d", count, MAXP);
    GemvParams<MAXP>& prm = pr.prm;
    prm.count = count;
    prm.batch = batch;
    // Longest rows first (stable by K, descending): the grid is dispatched roughly in order,
    // so the last wave holds the shortest CTAs and the tail of the launch stays short.
    GemvProblem sorted[MAXP];
    for (int i = 0; i < count; ++i) {
        int j = i;
        while (j > 0 && sorted[j - 1].k < probs[i].k) { sorted[j] = sorted[j - 1]; --j; }
        sorted[j] = probs[i];
    }
    probs = sorted;
    int64_t rows16 = 0;
    for (int i = 0; i < count; ++i) { prm.prob[i] = probs[i]; rows16 += (probs[i].n + 15) / 16; }
    const bool two = batch > 8;
    const int kind = (fmt == WQ_FMT_LUT16) ? kLut16 : (fmt == WQ_FMT_LLOYD8S) ? kLloyd8
                   : (group == 64 ? kDyadic64 : kDyadic32);
    if (kind == kLut16)
        return two ? pick_split<kLut16, 2, MAXP>(pr, probs, count, rows16, batch)
                   : pick_split<kLut16, 1, MAXP>(pr, probs, count, rows16, batch);
    if (kind == kLloyd8)
        return two ? pick_split<kLloyd8, 2, MAXP>(pr, probs, count, rows16, batch)
                   : pick_split<kLloyd8, 1, MAXP>(pr, probs, count, rows16, batch);
    if (kind == kDyadic64)
        return two ? pick_split<kDyadic64, 2, MAXP>(pr, probs, count, rows16, batch)
                   : pick_split<kDyadic64, 1, MAXP>(pr, probs, count, rows16, batch);
    return two ? pick_split<kDyadic32, 2, MAXP>(pr, probs, count, rows16, batch)
               : pick_split<kDyadic32, 1, MAXP>(pr, probs, count, rows16, batch);
}

template <int MAXP>
wq_status launch_prepared(const Prepared<MAXP>& pr, cudaStream_t s) {
    if (pr.cl == 1 && !pr.overlap) {
        pr.kern<<<pr.tiles, pr.threads, pr.smem, s>>>(pr.prm);
        return check_launch("gemv");
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pr.tiles * pr.cl);
    cfg.blockDim = dim3(pr.threads);
    cfg.dynamicSmemBytes = pr.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pr.cl > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = pr.cl;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pr.overlap) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    cudaLaunchKernelEx(&cfg, pr.kern, pr.prm);
    return check_launch(pr.cl > 1 ? "gemv (cluster)" : "gemv");
}

template <int MAXP>
wq_status launch_impl(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    Prepared<MAXP> pr;
    wq_status st = prepare<MAXP>(fmt, group, probs, count, batch, pr);
    if (st != WQ_OK) return st;
    return launch_prepared(pr, s);
}

}  // namespace

wq_status launch_gemv(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s) {
    if (count == 1) return launch_impl<1>(fmt, group, probs, count, batch, s);
    return launch_impl<kMaxProblems>(fmt, group, probs, count, batch, s);
}

wq_status gemv_plan_build(int fmt, int group, const GemvProblem* probs, int count, int batch,
                          void** plan) {
    auto* pr = new (std::nothrow) Prepared<kMaxProblems>;
    if (!pr) return fail(WQ_EINVAL, "out of host memory for the GEMV plan");
    wq_status st = prepare<kMaxProblems>(fmt, group, probs, count, batch, *pr);
    if (st != WQ_OK) { delete pr; return st; }
    *plan = pr;
    return WQ_OK;
}

void gemv_plan_set_overlap(void* plan, bool on) {
    static_cast<Prepared<kMaxProblems>*>(plan)->overlap = on;
}

wq_status gemv_plan_launch(const void* plan, cudaStream_t s) {
    return launch_prepared(*static_cast<const Prepared<kMaxProblems>*>(plan), s);
}

void gemv_plan_free(void* plan) { delete static_cast<Prepared<kMaxProblems>*>(plan); }

}  // namespace wq
