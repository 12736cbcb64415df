// wq_lloyd.cu -- codebook producers.
//
//  * Lloyd g32 with warm start, "int4-g32+warm 裸量化：原理与实验报告" §1.2-1.3, §2, §5.1:
//    per group of 32 magnitudes, the best of 112 candidate shapes (f-space 8-level
//    uniform quantisation, reconstruction through the inverse, group MSE) gives the
//    initial 8 levels; Lloyd rounds refine them; the sign is kept as bit 3 of the code.
//  * 16-centroid k-means per block of 64, "K-Means量化技术…" §1.2 (the LUT16 format).
//
// One warp per group. Lloyd g32 takes its candidate decision in two passes:
//  1. a fp32 screen, lane = candidate, on magnitudes normalised by the group maximum (the
//     shape family is scale-covariant after that, which keeps tiny and huge groups in
//     range). Besides each candidate's fp32 squared-error sum it bounds the exact sum from
//     both sides: the fp32 transforms and levels carry a bounded error, so a weight whose
//     f-space position lies within that error of a rounding boundary may belong to either
//     neighbouring level (both squared errors are kept), and the level and summation errors
//     widen the interval further (constants and their derivation at kEpsX below);
//  2. every candidate whose lower bound does not exceed the smallest upper bound -- a set
//     that provably holds the exact argmin -- is evaluated again in fp64, lane = weight,
//     with the reference steps (rint(f / fmax * 7), levels by the inverse, squared errors
//     summed in index order). The lowest fp64 MSE wins, the lowest candidate on a tie.
// The Lloyd rounds then run in fp64 with lane = weight. Each level's member sum is taken
// in index order (lane j walks the members of level j), so the rounds repeat the
// reference's arithmetic operation for operation. k-means does the same in fp64 for its
// 16 centroids. Both stop early once an assignment repeats (a fixed point: later rounds
// are identical).
#include <cmath>

#include "wq_internal.cuh"

namespace wq {

WQ_DEBUG_WORD(lloyd)
namespace {

constexpr int kCand = 112;
constexpr int kRational = 105;

struct CandTable {
    double brel[kCand];
    double beta[kCand];
    float brel_f[kCand];
    float beta_f[kCand];
    float log2_brel_f[kCand];
};

CandTable make_table() {
    static const double kBeta[7] = {0.50, 0.55, 0.65, 0.75, 0.85, 0.95, 1.00};
    static const double kTanh[7] = {0.25, 0.4, 0.6, 0.85, 1.2, 1.8, 3.0};
    CandTable t;
    for (int c = 0; c < kCand; ++c) {
        double br, be;
        if (c < kRational) {
            br = std::pow(10.0, -3.0 + 5.0 * (c / 7) / 14.0);   // logspace(-3, 2, 15)
            be = kBeta[c % 7];
        } else {
            br = kTanh[c - kRational];
            be = 1.0;
        }
        t.brel[c] = br;
        t.beta[c] = be;
        t.brel_f[c] = (float)br;
        t.beta_f[c] = (float)be;
        t.log2_brel_f[c] = (float)std::log2(br);
    }
    return t;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Root of v / (kappa + v^beta) = phi (beta < 1) by Newton on the concave increasing
// function u - log(kappa + e^(beta u)) - log(phi) of u = log v, started at the lower bound
// v = phi * kappa (monotone convergence). fp32, for screening.
__device__ __forceinline__ float inv_rational_f32(float phi, float kappa, float beta) {
    float u = __logf(phi * kappa);
    const float lphi = __logf(phi);
#pragma unroll 1
    for (int it = 0; it < 8; ++it) {
        const float e = __expf(beta * u);
        const float d = (kappa + (1.f - beta) * e) / (kappa + e);
        u -= (u - __logf(kappa + e) - lphi) / d;
    }
    return __expf(u);
}

// The same root in fp64, unnormalised (L / (b + L^beta) = fd), refined in linear space.
__device__ double inv_rational_f64(double fd, double b, double beta) {
    double u = log(fd * b);
    const double lfd = log(fd);
    for (int it = 0; it < 12; ++it) {
        const double e = exp(beta * u);
        const double d = (b + (1.0 - beta) * e) / (b + e);
        const double du = (u - log(b + e) - lfd) / d;
        u -= du;
        if (fabs(du) < 1e-15) break;
    }
    double L = exp(u);
    for (int it = 0; it < 2; ++it) {              // h(L) = L - fd b - fd L^beta, h' > 0 here
        const double p = pow(L, beta);
        const double h = L - fd * b - fd * p;
        const double hp = 1.0 - fd * beta * p / L;
        L -= h / hp;
    }
    return L;
}

// fp64 -> fp16 bits with a single rounding (to nearest even).
__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
    unsigned short h;
    asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
    return h;
}
__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
    return (double)__half2float(__ushort_as_half(h));
}

__device__ __forceinline__ double transform64(int fam, double a, double b, double beta) {
    return fam == 0 ? a / (b + pow(a, beta)) : tanh(a / b);
}

constexpr int kWarps = 8;

// Error model of the fp32 screen, in the normalised units (u = a / gmax in [0, 1], levels
// in [0, 1], x = 7 f(u) / f(1) in [0, 7]):
//  * x: the rational family forms u^beta and kappa = b_rel gmax^(1-beta) as exp2 of a
//    product with a log2 (|log2| <= 133 for bf16 magnitudes, a few ulp each), then one
//    correctly rounded division; tanh takes two tanhf calls and one division. Both stay
//    below 5e-5 relative; the screen assumes |x - x_exact| <= kEpsX x + kEtaX (kEpsX =
//    2.4e-4, about 5x that), and treats a weight within that distance of a half-integer
//    as belonging to either neighbouring level.
//  * levels: closed forms (beta = 1, tanh) and an 8-step log-space Newton iteration
//    (beta < 1) carry below 2e-5 relative; the screen assumes kEpsL absolute (levels are
//    at most 1), which moves each squared error by at most 2 kEpsL |d| + kEpsL^2.
//  * the fp32 sum of 32 fused multiply-adds: at most 32 * 2^-24 relative; kDelta is 4x.
constexpr float kEpsX = 1.0f / 4096.0f;      // 2^-12
constexpr float kEtaX = 1.0f / 1048576.0f;   // 2^-20
constexpr float kEpsL = 1.0f / 16384.0f;     // 2^-14
constexpr float kDelta = 1.0f / 131072.0f;   // 2^-17

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Sum over the 32 lanes in lane order (((v0 + v1) + v2) + ...), the order of a plain loop
// over the group's weights; every lane gets the result.
__device__ __forceinline__ double warp_sum_in_order(double v) {
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 32; ++i) s = __dadd_rn(s, __shfl_sync(0xFFFFFFFFu, v, i));
    return s;
}

// Candidate c on this group in fp64, the reference's steps: b = b_rel gmax, fmax = f(gmax),
// q = clamp(rint(f(a) / fmax * 7), 0, 7), levels L_0 = 0, L_q = f^-1(q / 7 * fmax), L_7 = gmax,
// MSE = (sum over the group in index order of (a - L_q)^2) / 32. Lane = weight; the whole
// warp calls it with the same c. Returns the MSE; L receives the 8 levels in every lane.
__device__ double candidate_mse64(int c, double a, double gmax, int lane, const CandTable& ct,
                                  double L[8]) {
    const int fam = c < kRational ? 0 : 1;
    const double beta = ct.beta[c];
    const double b = ct.brel[c] * gmax;
    const double fmx = transform64(fam, gmax, b, beta);
    double myL = 0.0;                                  // lane q (1..6) computes level q
    if (lane >= 1 && lane <= 6) {
        const double fd = (double)lane / 7.0 * fmx;
        if (fam == 1) myL = b * atanh(fd);
        else if (beta == 1.0) myL = fd * b / (1.0 - fd);
        else myL = inv_rational_f64(fd, b, beta);
    }
    if (lane == 7) myL = gmax;
#pragma unroll
    for (int q = 0; q < 8; ++q) L[q] = __shfl_sync(0xFFFFFFFFu, myL, q);
    const double f = transform64(fam, a, b, beta);
    double qq = rint(f / fmx * 7.0);
    qq = fmin(fmax(qq, 0.0), 7.0);
    const int qi = (int)qq;
    double sel = L[0];
#pragma unroll
    for (int q = 1; q < 8; ++q) sel = (qi == q) ? L[q] : sel;
    const double d = a - sel;
    return warp_sum_in_order(__dmul_rn(d, d)) / 32.0;
}

__global__ void __launch_bounds__(kWarps * 32)
lloyd_g32_kernel(const uint16_t* __restrict__ w, int64_t n_groups, int rounds,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ packed,
                 float* __restrict__ levels_out, uint8_t* __restrict__ params_out,
                 float* __restrict__ trace_out, const __grid_constant__ CandTable ct) {
    __shared__ float s_u[kWarps][32];            // normalised magnitudes a / gmax
    __shared__ float s_pw[kWarps][6][32];        // u^beta for the six beta < 1
    __shared__ float s_lv[kWarps][32 * 9];       // per-lane level tables, stride 9
    __shared__ float s_lo[kWarps][128];          // per-candidate bounds of the exact
    __shared__ float s_hi[kWarps][128];          // normalised squared-error sum
    __shared__ double s_a[kWarps][32];           // magnitudes, for the in-order member sums
    const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * kWarps;
    const int T = rounds + 2;

    for (int64_t g = (int64_t)blockIdx.x * kWarps + wi; g < n_groups; g += warps_total) {
        const uint32_t hb = w[g * 32 + lane];
        WQ_DCHECK((hb & 0x7F80u) != 0x7F80u, kDbgNonFiniteWeight + 2);
        const float wf = bf16_bits_to_float(hb);
        const float af = fabsf(wf);
        const int sgn = wf < 0.f ? 1 : 0;                 // -0.0 counts as positive
        const float gmaxf = warp_max(af);
        if (gmaxf == 0.f) {
            const uint8_t code = 0;
            if (codes) codes[g * 32 + lane] = code;
            if (packed && (lane & 1) == 0) packed[g * 16 + lane / 2] = 0;
            if (lane < 8) levels_out[g * 8 + lane] = 0.f;
            if (params_out && lane == 0) params_out[g] = 0;
            if (trace_out)
                for (int t = lane; t < T; t += 32) trace_out[g * T + t] = 0.f;
            continue;
        }
        // ---- 1. fp32 screen with bounds, lane = candidate -------------------------------
        const float u = af / gmaxf;
        s_u[wi][lane] = u;
        const float l2u = __log2f(u);
#pragma unroll
        for (int t = 0; t < 6; ++t) s_pw[wi][t][lane] = (u > 0.f) ? exp2f(ct.beta_f[t] * l2u) : 0.f;
        __syncwarp();
        const float l2g = __log2f(gmaxf);
        float* lv = &s_lv[wi][lane * 9];
        for (int c = lane; c < kCand; c += 32) {
            const bool rat = c < kRational;
            const int t = c % 7;
            const float beta = ct.beta_f[c];
            float kappa, scale7;
            if (rat) {
                // b = b_rel gmax;  f(a)/fmax = F(u)/F(1), F(u) = u / (kappa + u^beta),
                // kappa = b_rel gmax^(1 - beta)
                kappa = (t == 6) ? ct.brel_f[c] : exp2f(ct.log2_brel_f[c] + (1.f - beta) * l2g);
                scale7 = 7.f * (kappa + 1.f);             // 7 / F(1)
                lv[0] = 0.f;
                lv[7] = 1.f;
                const float fmaxn = 1.f / (kappa + 1.f);
                for (int q = 1; q < 7; ++q) {
                    const float phi = (float)q / 7.f * fmaxn;
                    lv[q] = (t == 6) ? phi * kappa / (1.f - phi) : inv_rational_f32(phi, kappa, beta);
                }
            } else {
                const float br = ct.brel_f[c];            // F(u) = tanh(u / b_rel)
                const float fmaxn = tanhf(1.f / br);
                kappa = br;
                scale7 = 7.f / fmaxn;
                lv[0] = 0.f;
                lv[7] = 1.f;
                for (int q = 1; q < 7; ++q) lv[q] = br * atanhf((float)q / 7.f * fmaxn);
            }
            float se = 0.f, sabs = 0.f, spread = 0.f;
            for (int i = 0; i < 32; ++i) {
                const float ui = s_u[wi][i];
                float F;
                if (rat) F = ui / (kappa + (t == 6 ? ui : s_pw[wi][t][i]));
                else F = tanhf(ui / kappa);
                const float xs = F * scale7;
                const float qf = fminf(fmaxf(rintf(xs), 0.f), 7.f);
                const float d = ui - lv[(int)qf];
                se = fmaf(d, d, se);
                // a rounding decision within the screen's error of a half-integer could go
                // either way: keep the other neighbour's squared error too
                const float fl = floorf(xs);
                float da = d;
                if (fabsf(xs - fl - 0.5f) <= fmaf(kEpsX, xs, kEtaX)) {
                    const float qa = fminf(fmaxf(qf == fl ? fl + 1.f : fl, 0.f), 7.f);
                    da = ui - lv[(int)qa];
                    spread += fabsf(fmaf(da, da, -(d * d)));
                }
                sabs += fmaxf(fabsf(d), fabsf(da));
            }
            const float slack = fmaf(2.f * kEpsL, sabs, 32.f * kEpsL * kEpsL) + spread * (1.f + kDelta);
            s_lo[wi][c] = fmaf(-kDelta, se, se) - slack;
            s_hi[wi][c] = fmaf(kDelta, se, se) + slack;
        }
        __syncwarp();
        // smallest upper bound: the exact argmin's lower bound cannot lie above it
        float thr = INFINITY;
        for (int c = lane; c < kCand; c += 32) thr = fminf(thr, s_hi[wi][c]);
        thr = warp_min(thr);

        // ---- 2. fp64 re-evaluation of every candidate that can still be the argmin ------
        const double a = (double)af, gmax = (double)gmaxf;
        double L[8], best = INFINITY;
        int c = 0;
#pragma unroll 1
        for (int base = 0; base < kCand; base += 32) {
            const int cl = base + lane;
            // (a NaN bound, which the screen should never produce, keeps its candidate)
            unsigned m = __ballot_sync(0xFFFFFFFFu, cl < kCand && !(s_lo[wi][cl] > thr));
            while (m) {
                const int cc = base + __ffs(m) - 1;
                WQ_DCHECK(cc < kCand, kDbgIndex + 30);
                m &= m - 1;
                double Lc[8];
                const double mse = candidate_mse64(cc, a, gmax, lane, ct, Lc);
                if (mse < best) {                          // increasing cc: lowest on a tie
                    best = mse;
                    c = cc;
#pragma unroll
                    for (int q = 0; q < 8; ++q) L[q] = Lc[q];
                }
            }
        }
        if (trace_out && lane == 0) trace_out[g * T] = (float)best;

        // ---- 3. Lloyd rounds in fp64, lane = weight --------------------------------------
        s_a[wi][lane] = a;
        __syncwarp();
        int q = 0, prev_q = -1;
        double mse = 0.0;
        for (int t = 0; t <= rounds; ++t) {
            double bd = fabs(a - L[0]);
            q = 0;
#pragma unroll
            for (int j = 1; j < 8; ++j) {
                const double d = fabs(a - L[j]);
                if (d < bd) { bd = d; q = j; }
            }
            const double se = warp_sum(__dmul_rn(bd, bd));
            mse = se / 32.0;
            if (trace_out && lane == 0) trace_out[g * T + 1 + t] = (float)mse;
            const bool same = __all_sync(0xFFFFFFFFu, q == prev_q);
            if (t == rounds) break;
            if (same) {                                   // fixed point: the rest repeats
                if (trace_out && lane == 0)
                    for (int t2 = t + 1; t2 <= rounds; ++t2) trace_out[g * T + 1 + t2] = (float)mse;
                break;
            }
            prev_q = q;
            // level j <- mean of its members, summed in index order by lane j; an empty
            // level keeps its value
            unsigned mine = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const unsigned mj = __ballot_sync(0xFFFFFFFFu, q == j);
                mine = (lane == j) ? mj : mine;
            }
            const int cnt = __popc(mine);
            double s = 0.0;
            while (mine) {
                s = __dadd_rn(s, s_a[wi][__ffs(mine) - 1]);
                mine &= mine - 1;
            }
            double old = L[0];
#pragma unroll
            for (int j = 1; j < 8; ++j) old = (lane == j) ? L[j] : old;
            const double nl = cnt > 0 ? s / (double)cnt : old;
#pragma unroll
            for (int j = 0; j < 8; ++j) L[j] = __shfl_sync(0xFFFFFFFFu, nl, j);
        }
        __syncwarp();
        const uint32_t code = (uint32_t)q | ((uint32_t)sgn << 3);
        if (codes) codes[g * 32 + lane] = (uint8_t)code;
        const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, code, 1);
        if (packed && (lane & 1) == 0) packed[g * 16 + lane / 2] = (uint8_t)(code | (other << 4));
        if (lane < 8) {
            double lvq = L[0];
#pragma unroll
            for (int j = 1; j < 8; ++j) lvq = (lane == j) ? L[j] : lvq;
            levels_out[g * 8 + lane] = (float)lvq;
        }
        if (params_out && lane == 0)
            params_out[g] = (uint8_t)(c < kRational ? (((c / 7) << 3) | (c % 7)) : (0x80 | ((c - kRational) << 3)));
    }
}

// ---------------------------------------------------------------------------------------
// k-means, 16 centroids per block of 64, fp64. Lane l holds values l and l + 32, so that
// the two ballots of a centroid's members are the low and high halves of its membership
// mask in index order.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kWarps * 32)
kmeans16_kernel(const uint16_t* __restrict__ w, int64_t n_blocks, int rounds,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ packed,
                uint16_t* __restrict__ lut, float* __restrict__ trace_out) {
    __shared__ double s_v[kWarps][64];
    __shared__ double s_c[kWarps][16];
    const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * kWarps;
    const int T = rounds + 1;
    for (int64_t g = (int64_t)blockIdx.x * kWarps + wi; g < n_blocks; g += warps_total) {
        WQ_DCHECK((w[g * 64 + lane] & 0x7F80u) != 0x7F80u && (w[g * 64 + 32 + lane] & 0x7F80u) != 0x7F80u,
                  kDbgNonFiniteWeight + 3);
        const double v0 = (double)bf16_bits_to_float(w[g * 64 + lane]);
        const double v1 = (double)bf16_bits_to_float(w[g * 64 + 32 + lane]);
        s_v[wi][lane] = v0;
        s_v[wi][lane + 32] = v1;
        __syncwarp();
        // initial centroid i = the (4i+2)-th smallest value (rank with index tie-break)
        int r0 = 0, r1 = 0;
        const int i0 = lane, i1 = lane + 32;
        for (int m = 0; m < 64; ++m) {
            const double vm = s_v[wi][m];
            r0 += (vm < v0) || (vm == v0 && m < i0);
            r1 += (vm < v1) || (vm == v1 && m < i1);
        }
        WQ_DCHECK(r0 < 64 && r1 < 64 && r0 != r1, kDbgIndex + 31);
        if ((r0 & 3) == 2) s_c[wi][r0 >> 2] = v0;
        if ((r1 & 3) == 2) s_c[wi][r1 >> 2] = v1;
        __syncwarp();
        double cen[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) cen[j] = s_c[wi][j];
        int q0 = 0, q1 = 0, p0 = -1, p1 = -1;
        for (int t = 0; t <= rounds; ++t) {
            if (t == rounds) {
#pragma unroll
                for (int j = 0; j < 16; ++j) cen[j] = f16_bits_to_f64(f64_to_f16_bits(cen[j]));
            }
            double b0 = fabs(v0 - cen[0]), b1 = fabs(v1 - cen[0]);
            q0 = q1 = 0;
#pragma unroll
            for (int j = 1; j < 16; ++j) {
                const double d0 = fabs(v0 - cen[j]), d1 = fabs(v1 - cen[j]);
                if (d0 < b0) { b0 = d0; q0 = j; }
                if (d1 < b1) { b1 = d1; q1 = j; }
            }
            const double se = warp_sum(__dadd_rn(__dmul_rn(b0, b0), __dmul_rn(b1, b1)));
            if (trace_out && lane == 0) trace_out[g * T + t] = (float)(se / 64.0);
            if (t == rounds) break;
            const bool same = __all_sync(0xFFFFFFFFu, q0 == p0 && q1 == p1);
            if (same) {                                   // fixed point until the final step
                if (trace_out && lane == 0)
                    for (int t2 = t + 1; t2 < rounds; ++t2) trace_out[g * T + t2] = (float)(se / 64.0);
                t = rounds - 1;                           // go straight to the final step
                continue;
            }
            p0 = q0;
            p1 = q1;
            // centroid j <- mean of its members, summed in index order by lane j (values
            // 0..31, then 32..63); an empty centroid keeps its value
            unsigned lo = 0, hi = 0;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const unsigned mlo = __ballot_sync(0xFFFFFFFFu, q0 == j);
                const unsigned mhi = __ballot_sync(0xFFFFFFFFu, q1 == j);
                lo = (lane == j) ? mlo : lo;
                hi = (lane == j) ? mhi : hi;
            }
            const int cnt = __popc(lo) + __popc(hi);
            double s = 0.0;
            while (lo) {
                s = __dadd_rn(s, s_v[wi][__ffs(lo) - 1]);
                lo &= lo - 1;
            }
            while (hi) {
                s = __dadd_rn(s, s_v[wi][32 + __ffs(hi) - 1]);
                hi &= hi - 1;
            }
            if (lane < 16 && cnt > 0) s_c[wi][lane] = s / (double)cnt;
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 16; ++j) cen[j] = s_c[wi][j];
            __syncwarp();
        }
        if (codes) {
            codes[g * 64 + lane] = (uint8_t)q0;
            codes[g * 64 + 32 + lane] = (uint8_t)q1;
        }
        // byte l = code[2l] | code[2l+1] << 4: codes 2l, 2l+1 sit in lanes (2l) mod 32 and
        // the next, as their first value below 32 and as their second from 32 on
        const int src = (2 * lane) & 31;
        const int a0 = __shfl_sync(0xFFFFFFFFu, q0, src), a1 = __shfl_sync(0xFFFFFFFFu, q0, src + 1);
        const int c0 = __shfl_sync(0xFFFFFFFFu, q1, src), c1 = __shfl_sync(0xFFFFFFFFu, q1, src + 1);
        if (packed) packed[g * 32 + lane] = (uint8_t)(lane < 16 ? (a0 | (a1 << 4)) : (c0 | (c1 << 4)));
        if (lane < 16) lut[g * 16 + lane] = f64_to_f16_bits(s_c[wi][lane]);
        __syncwarp();
    }
}

int producer_grid(int64_t groups) {
    int64_t blocks = (groups + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * 8;
    return (int)(blocks < cap ? (blocks < 1 ? 1 : blocks) : cap);
}

}  // namespace

wq_status launch_lloyd_g32(const uint16_t* w, int64_t n, int64_t k, int rounds, uint8_t* codes,
                           uint8_t* packed, float* levels, uint8_t* params, float* trace,
                           cudaStream_t s) {
    static const CandTable table = make_table();
    const int64_t groups = n * k / 32;
    lloyd_g32_kernel<<<producer_grid(groups), kWarps * 32, 0, s>>>(w, groups, rounds, codes, packed,
                                                                   levels, params, trace, table);
    return check_launch("lloyd_g32");
}

wq_status launch_kmeans16(const uint16_t* w, int64_t n, int64_t k, int rounds, uint8_t* codes,
                          uint8_t* packed, uint16_t* lut, float* trace, cudaStream_t s) {
    const int64_t blocks = n * k / 64;
    kmeans16_kernel<<<producer_grid(blocks), kWarps * 32, 0, s>>>(w, blocks, rounds, codes, packed,
                                                                  lut, trace);
    return check_launch("kmeans16");
}

}  // namespace wq
