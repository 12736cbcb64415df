// wq_lloyd.cu -- codebook producers.
//
//  * Lloyd g32 with warm start, "int4-g32+warm 裸量化：原理与实验报告" §1.2-1.3, §2, §5.1:
//    per group of 32 magnitudes, the best of 112 candidate shapes (f-space 8-level
//    uniform quantisation, reconstruction through the inverse, group MSE) gives the
//    initial 8 levels; Lloyd rounds refine them; the sign is kept as bit 3 of the code.
//  * 16-centroid k-means per block of 64, "K-Means量化技术…" §1.2 (the LUT16 format).
//
// One warp per group. Lloyd g32 screens the 112 candidates in fp32 with lane = candidate
// (the shape family is scale-covariant after normalising by the group maximum, which keeps
// tiny and huge groups in range), then recomputes the winner's levels in fp64 and runs
// the Lloyd rounds in fp64 with lane = weight, so the refinement takes the same decisions
// as a double-precision reference would. k-means runs entirely in fp64; member sums of
// bf16 values are exact in fp64, so centroids do not depend on summation order.
// Both stop early once an assignment repeats (a fixed point: later rounds are identical).
#include <cmath>

#include "wq_internal.cuh"

namespace wq {
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

__global__ void __launch_bounds__(kWarps * 32)
lloyd_g32_kernel(const uint16_t* __restrict__ w, int64_t n_groups, int rounds,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ packed,
                 float* __restrict__ levels_out, uint8_t* __restrict__ params_out,
                 float* __restrict__ trace_out, const __grid_constant__ CandTable ct) {
    __shared__ float s_u[kWarps][32];            // normalised magnitudes a / gmax
    __shared__ float s_pw[kWarps][6][32];        // u^beta for the six beta < 1
    __shared__ float s_lv[kWarps][32 * 9];       // per-lane level tables, stride 9
    const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * kWarps;
    const int T = rounds + 2;

    for (int64_t g = (int64_t)blockIdx.x * kWarps + wi; g < n_groups; g += warps_total) {
        const uint32_t hb = w[g * 32 + lane];
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
        // ---- fp32 screening, lane = candidate -----------------------------------------
        const float u = af / gmaxf;
        s_u[wi][lane] = u;
        const float l2u = __log2f(u);
#pragma unroll
        for (int t = 0; t < 6; ++t) s_pw[wi][t][lane] = (u > 0.f) ? exp2f(ct.beta_f[t] * l2u) : 0.f;
        __syncwarp();
        const float l2g = __log2f(gmaxf);
        float best = INFINITY;
        int bestc = 0;
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
            float se = 0.f;
            for (int i = 0; i < 32; ++i) {
                const float ui = s_u[wi][i];
                float F;
                if (rat) F = ui / (kappa + (t == 6 ? ui : s_pw[wi][t][i]));
                else F = tanhf(ui / kappa);
                const float qf = fminf(fmaxf(rintf(F * scale7), 0.f), 7.f);
                const float d = ui - lv[(int)qf];
                se = fmaf(d, d, se);
            }
            if (se < best) { best = se; bestc = c; }
        }
        // lowest MSE, lowest candidate index on a tie
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
            const int oc = __shfl_xor_sync(0xFFFFFFFFu, bestc, o);
            if (ob < best || (ob == best && oc < bestc)) { best = ob; bestc = oc; }
        }
        const int c = bestc;
        __syncwarp();

        // ---- fp64: the winner's levels, its candidate MSE, Lloyd -------------------------
        const double a = (double)af, gmax = (double)gmaxf;
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
        double L[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) L[q] = __shfl_sync(0xFFFFFFFFu, myL, q);
        // candidate MSE (the f-space assignment), for the trace
        {
            const double f = transform64(fam, a, b, beta);
            double qq = rint(f / fmx * 7.0);
            qq = fmin(fmax(qq, 0.0), 7.0);
            const int qi = (int)qq;
            double sel = L[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) sel = (qi == q) ? L[q] : sel;
            const double d = a - sel;
            const double se = warp_sum(d * d);
            if (trace_out && lane == 0) trace_out[g * T] = (float)(se / 32.0);
        }
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
            const double se = warp_sum(bd * bd);
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
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const unsigned m = __ballot_sync(0xFFFFFFFFu, q == j);
                const double s = warp_sum(q == j ? a : 0.0);
                if (m) L[j] = s / (double)__popc(m);
            }
        }
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
// k-means, 16 centroids per block of 64, fp64. Lane l holds values 2l and 2l+1.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kWarps * 32)
kmeans16_kernel(const uint32_t* __restrict__ w, int64_t n_blocks, int rounds,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ packed,
                uint16_t* __restrict__ lut, float* __restrict__ trace_out) {
    __shared__ double s_v[kWarps][64];
    __shared__ double s_c[kWarps][16];
    __shared__ double s_sum[kWarps][16];
    __shared__ int s_cnt[kWarps][16];
    const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t warps_total = (int64_t)gridDim.x * kWarps;
    const int T = rounds + 1;
    for (int64_t g = (int64_t)blockIdx.x * kWarps + wi; g < n_blocks; g += warps_total) {
        const uint32_t pair = w[g * 32 + lane];
        const double v0 = (double)bf16_bits_to_float(pair & 0xFFFF);
        const double v1 = (double)bf16_bits_to_float(pair >> 16);
        s_v[wi][2 * lane] = v0;
        s_v[wi][2 * lane + 1] = v1;
        __syncwarp();
        // initial centroid i = the (4i+2)-th smallest value (rank with index tie-break)
        int r0 = 0, r1 = 0;
        const int i0 = 2 * lane, i1 = 2 * lane + 1;
        for (int m = 0; m < 64; ++m) {
            const double vm = s_v[wi][m];
            r0 += (vm < v0) || (vm == v0 && m < i0);
            r1 += (vm < v1) || (vm == v1 && m < i1);
        }
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
            const double se = warp_sum(b0 * b0 + b1 * b1);
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
            if (lane < 16) { s_sum[wi][lane] = 0.0; s_cnt[wi][lane] = 0; }
            __syncwarp();
            atomicAdd(&s_sum[wi][q0], v0);
            atomicAdd(&s_sum[wi][q1], v1);
            atomicAdd(&s_cnt[wi][q0], 1);
            atomicAdd(&s_cnt[wi][q1], 1);
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (s_cnt[wi][j] > 0) cen[j] = s_sum[wi][j] / (double)s_cnt[wi][j];
            __syncwarp();
        }
        if (codes) {
            codes[g * 64 + 2 * lane] = (uint8_t)q0;
            codes[g * 64 + 2 * lane + 1] = (uint8_t)q1;
        }
        if (packed) packed[g * 32 + lane] = (uint8_t)(q0 | (q1 << 4));
        if (lane < 16) {
            double cv = cen[0];
#pragma unroll
            for (int j = 1; j < 16; ++j) cv = (lane == j) ? cen[j] : cv;
            lut[g * 16 + lane] = f64_to_f16_bits(cv);
        }
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
    kmeans16_kernel<<<producer_grid(blocks), kWarps * 32, 0, s>>>((const uint32_t*)w, blocks, rounds,
                                                                  codes, packed, lut, trace);
    return check_launch("kmeans16");
}

}  // namespace wq
