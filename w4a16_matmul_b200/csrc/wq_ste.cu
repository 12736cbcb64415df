// wq_ste.cu -- STE fake quantisation, forward ("MiniCPM5-1B 验证: 6× 压缩…" §2.3 "STE").
//
// A QAT step keeps an fp32 latent z per weight and the block's bf16 scale; its forward pass
// replaces z by the nearest dyadic code value, q = step * (idx - 8), step = scale / 8, with
// idx = argmin_j |z - step * (j - 8)| (lowest index on a tie), and its backward pass passes
// the gradient through unchanged (the straight-through estimator), which needs no kernel.
// The same pass can emit the codes or the packed nibbles: the deployment path "z -> hard
// argmin -> level_idx -> pack" of §2.5.
//
// HBM-bound stream: 4 B read, 4 B written per element (plus 1 B or 0.5 B of codes when asked).
//
// The same file holds the backward of the page's other estimator, Gumbel-ST (§2.3):
// soft = softmax(-dist/tau) . codes, hard = codes[argmin dist], q = hard + (soft - soft.detach()),
// dist_j = (z - codes_j)^2. Its forward value is hard (the STE forward above); its backward,
// for an upstream gradient gq, is gz = gq * d soft/d z per element and, per group,
// gscale = sum gq * (d hard/d scale + d soft/d scale) (the codes are step * (j - 8) with
// step = scale / 8, a function of the trained scale). With p the softmax weights and
// u_j = j - idx the code offset from the nearest code, both derivatives are moments of p:
//   d soft/d z     = (2/tau) step^2 M2,                     M2 = sum p (u - mu)^2
//   d soft/d scale = (mu + idx - 8)/8
//                    + (2/tau) (step/8) ((z - 2 c_idx - 2 step mu) M2 - step M3),
// mu = sum p u, M3 = sum p (u - mu)^3 (p normalised), c_idx = step (idx - 8). The weights
// come from their logits relative to the nearest code, log2 p_j = u (A - B u) with
// A = 2 (z - c_idx) step log2(e)/tau and B = step^2 log2(e)/tau, so no term is a difference
// of two large numbers, and the central moments stay accurate in fp32 at any temperature.
// Per element: 16 ex2 on the special-function unit and 9 fp32 operations per code, issued
// two elements at a time as packed fp32x2 instructions; the special-function unit (16 ex2
// per element) then bounds the kernel, not HBM (12 B per element).
#include "wq_internal.cuh"

namespace wq {

WQ_DEBUG_WORD(ste)
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float rcp_fast(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// idx for one element, idx = #{j in 1..15 : z > m_j} with m_j = (2j - 17) s / 16.
//   Fast path (s in [2^-96, 2^96]): every m_j is exact in fp32 (an 8-bit significand times an
//   odd integer <= 17, over 16). u = 8 z / s + 8.5, clamped to [0, 16.5], approximates the
//   real count boundary to better than 2^-18, so ceil(u) - 1 is the count or one off either
//   way; one exact comparison each way settles it.
//   Other scales: the count itself, with each midpoint formed exactly in double.
// The index as a float (an exact small integer): the callers form the code value from it
// without an int-to-float conversion, and the integer code as float_as_uint(x + 2^23) & 15.
__device__ __forceinline__ float ste_index_f(float z, float s, float c8, float s8, float m17,
                                             bool fast) {
    if (s == 0.0f) return 0.0f;                                // every code ties
    if (fast) {
        const float u = fminf(fmaxf(fmaf(z, c8, 8.5f), 0.0f), 16.5f);
        float x = fminf(fmaxf(__fadd_ru(u, 8388608.0f) - 8388609.0f, 0.0f), 15.0f);
        if (x > 0.0f && !(z > fmaf(x, s8, m17))) x -= 1.0f;               // z <= m_x
        else if (x < 15.0f && z > fmaf(x + 1.0f, s8, m17)) x += 1.0f;     // z > m_{x+1}
        return x;
    }
    const double sd = (double)s, zd = (double)z;
    float n = 0.0f;
#pragma unroll
    for (int j = 1; j < 16; ++j) n += zd > (double)(2 * j - 17) * sd * 0.0625 ? 1.0f : 0.0f;
    return n;
}

__device__ __forceinline__ uint32_t index_bits(float x) { return __float_as_uint(x + 8388608.0f) & 15u; }

// One thread: 8 consecutive elements (one quarter or eighth of a group), U such blocks in
// flight, grid-stride.
__global__ void __launch_bounds__(kThreads)
fake_quant_ste_kernel(const float4* __restrict__ z, const uint16_t* __restrict__ scale, int64_t n8,
                      int group, float4* __restrict__ q, uint2* __restrict__ codes,
                      uint32_t* __restrict__ packed) {
    constexpr int U = 2;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int per_group = group / 8;
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n8; i0 += stride * U) {
        float4 a[U], b[U];
        uint32_t sc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            a[u] = b[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            sc[u] = 0;
            if (i < n8) {
                const uint4 va = ldg_nc_v4(z + 2 * i), vb = ldg_nc_v4(z + 2 * i + 1);
                WQ_DCHECK(f32x4_finite(va) && f32x4_finite(vb), kDbgNonFiniteLatent + 1);
                a[u] = make_float4(__uint_as_float(va.x), __uint_as_float(va.y), __uint_as_float(va.z), __uint_as_float(va.w));
                b[u] = make_float4(__uint_as_float(vb.x), __uint_as_float(vb.y), __uint_as_float(vb.z), __uint_as_float(vb.w));
                sc[u] = ldg_u16(scale + i / per_group);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t i = i0 + u * stride;
            if (i >= n8) break;
            const float s = bf16_bits_to_float(sc[u]);
            const bool fast = s >= 0x1p-96f && s <= 0x1p96f;
            const float c8 = fast ? 8.0f * rcp_fast(s) : 0.0f;
            const float s8 = s * 0.125f, m17 = -17.0f * s * 0.0625f;
            const float zv[8] = {a[u].x, a[u].y, a[u].z, a[u].w, b[u].x, b[u].y, b[u].z, b[u].w};
            uint32_t idx[8];
            float qv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float xf = ste_index_f(zv[j], s, c8, s8, m17, fast);
                idx[j] = index_bits(xf);
                // the code value: exact in fp32 on the fast path; otherwise the double value
                // rounded once, as the definition reads
                qv[j] = fast ? s8 * (xf - 8.0f) : (float)((double)s * 0.125 * (double)(xf - 8.0f));
            }
            stg_cs_v4(q + 2 * i, make_uint4(__float_as_uint(qv[0]), __float_as_uint(qv[1]),
                                            __float_as_uint(qv[2]), __float_as_uint(qv[3])));
            stg_cs_v4(q + 2 * i + 1, make_uint4(__float_as_uint(qv[4]), __float_as_uint(qv[5]),
                                                __float_as_uint(qv[6]), __float_as_uint(qv[7])));
            if (codes)
                codes[i] = make_uint2(idx[0] | idx[1] << 8 | idx[2] << 16 | idx[3] << 24,
                                      idx[4] | idx[5] << 8 | idx[6] << 16 | idx[7] << 24);
            if (packed)
                packed[i] = idx[0] | idx[1] << 4 | idx[2] << 8 | idx[3] << 12 | idx[4] << 16 |
                            idx[5] << 20 | idx[6] << 24 | idx[7] << 28;
        }
    }
}

__device__ __forceinline__ float ex2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Two elements of the Gumbel-ST backward (formulas at the top of this file) on the packed
// fp32x2 pipe. The moments are taken in one pass as raw moments about the nearest code,
// E[u^k] = sum p u^k / sum p, and centred afterwards: u stays within [-15, 15], so the
// centring loses at most a few bits, far inside the tolerance. Both elements share the
// group's step.  l2t = 2 log2(e) / tau, r2 = 2 / tau.
__device__ __forceinline__ void gumbel_st_pair(float2 z, float2 up, float s, float c8, float step,
                                               float m17, bool fast, float l2t, float r2,
                                               float2& gz, float2& gs) {
    const float2 fi = make_float2(ste_index_f(z.x, s, c8, step, m17, fast),
                                  ste_index_f(z.y, s, c8, step, m17, fast));
    const float2 c_idx = __fmul2_rn(f2(step), __fadd2_rn(fi, f2(-8.0f)));
    const float2 e = __fadd2_rn(z, make_float2(-c_idx.x, -c_idx.y));
    const float B = step * step * (0.5f * l2t);
    float2 mu, m2, m3;
    if (B > 0x1p-6f) {
        // weights concentrated near the nearest code: logits and moments about it
        const float2 A = __fmul2_rn(e, f2(step * l2t));
        const float2 nB = f2(-B);
        const float2 nfi = make_float2(-fi.x, -fi.y);
        float2 s0 = f2(0.0f), s1 = f2(0.0f), s2 = f2(0.0f), s3 = f2(0.0f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float2 u = __fadd2_rn(f2((float)j), nfi);
            const float2 arg = __fmul2_rn(u, __ffma2_rn(nB, u, A));
            const float2 p = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            s0 = __fadd2_rn(s0, p);
            const float2 pu = __fmul2_rn(p, u);
            s1 = __fadd2_rn(s1, pu);
            s2 = __ffma2_rn(pu, u, s2);
            s3 = __ffma2_rn(__fmul2_rn(pu, u), u, s3);
        }
        // s0 is in [1, 16]: the nearest code has weight 1
        const float2 inv = make_float2(rcp_approx(s0.x), rcp_approx(s0.y));
        mu = __fmul2_rn(s1, inv);
        const float2 e2 = __fmul2_rn(s2, inv), e3 = __fmul2_rn(s3, inv);
        m2 = __ffma2_rn(make_float2(-mu.x, -mu.y), mu, e2);                          // E[u^2] - mu^2
        // E[u^3] - 3 mu E[u^2] + 2 mu^3 = E[u^3] - mu (3 E[u^2] - 2 mu^2)
        m3 = __ffma2_rn(make_float2(-mu.x, -mu.y),
                        __ffma2_rn(f2(-2.0f), __fmul2_rn(mu, mu), __fmul2_rn(f2(3.0f), e2)), e3);
    } else {
        // B <= 2^-6 (the page's temperatures on weight-scale latents): log2 p_j varies by at
        // most 225 B over the 16 codes within the scale, so the weights are spread and the
        // logits are a quadratic in the code index j (constant coefficients per element;
        // rounding error below 1e-5 in the exponent), with the moments accumulated about the fixed centre
        // j' = j - 7.5 (constant powers of j'; the spread distribution keeps the centring to
        // a few lost bits). With f = z + 8 step: log2 p_j - log2 p_idx =
        //   -B j^2 + 2 K f step j + K (e^2 - f^2),  K = log2(e) / tau,
        // and K (e^2 - f^2) = -K step idx (e + f) without cancellation.
        const float K = 0.5f * l2t;
        const float2 f = __ffma2_rn(f2(8.0f), f2(step), z);
        const float2 c1 = __fmul2_rn(f, f2(2.0f * K * step));
        const float2 c0 = __fmul2_rn(__fmul2_rn(fi, f2(-K * step)), __fadd2_rn(e, f));
        // The weights of consecutive codes have the ratio r_j = p_(j+1) / p_j =
        // 2^(c1 - B (2 j + 1)), and r_(j+1) = r_j * 2^(-2 B): every 4 codes an anchor takes p
        // and r from the special-function unit, the next 3 codes follow by multiplication
        // (at most 3 roundings and ex2 errors each: about 1e-6 relative), so 8 ex2 per
        // element are spent instead of 16.
        const float rho = ex2_approx(-2.0f * B);
        float2 s0 = f2(0.0f), s1 = f2(0.0f), s2 = f2(0.0f), s3 = f2(0.0f);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const float j0 = (float)(4 * a);
            const float2 arg = __ffma2_rn(__ffma2_rn(f2(-B), f2(j0), c1), f2(j0), c0);
            const float2 argr = __fadd2_rn(c1, f2(-B * (2.0f * j0 + 1.0f)));
            float2 p = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
            float2 r = make_float2(ex2_approx(argr.x), ex2_approx(argr.y));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float jc = j0 + (float)q - 7.5f;
                s0 = __fadd2_rn(s0, p);
                s1 = __ffma2_rn(p, f2(jc), s1);
                s2 = __ffma2_rn(p, f2(jc * jc), s2);
                s3 = __ffma2_rn(p, f2(jc * jc * jc), s3);
                if (q < 3) {
                    p = __fmul2_rn(p, r);
                    r = __fmul2_rn(r, f2(rho));
                }
            }
        }
        const float2 inv = make_float2(rcp_approx(s0.x), rcp_approx(s0.y));
        const float2 mc = __fmul2_rn(s1, inv);                                      // E[j'], about 7.5
        const float2 e2 = __fmul2_rn(s2, inv), e3 = __fmul2_rn(s3, inv);
        m2 = __ffma2_rn(make_float2(-mc.x, -mc.y), mc, e2);
        m3 = __ffma2_rn(make_float2(-mc.x, -mc.y),
                        __ffma2_rn(f2(-2.0f), __fmul2_rn(mc, mc), __fmul2_rn(f2(3.0f), e2)), e3);
        mu = __fadd2_rn(mc, __fadd2_rn(f2(7.5f), make_float2(-fi.x, -fi.y)));       // about idx
    }
    gz = __fmul2_rn(up, __fmul2_rn(f2((r2 * step) * step), m2));
    // z - 2 c_idx - 2 step mu
    const float2 lin = __ffma2_rn(f2(-2.0f * step), mu, __ffma2_rn(f2(-2.0f), c_idx, z));
    const float2 cov = __fmul2_rn(f2(step * 0.125f), __ffma2_rn(lin, m2, __fmul2_rn(f2(-step), m3)));
    // (idx - 8)/8 from the hard term plus (mu + idx - 8)/8 + (2/tau) cov from the soft one
    const float2 hard_soft = __fmul2_rn(__fadd2_rn(__ffma2_rn(f2(2.0f), fi, f2(-16.0f)), mu), f2(0.125f));
    gs = __fmul2_rn(up, __ffma2_rn(f2(r2), cov, hard_soft));
}

// One thread: 8 consecutive elements; the 8 (group 64) or 4 (group 32) threads of a group
// sit in adjacent lanes and add their scale gradients with shuffles. The loop runs on a
// warp-uniform index, so every lane reaches every shuffle; n8 is a multiple of the lanes
// per group, so the idle lanes of the last trip hold whole groups.
__global__ void __launch_bounds__(kThreads)
gumbel_st_backward_kernel(const float4* __restrict__ z, const uint16_t* __restrict__ scale,
                          const float4* __restrict__ gq, int64_t n8, int group, float l2t, float r2,
                          float4* __restrict__ gz, float* __restrict__ gscale) {
    const int lane = threadIdx.x & 31;
    const int per_group = group / 8;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < n8; base += stride) {
        const int64_t i = base + lane;
        float gsum = 0.0f;
        if (i < n8) {
            const uint4 za = ldg_nc_v4(z + 2 * i), zb = ldg_nc_v4(z + 2 * i + 1);
            const uint4 ga = ldg_nc_v4(gq + 2 * i), gb = ldg_nc_v4(gq + 2 * i + 1);
            WQ_DCHECK(f32x4_finite(za) && f32x4_finite(zb), kDbgNonFiniteLatent + 2);
            WQ_DCHECK(f32x4_finite(ga) && f32x4_finite(gb), kDbgNonFiniteLatent + 3);
            const float s = bf16_bits_to_float(ldg_u16(scale + i / per_group));
            const bool fast = s >= 0x1p-96f && s <= 0x1p96f;
            const float c8 = fast ? 8.0f * rcp_fast(s) : 0.0f;
            const float step = s * 0.125f, m17 = -17.0f * s * 0.0625f;
            const float2 zp[4] = {make_float2(__uint_as_float(za.x), __uint_as_float(za.y)),
                                  make_float2(__uint_as_float(za.z), __uint_as_float(za.w)),
                                  make_float2(__uint_as_float(zb.x), __uint_as_float(zb.y)),
                                  make_float2(__uint_as_float(zb.z), __uint_as_float(zb.w))};
            const float2 gp[4] = {make_float2(__uint_as_float(ga.x), __uint_as_float(ga.y)),
                                  make_float2(__uint_as_float(ga.z), __uint_as_float(ga.w)),
                                  make_float2(__uint_as_float(gb.x), __uint_as_float(gb.y)),
                                  make_float2(__uint_as_float(gb.z), __uint_as_float(gb.w))};
            uint32_t out[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 g, gsj;
                gumbel_st_pair(zp[j], gp[j], s, c8, step, m17, fast, l2t, r2, g, gsj);
                out[2 * j] = __float_as_uint(g.x);
                out[2 * j + 1] = __float_as_uint(g.y);
                gsum += gsj.x + gsj.y;
            }
            stg_cs_v4(gz + 2 * i, make_uint4(out[0], out[1], out[2], out[3]));
            stg_cs_v4(gz + 2 * i + 1, make_uint4(out[4], out[5], out[6], out[7]));
        }
        for (int off = 1; off < per_group; off <<= 1) gsum += __shfl_xor_sync(0xffffffffu, gsum, off);
        if (gscale && i < n8 && (lane & (per_group - 1)) == 0) gscale[i / per_group] = gsum;
    }
}

}  // namespace

wq_status launch_gumbel_st_backward(const float* z, int64_t n, int64_t k, int group,
                                    const uint16_t* scale, float tau, const float* gq, float* gz,
                                    float* gscale, cudaStream_t s) {
    const int64_t n8 = n * k / 8;
    int64_t blocks = (n8 + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    const double l2e = 1.4426950408889634;
    gumbel_st_backward_kernel<<<(int)(blocks < 1 ? 1 : blocks), kThreads, 0, s>>>(
        (const float4*)z, scale, (const float4*)gq, n8, group, (float)(2.0 * l2e / (double)tau),
        (float)(2.0 / (double)tau), (float4*)gz, gscale);
    return check_launch("gumbel_st_backward");
}

wq_status launch_fake_quant_ste(const float* z, int64_t n, int64_t k, int group,
                                const uint16_t* scale, float* q, uint8_t* codes, uint8_t* packed,
                                cudaStream_t s) {
    const int64_t n8 = n * k / 8;
    int64_t blocks = (n8 + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    fake_quant_ste_kernel<<<(int)(blocks < 1 ? 1 : blocks), kThreads, 0, s>>>(
        (const float4*)z, scale, n8, group, (float4*)q, (uint2*)codes, (uint32_t*)packed);
    return check_launch("fake_quant_ste");
}

}  // namespace wq
