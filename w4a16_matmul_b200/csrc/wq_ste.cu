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
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float rcp_fast(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// idx for one element. idx = #{j in 1..15 : z > m_j} with m_j = (2j - 17) s / 16.
//   Fast path (s in [2^-96, 2^96]): every m_j is exact in fp32 (an 8-bit significand times an
//   odd integer <= 17, over 16). u = 8 z / s + 8.5, clamped to [0, 16.5], approximates the
//   real count boundary to better than 2^-18, so ceil(u) - 1 is the count or one off either
//   way; one exact comparison each way settles it.
//   Other scales: the count itself, with each midpoint formed exactly in double.
__device__ __forceinline__ uint32_t ste_index(float z, float s, float c8, float s8, float m17,
                                              bool fast) {
    if (s == 0.0f) return 0;                                   // every code ties
    if (fast) {
        const float u = fminf(fmaxf(fmaf(z, c8, 8.5f), 0.0f), 16.5f);
        float x = fminf(fmaxf(__fadd_ru(u, 8388608.0f) - 8388609.0f, 0.0f), 15.0f);
        if (x > 0.0f && !(z > fmaf(x, s8, m17))) x -= 1.0f;               // z <= m_x
        else if (x < 15.0f && z > fmaf(x + 1.0f, s8, m17)) x += 1.0f;     // z > m_{x+1}
        return __float_as_uint(x + 8388608.0f) & 15u;
    }
    const double sd = (double)s, zd = (double)z;
    uint32_t n = 0;
#pragma unroll
    for (int j = 1; j < 16; ++j) n += zd > (double)(2 * j - 17) * sd * 0.0625 ? 1u : 0u;
    return n;
}

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
                idx[j] = ste_index(zv[j], s, c8, s8, m17, fast);
                // the code value: exact in fp32 on the fast path; otherwise the double value
                // rounded once, as the definition reads
                qv[j] = fast ? s8 * (float)((int)idx[j] - 8)
                             : (float)((double)s * 0.125 * (double)((int)idx[j] - 8));
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

}  // namespace

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
