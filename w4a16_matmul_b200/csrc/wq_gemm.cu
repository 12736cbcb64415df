// wq_gemm.cu -- W4A16 GEMM for prefill on the 5th-generation tensor cores (tcgen05).
//
// y[m, n] = sum_k x[m, k] Wdeq[n, k], Wdeq the dyadic reconstruction of
// "MiniCPM5-1B 验证: 6× 压缩…" §2.2 (bf16(step*(idx-8)), one rounding), fused into the
// GEMM instead of materialised (the "materialized bf16 cache" of that article's §3.2 is
// the unfused alternative); the large-batch branch of "K-Means量化技术…" §4.1.
//
// One CTA computes a 128 (weight rows) x BN (activation rows) tile over a K range:
//   warp 0     TMA producer: per 64-column stage, the activation tile [BN x 64] bf16
//              (128-byte swizzle) and the packed weight tile [128 x 32 bytes];
//   warp 1     allocates tensor memory, and one lane issues tcgen05.mma (kind::f16,
//              bf16 x bf16 -> fp32 in TMEM, M=128, N=BN, K=16 x 4 per stage) and commits
//              each stage back to the producers;
//   warps 2-5  reconstruct the weight tile: thread i owns weight row i, turns its 64
//              codes into bf16 exactly as wq_dequant does, and writes them into the
//              K-major 128-byte-swizzled layout the MMA descriptor reads; afterwards they
//              drain the accumulator with tcgen05.ld and store bf16 (or fp32 partial sums
//              when K is split across CTAs, reduced by a second small kernel).
// Every wait on an mbarrier is bounded; a wait that expires records an error word on the
// device (see wq_device_error) and the CTA skips the rest of its work, still releasing its
// tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "wq_internal.cuh"

namespace wq {

__device__ int g_device_error;     // 0, or the code of the first expired device wait

namespace {

constexpr int BM = 128;            // weight rows per CTA (MMA M)
constexpr int BK = 64;             // columns per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 2000000000ull;   // a wait longer than 2 s is declared dead

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the completion of phase `parity`: gives up after about two seconds of
// wall time (checked every 64 polls) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
    const uint32_t a = smem_u32(b);
    uint64_t deadline = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
            : "=r"(done) : "r"(a), "r"(parity) : "memory");
        if (done) return true;
        if ((i & 63) == 0) {
            const uint64_t now = global_ns();
            if (deadline == 0) deadline = now + kWaitNs;
            else if (now > deadline) return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);   // start address
    d |= (uint64_t)1 << 16;                               // leading offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;                     // stride between 8-row atoms
    d |= (uint64_t)1 << 46;                               // descriptor version
    d |= (uint64_t)2 << 61;                               // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
          "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

// bf16 of the 8 codes of one packed word, in column order: (c0,c1), (c2,c3), (c4,c5),
// (c6,c7), each bf16(step * (idx - 8)) rounded once. A bf16 pattern below 0x0100 is worth
// exactly pattern * 2^-133 (subnormals and the first normal binade share that spacing), so
// masked nibble pairs need no shift; two FMAs then form scale * (idx - 8) / 8 exactly and
// round it once. cs / cn = (16 * scale, -scale) as bf16 pairs.
__device__ __forceinline__ uint4 dyadic_row8(uint32_t w, uint32_t cs, uint32_t cn) {
    const uint32_t kP126 = 0x7E807E80u, kP122 = 0x7C807C80u, kNegZero = 0x80008000u;
    const uint32_t t = w >> 8;
    const uint32_t p0 = bf16x2_fma(bf16x2_fma(w & 0x000F000Fu, kP126, kNegZero), cs, cn);   // (c0, c4)
    const uint32_t p1 = bf16x2_fma(bf16x2_fma(w & 0x00F000F0u, kP122, kNegZero), cs, cn);   // (c1, c5)
    const uint32_t p2 = bf16x2_fma(bf16x2_fma(t & 0x000F000Fu, kP126, kNegZero), cs, cn);   // (c2, c6)
    const uint32_t p3 = bf16x2_fma(bf16x2_fma(t & 0x00F000F0u, kP122, kNegZero), cs, cn);   // (c3, c7)
    return make_uint4(prmt(p0, p1, 0x5410u), prmt(p2, p3, 0x5410u), prmt(p0, p1, 0x7632u),
                      prmt(p2, p3, 0x7632u));
}
// The same in fp32, for scales of 2^124 and above (16 * scale would overflow bf16).
__device__ __forceinline__ uint4 dyadic_row8_f32(uint32_t w, float step) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = step * (float)((int)((w >> (4 * j)) & 15) - 8);
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
}

template <int BN>
struct Smem {
    static constexpr int A_BYTES = BM * BK * 2;          // 16 KB bf16 weight tile
    static constexpr int B_BYTES = BN * BK * 2;          // activation tile
    static constexpr int P_BYTES = BM * BK / 2;          // 4 KB packed weight tile
    static constexpr int STAGE = A_BYTES + B_BYTES + P_BYTES;
    static constexpr int BARS = 3 * STAGES + 1;
    static constexpr int TOTAL = STAGES * STAGE + BARS * 8 + 16 + 1024;   // + alignment slack
};

template <int BN, int G, bool PARTIAL>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
            const uint16_t* __restrict__ scale, void* __restrict__ out, int M, int N, int K,
            int kt_per_split) {
    using S = Smem<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full_tma = (uint64_t*)(smem + STAGES * S::STAGE);
    uint64_t* full_w = full_tma + STAGES;
    uint64_t* empty = full_w + STAGES;
    uint64_t* acc_full = empty + STAGES;
    uint32_t* s_tmem = (uint32_t*)(acc_full + 1);
    int* s_abort = (int*)(s_tmem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BM, m0 = blockIdx.y * BN;
    const int KT = K / BK;
    const int kt0 = blockIdx.z * kt_per_split;
    const int kt1 = min(KT, kt0 + kt_per_split);
    const int nk = kt1 - kt0;
    constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&full_w[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(s_tmem)), "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        asm volatile("tcgen05.fence::before_thread_sync;");
    }
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *s_tmem;

    auto stage_a = [&](int s) { return smem + s * S::STAGE; };
    auto stage_b = [&](int s) { return smem + s * S::STAGE + S::A_BYTES; };
    auto stage_p = [&](int s) { return smem + s * S::STAGE + S::A_BYTES + S::B_BYTES; };
    auto dead = [&](int code) {
        *(volatile int*)s_abort = 1;
        atomicCAS(&g_device_error, 0, code);
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (i / STAGES) & 1;
                if (*(volatile int*)s_abort) break;
                if (!mbar_wait(&empty[s], ph ^ 1)) { dead(1); break; }
                mbar_expect_tx(&full_tma[s], S::B_BYTES + S::P_BYTES);
                const int kt = kt0 + i;
                tma_load_2d(stage_b(s), &tmap_x, kt * BK, m0, &full_tma[s]);
                tma_load_2d(stage_p(s), &tmap_p, kt * (BK / 2), n0, &full_tma[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                       ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
            bool ok = true;
            for (int i = 0; i < nk; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (i / STAGES) & 1;
                if (*(volatile int*)s_abort) { ok = false; break; }
                if (!mbar_wait(&full_w[s], ph)) { dead(2); ok = false; break; }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint64_t da = sw128_desc(smem_u32(stage_a(s)));
                const uint64_t db = sw128_desc(smem_u32(stage_b(s)));
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)   // 32 bytes of K per MMA: +2 in descriptor units
                    umma_f16(tmem, da + 2 * k, db + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
                umma_commit(&empty[s]);
            }
            // commit (not a plain arrive) even after an abort: it fires only once every MMA
            // issued so far has finished, so tensor memory is never freed under a running MMA
            (void)ok;
            umma_commit(acc_full);
        }
    } else {
        // ---------------- reconstruction, then epilogue ----------------
        const int i = threadIdx.x - 64;                  // weight row within the tile
        const int n = n0 + i;
        const bool row_ok = n < N;
        const uint16_t* srow = scale + (size_t)(row_ok ? n : 0) * (K / G);
        // the per-group scales of this row, loaded kPre stages ahead (a ring of registers)
        constexpr int kPre = 4;
        uint32_t ring0[kPre], ring1[kPre];
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
            ring0[u] = ring1[u] = 0;
            if (row_ok && u < nk) {
                ring0[u] = ldg_u16(srow + (kt0 + u) * BK / G);
                ring1[u] = (G == 32) ? ldg_u16(srow + (kt0 + u) * BK / G + 1) : ring0[u];
            }
        }
        bool live = true;
        for (int base = 0; base < nk && live; base += kPre) {
#pragma unroll
            for (int u = 0; u < kPre; ++u) {
                const int it = base + u;
                if (it >= nk) break;
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                // every exit below is taken by the whole warp (it ends in __syncwarp)
                if (__any_sync(0xFFFFFFFFu, *(volatile int*)s_abort != 0)) { live = false; break; }
                const uint32_t sc0 = ring0[u], sc1 = ring1[u];
                if (row_ok && it + kPre < nk) {
                    ring0[u] = ldg_u16(srow + (kt0 + it + kPre) * BK / G);
                    ring1[u] = (G == 32) ? ldg_u16(srow + (kt0 + it + kPre) * BK / G + 1) : ring0[u];
                }
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full_tma[s], ph))) { dead(3); live = false; break; }
                const uint4* pk = (const uint4*)(stage_p(s) + i * 32);
                const uint4 q0 = pk[0], q1 = pk[1];
                const uint32_t wv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                uint8_t* arow = stage_a(s) + i * 128;
                const bool huge = ((sc0 & 0x7FFFu) >= 0x7D80u) || ((sc1 & 0x7FFFu) >= 0x7D80u);
                const uint32_t s20 = prmt(sc0, 0, 0x1010u), s21 = prmt(sc1, 0, 0x1010u);
                const uint32_t cs0 = bf16x2_fma(s20, 0x41804180u, 0x80008000u), cn0 = s20 ^ 0x80008000u;
                const uint32_t cs1 = bf16x2_fma(s21, 0x41804180u, 0x80008000u), cn1 = s21 ^ 0x80008000u;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const bool second = (G == 32) && c >= 4;
                    const uint4 v = huge ? dyadic_row8_f32(wv[c], bf16_bits_to_float(second ? sc1 : sc0) * 0.125f)
                                         : dyadic_row8(wv[c], second ? cs1 : cs0, second ? cn1 : cn0);
                    *(uint4*)(arow + ((c ^ (i & 7)) << 4)) = v;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_w[s]);
            }
        }
        // ---- epilogue: TMEM lanes 32*(warp%4).. hold weight rows, columns = activation rows
        // tcgen05.ld is warp-collective: the decision to drain is taken per warp
        const bool drain = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0)) &&
                           !__any_sync(0xFFFFFFFFu, *(volatile int*)s_abort != 0);
        if (drain) {
            asm volatile("tcgen05.fence::after_thread_sync;");
            const int q = warp & 3;
            const int nrow = n0 + 32 * q + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (nrow < N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < M) {
                            if (PARTIAL)
                                ((float*)out)[((size_t)blockIdx.z * M + m) * N + nrow] = __uint_as_float(v[j]);
                            else
                                ((uint16_t*)out)[(size_t)m * N + nrow] =
                                    (uint16_t)float_to_bf16_bits(__uint_as_float(v[j]));
                        }
                    }
                }
            }
        } else {
            dead(4);
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// y[m, n] = bf16(sum over splits of the fp32 partial sums)
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float* __restrict__ part, int splits, int64_t mn, uint16_t* __restrict__ y) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < mn; i += (int64_t)gridDim.x * blockDim.x) {
        float v = 0.f;
        for (int s = 0; s < splits; ++s) v += part[s * mn + i];
        y[i] = (uint16_t)float_to_bf16_bits(v);
    }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
        else
            cudaGetLastError();
    }
    return fn;
}

struct Plan {
    int bn, splits, kt_per_split, grid_n, grid_m;
};

Plan plan_for(int64_t M, int64_t N, int64_t K) {
    Plan p;
    p.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= 128 ? 128 : 256;
    p.grid_n = (int)((N + BM - 1) / BM);
    p.grid_m = (int)((M + p.bn - 1) / p.bn);
    const int KT = (int)(K / BK);
    const int64_t tiles = (int64_t)p.grid_n * p.grid_m;
    const int sms = sm_count();
    int splits = 1;
    // split K while the grid is below one wave and every split keeps >= 16 stages
    while (tiles * splits * 2 <= sms && KT / (splits * 2) >= 16) splits *= 2;
    p.kt_per_split = (KT + splits - 1) / splits;
    p.splits = (KT + p.kt_per_split - 1) / p.kt_per_split;
    return p;
}

template <int BN, int G>
wq_status launch_bn(const Plan& p, const CUtensorMap& tx, const CUtensorMap& tp, const uint16_t* scale,
                    void* out, int M, int N, int K, cudaStream_t s) {
    const int smem = Smem<BN>::TOTAL;
    const dim3 grid(p.grid_n, p.grid_m, p.splits);
    if (p.splits > 1) {
        auto k = gemm_kernel<BN, G, true>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        k<<<grid, kThreads, smem, s>>>(tx, tp, scale, out, M, N, K, p.kt_per_split);
    } else {
        auto k = gemm_kernel<BN, G, false>;
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        k<<<grid, kThreads, smem, s>>>(tx, tp, scale, out, M, N, K, p.kt_per_split);
    }
    return check_launch("gemm");
}

}  // namespace

size_t gemm_workspace_bytes(const wq_weight& w, int64_t m) {
    const Plan p = plan_for(m, w.n, w.k);
    return p.splits > 1 ? (size_t)p.splits * (size_t)m * (size_t)w.n * sizeof(float) : 0;
}

wq_status launch_gemm(const wq_weight& w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
    const int M = (int)m, N = (int)w.n, K = (int)w.k;
    const Plan p = plan_for(M, N, K);
    auto enc = encode_fn();
    if (!enc) return fail(WQ_ECUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    CUtensorMap tx, tp;
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)p.bn};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void*)x, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for x failed (%d)", (int)r);
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K / 2};
        cuuint32_t box[2] = {(cuuint32_t)(BK / 2), (cuuint32_t)BM};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)w.packed, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for packed weights failed (%d)", (int)r);
    }
    void* out = p.splits > 1 ? ws : (void*)y;
    if (p.splits > 1 && (ws == nullptr || ws_bytes < gemm_workspace_bytes(w, m)))
        return fail(WQ_EINVAL, "workspace too small");
    const uint16_t* sc = (const uint16_t*)w.aux;
    wq_status st;
#define WQ_BN(BNV)                                                                                  \
    st = (w.group == 64) ? launch_bn<BNV, 64>(p, tx, tp, sc, out, M, N, K, s)                     \
                         : launch_bn<BNV, 32>(p, tx, tp, sc, out, M, N, K, s)
    switch (p.bn) {
        case 16: WQ_BN(16); break;
        case 32: WQ_BN(32); break;
        case 64: WQ_BN(64); break;
        case 128: WQ_BN(128); break;
        default: WQ_BN(256); break;
    }
#undef WQ_BN
    if (st != WQ_OK || p.splits == 1) return st;
    const int64_t mn = (int64_t)M * N;
    int grid = (int)((mn + 255) / 256);
    if (grid > sm_count() * 8) grid = sm_count() * 8;
    splitk_reduce_kernel<<<grid, 256, 0, s>>>((const float*)ws, p.splits, mn, y);
    return check_launch("gemm split-k reduce");
}

wq_status read_device_error(int32_t* code) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    if (e != cudaSuccess) return fail(WQ_ECUDA, "reading the device error word: %s", cudaGetErrorString(e));
    if (v != 0) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    }
    *code = v;
    return WQ_OK;
}

}  // namespace wq
