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
//              bf16 x bf16 -> fp32 in TMEM, M=128, N=BN, K=16 x 4 per stage) with the
//              weight operand A read from tensor memory and the activations B from shared
//              memory, and commits each stage back to the producer;
//   warps 2-5  reconstruct the weight tile: the thread of tensor-memory lane i owns weight
//              row i, turns its 64 codes into bf16 exactly as wq_dequant does and stores
//              them into that lane's 32-column slot of the stage (tcgen05.st); afterwards
//              they drain the accumulator with tcgen05.ld and store bf16 (or fp32 partial
//              sums when K is split across CTAs, reduced by a second small kernel).
// Keeping the reconstructed operand in tensor memory leaves shared memory to the TMA tiles
// alone: no bf16 tile is written to and read back from shared memory, whose bandwidth the
// MMA's activation reads and the TMA writes already share, and the freed space holds six
// pipeline stages.
// The LLOYD8S and LUT16 formats run in the same pipeline: their per-group tables (8 fp32
// levels per 32 columns, 16 fp16 centroids per 64) arrive by TMA with each stage and the
// reconstruction warps look the codes up in them. LUT16 runs an fp16 MMA, so that its
// centroids enter the product unrounded: its activations are converted to fp16 once, into
// the workspace, by a small kernel ahead of the GEMM.
// Every wait on an mbarrier is bounded; a wait that expires records an error word on the
// device (see wq_device_error) and the CTA skips the rest of its work, still releasing its
// tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "wq_internal.cuh"

namespace wq {

WQ_DEBUG_WORD(gemm)

__device__ int g_device_error;     // 0, or the code of the first expired device wait

namespace {

constexpr int BM = 128;            // weight rows per CTA (MMA M)
// Columns per stage, KB: 64 (one 128-byte swizzle row of bf16) or 128 (two such tiles, used
// when K % 128 == 0: twice the reconstruction work per stage for the same bookkeeping).

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

// Pipeline depths per activation-tile width. Shared-memory stages (the [BN x 64] bf16
// activation tile and the [128 x 32 B] packed tile each) hold the bytes in flight: as many
// as 216 KB hold, up to 16. Tensor-memory slots (32 columns each, the reconstructed
// weights of one stage) only need to cover reconstruction-to-MMA latency; for BN <= 64 the
// allocation stays at 256 columns so that two CTAs can share an SM.
// Weight formats of the kernel (template parameter F): the dyadic step, the LLOYD8S levels
// or the LUT16 table.
constexpr int kFDy = 0, kFLl = 1, kFLu = 2;

template <int BN, int F = kFDy, int KB = 64>
struct Smem {
    static constexpr int B_BYTES = BN * KB * 2;          // KB/64 activation tiles (128-byte swizzle)
    static constexpr int P_BYTES = BM * KB / 2;          // packed weight tile
    // the stage's per-group tables: LLOYD8S 8 fp32 levels per 32 columns, LUT16 16 fp16
    // centroids per 64 columns
    static constexpr int L_BYTES = F == kFLl ? BM * KB : F == kFLu ? BM * KB / 2 : 0;
    static constexpr int STAGE = B_BYTES + P_BYTES + L_BYTES;   // a multiple of 1024
    static constexpr int STAGES = (216 * 1024 / STAGE) < 16 ? (216 * 1024 / STAGE) : 16;
    static constexpr int BARS = 2 * STAGES + 2 * 8 + 1;
    static constexpr int TOTAL = STAGES * STAGE + BARS * 8 + 16 + 1024;   // + alignment slack
    // tensor memory: the fp32 accumulator [128 lanes x BN columns], then SLOTS 32-column
    // slots for reconstructed bf16 weight tiles (64 values of a row per lane, two per 32-bit
    // column, lower k in the low half)
    static constexpr uint32_t ACC_COLS = BN < 32 ? 32 : BN;
    static constexpr int SLOT_COLS = KB / 2;              // bf16 pairs of one stage's row
    // BN >= 128: one slot per stage where tensor memory holds them (the rings coincide, and
    // the producer's wait for a free stage already orders slot reuse); BN <= 64: up to six
    // slots under a deep ring, within 256 columns
    static constexpr int NARROW_SLOTS = (int)((256 - ACC_COLS) / SLOT_COLS) < 6 ? (int)((256 - ACC_COLS) / SLOT_COLS) : 6;
    static constexpr int WIDE_FIT = (int)((512 - ACC_COLS) / SLOT_COLS) < 8 ? (int)((512 - ACC_COLS) / SLOT_COLS) : 8;
    static constexpr int SLOTS = BN <= 64 ? NARROW_SLOTS : (STAGES < WIDE_FIT ? STAGES : WIDE_FIT);
    static constexpr bool COUPLED = SLOTS == STAGES;
    static constexpr uint32_t USED_COLS = ACC_COLS + SLOT_COLS * SLOTS;
    static constexpr uint32_t TMEM_COLS = USED_COLS <= 64 ? 64 : USED_COLS <= 128 ? 128
                                        : USED_COLS <= 256 ? 256 : 512;
};

__device__ __forceinline__ void umma_f16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }"
        ::"r"(tmem_d), "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate));
}

// Stores 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
          "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
          "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
          "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
          "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

#ifndef WQ_GEMM_RW
#define WQ_GEMM_RW 4
#endif
#ifndef WQ_GEMM_RW_NARROW
#define WQ_GEMM_RW_NARROW 2
#endif
// Reconstruction warps per tensor-memory lane group: RW warps share each 32-lane group, each
// filling 1 / RW of the row's packed words per stage (more warps hide more latency; fewer
// repeat less per-stage bookkeeping).
constexpr int rw_for(int bn) { return bn >= 128 ? WQ_GEMM_RW : WQ_GEMM_RW_NARROW; }
constexpr int threads_for(int bn) { return 64 + 128 * rw_for(bn); }

// Stores NC (8, 16 or 32) consecutive 32-bit columns of this thread's tensor-memory lane.
template <int NC>
__device__ __forceinline__ void tmem_st_part(uint32_t taddr, const uint32_t* v) {
    static_assert(NC == 8 || NC == 16 || NC == 32, "8, 16 or 32 columns");
    if constexpr (NC == 32) {
        tmem_st32(taddr, *reinterpret_cast<const uint32_t(*)[32]>(v));
    } else if constexpr (NC == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
            "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
            ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
              "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
              "r"(v[15])
            : "memory");
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
            ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
              "r"(v[7])
            : "memory");
    }
}

// F == kFLl: LLOYD8S weights (groups of 32, 8 fp32 levels each, loaded per stage by TMA
// through tmap_l; `scale` unused). F == kFLu: LUT16 weights (groups of 64, 16 fp16 centroids
// each, loaded the same way), with fp16 activations and an fp16 MMA. Otherwise DYADIC4 with
// group G.
template <int BN, int G, bool PARTIAL, int F, int KB>
__global__ void __launch_bounds__(threads_for(BN), 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_p,
            const __grid_constant__ CUtensorMap tmap_l, const uint16_t* __restrict__ scale,
            void* __restrict__ out, int M, int N, int K, int kt_per_split, int grid_n, int tile0) {
    using S = Smem<BN, F, KB>;
    constexpr bool LL = F == kFLl, LU = F == kFLu;
    constexpr int XBOXES = BN > 256 ? 2 : 1;        // TMA boxes span at most 256 rows
    constexpr int STAGES = S::STAGES;
    constexpr int RW = rw_for(BN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int SLOTS = S::SLOTS;
    uint64_t* full_tma = (uint64_t*)(smem + STAGES * S::STAGE);   // stage landed (TMA bytes)
    uint64_t* empty = full_tma + STAGES;                            // stage consumed (MMA done)
    uint64_t* full_w = empty + STAGES;                              // slot reconstructed
    uint64_t* slot_free = full_w + 8;                               // slot read by its MMAs
    uint64_t* acc_full = slot_free + 8;
    uint32_t* s_tmem = (uint32_t*)(acc_full + 1);
    int* s_abort = (int*)(s_tmem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tile (weight-row tile fastest, the launch order the grid had as a 2D grid); a launch
    // may cover a contiguous range of tiles starting at tile0
    const int lin = tile0 + (int)blockIdx.x;
    const int n0 = (lin % grid_n) * BM, m0 = (lin / grid_n) * BN;
    const int KT = K / KB;
    const int kt0 = blockIdx.y * kt_per_split;
    const int kt1 = min(KT, kt0 + kt_per_split);
    const int nk = kt1 - kt0;
    WQ_DCHECK(n0 < N && m0 < M && kt0 < KT && kt1 <= KT, kDbgIndex + 20);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < SLOTS; ++a) {
            mbar_init(&full_w[a], 4 * RW);
            mbar_init(&slot_free[a], 1);
        }
        mbar_init(acc_full, 1);
        *s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(s_tmem)), "r"(S::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        asm volatile("tcgen05.fence::before_thread_sync;");
    }
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;");
    const uint32_t tmem = *s_tmem;

    auto stage_b = [&](int s) { return smem + s * S::STAGE; };
    auto stage_p = [&](int s) { return smem + s * S::STAGE + S::B_BYTES; };
    auto stage_l = [&](int s) { return smem + s * S::STAGE + S::B_BYTES + S::P_BYTES; };
    auto dead = [&](int code) {
        *(volatile int*)s_abort = 1;
        atomicCAS(&g_device_error, 0, code);
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nk; ++i, s = (s + 1 == STAGES) ? 0 : s + 1, ph ^= (s == 0)) {
                if (!mbar_wait(&empty[s], ph ^ 1, s_abort)) { dead(1); break; }
                mbar_expect_tx(&full_tma[s], S::B_BYTES + S::P_BYTES + S::L_BYTES);
                const int kt = kt0 + i;
#pragma unroll
                for (int j = 0; j < KB / 64; ++j)
#pragma unroll
                    for (int h = 0; h < XBOXES; ++h)   // activation boxes of BN / XBOXES rows
                        tma_load_2d(stage_b(s) + j * BN * 128 + h * (BN / XBOXES) * 128, &tmap_x,
                                    kt * KB + 64 * j, m0 + h * (BN / XBOXES), &full_tma[s]);
                tma_load_2d(stage_p(s), &tmap_p, kt * (KB / 2), n0, &full_tma[s]);
                // both tables hold KB / 4 elements of a row per stage
                if (F != kFDy) tma_load_2d(stage_l(s), &tmap_l, kt * (KB / 4), n0, &full_tma[s]);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: A (weights) from tensor memory, B from shared ------
        if (lane == 0) {
            // fp32 accumulator; A and B both bf16 (format 1), or both fp16 (format 0) for LUT16
            constexpr uint32_t ab = LU ? 0u : (1u << 7) | (1u << 10);
            // BN = 384: two MMAs of N = 192 per K step read the same weight slot, into the two
            // halves of the accumulator, from the two halves of the activation tile
            constexpr int NH = BN > 256 ? 2 : 1, NM = BN / NH;
            constexpr uint32_t idesc = (1u << 4) | ab | ((uint32_t)(NM >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
            int s = 0, a = 0;
            uint32_t aph = 0;
            for (int i = 0; i < nk; ++i) {
                // the slot is reconstructed, which also means the stage's tiles have landed
                if (!mbar_wait(&full_w[a], aph, s_abort)) { dead(2); break; }
                asm volatile("tcgen05.fence::after_thread_sync;");
                const uint32_t ta = tmem + S::ACC_COLS + (uint32_t)(S::SLOT_COLS * a);
#pragma unroll
                for (int k = 0; k < KB / 16; ++k) {  // 16 values of K: 8 A columns, +2 in B descriptor units
                    const uint64_t db = sw128_desc(smem_u32(stage_b(s) + (k / 4) * BN * 128));
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        // descriptor address units are 16 bytes: + NM rows of 128 bytes
                        const uint64_t dbh = db + (uint64_t)(h * NM * 128 / 16);
                        umma_f16_ts(tmem + (uint32_t)(h * NM), ta + 8u * (uint32_t)k, dbh + 2 * (k % 4), idesc,
                                    (i > 0 || k > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&empty[s]);           // fire once these MMAs have read the stage ...
                if constexpr (!S::COUPLED) umma_commit(&slot_free[a]);   // ... and the slot
                if (++s == STAGES) s = 0;
                if (++a == SLOTS) { a = 0; aph ^= 1; }
            }
            // commit (not a plain arrive) even after an abort: it fires only once every MMA
            // issued so far has finished, so tensor memory is never freed under a running MMA
            umma_commit(acc_full);
        }
    } else {
        // ---------------- reconstruction into tensor memory, then epilogue ----------------
        // a warp may touch only the tensor-memory lanes 32 * (warp % 4) .. + 31: thread
        // (warp, lane) owns weight row 32 * (warp % 4) + lane of the tile, and of that row's
        // KB / 8 packed words per stage the words [part * WPT, part * WPT + WPT), columns
        // colbase .. colbase + 8 WPT - 1 of the stage
        constexpr int WPT = (KB / 8) / RW;
        // a thread's columns span one group, or two g32 groups (then aligned to them)
        constexpr bool SPAN2 = F == kFDy && WPT * 8 > G;
        static_assert(WPT * 8 <= 2 * G || F != kFDy, "at most two scale groups per thread and stage");
        static_assert(!LU || WPT * 8 <= 64, "a thread's LUT16 columns lie in one group of 64");
        const int q = warp & 3, part = (warp - 2) >> 2;
        const int colbase = part * WPT * 8;
        const int i = 32 * q + lane;
        const int n = n0 + i;
        const bool row_ok = n < N;
        const uint16_t* srow = scale + (size_t)(row_ok ? n : 0) * (K / G) + colbase / G;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        // the scales of this thread's group(s), loaded kPre stages ahead (a ring of registers)
        constexpr int kPre = 4;
        uint32_t ring0[kPre], ring1[kPre];
#pragma unroll
        for (int u = 0; u < kPre; ++u) {
            ring0[u] = ring1[u] = 0;
            if (F == kFDy && row_ok && u < nk) {
                ring0[u] = ldg_u16(srow + (kt0 + u) * (KB / G));
                ring1[u] = SPAN2 ? ldg_u16(srow + (kt0 + u) * (KB / G) + 1) : ring0[u];
            }
        }
        bool live = true;
        int s = 0, a = 0;                                  // stage and slot of iteration it
        uint32_t ph = 0, aph = 0;                          // their phase parities
        for (int base = 0; base < nk && live; base += kPre) {
#pragma unroll
            for (int u = 0; u < kPre; ++u) {
                const int it = base + u;
                if (it >= nk) break;
                const uint32_t sc0 = ring0[u], sc1 = ring1[u];
                if (F == kFDy && row_ok && it + kPre < nk) {
                    ring0[u] = ldg_u16(srow + (kt0 + it + kPre) * (KB / G));
                    ring1[u] = SPAN2 ? ldg_u16(srow + (kt0 + it + kPre) * (KB / G) + 1) : ring0[u];
                }
                // the packed tile has landed, and the MMAs that last read this tensor-memory
                // slot (iteration it - SLOTS) have completed (with coupled rings the first
                // implies the second: the TMA for this iteration was issued only after the
                // stage's previous MMAs completed). Every exit is taken by the whole warp.
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full_tma[s], ph, s_abort) &&
                                             (S::COUPLED || it < SLOTS ||
                                              mbar_wait(&slot_free[a], aph ^ 1, s_abort)))) {
                    dead(3); live = false; break;
                }
                uint32_t wv[WPT];
                {
                    const uint32_t* pk = (const uint32_t*)(stage_p(s) + i * (KB / 2) + colbase / 2);
                    if constexpr (WPT >= 4) {
#pragma unroll
                        for (int c = 0; c < WPT; c += 4) {
                            const uint4 t4 = *(const uint4*)(pk + c);
                            wv[c] = t4.x; wv[c + 1] = t4.y; wv[c + 2] = t4.z; wv[c + 3] = t4.w;
                        }
                    } else {
                        const uint2 t2 = *(const uint2*)pk;
                        wv[0] = t2.x; wv[1] = t2.y;
                    }
                }
                uint32_t v[4 * WPT];
                if constexpr (LL) {
                    // bf16(level) byte planes of the group(s) this thread's words lie in (4
                    // words per group of 32), then one permute per plane and a sign flip per
                    // code, as the GEMV's register codebook does
                    constexpr int NG = (WPT + 3) / 4;
                    uint32_t plo[NG][2], phi[NG][2];
#pragma unroll
                    for (int gi = 0; gi < NG; ++gi) {
                        const int grp = colbase / 32 + gi;
                        const float4* lv = (const float4*)(stage_l(s) + i * KB + grp * 32);
                        const float4 l0 = lv[0], l1 = lv[1];
                        const uint32_t b01 = pack_bf16x2(l0.x, l0.y), b23 = pack_bf16x2(l0.z, l0.w);
                        const uint32_t b45 = pack_bf16x2(l1.x, l1.y), b67 = pack_bf16x2(l1.z, l1.w);
                        plo[gi][0] = prmt(b01, b23, 0x6420u); plo[gi][1] = prmt(b45, b67, 0x6420u);
                        phi[gi][0] = prmt(b01, b23, 0x7531u); phi[gi][1] = prmt(b45, b67, 0x7531u);
                    }
#pragma unroll
                    for (int c = 0; c < WPT; ++c) {
                        const int gi = c >> 2;
                        lloyd8_lookup4(wv[c], plo[gi], phi[gi], v[4 * c], v[4 * c + 1]);
                        lloyd8_lookup4(wv[c] >> 16, plo[gi], phi[gi], v[4 * c + 2], v[4 * c + 3]);
                    }
                } else if constexpr (LU) {
                    // the 16 fp16 centroids of the group this thread's words lie in, as byte
                    // planes (lo / hi[q]: low / high bytes of entries 4q .. 4q + 3), then the
                    // same lookup as the GEMV's: the centroids enter the product unrounded
                    const uint4* tv = (const uint4*)(stage_l(s) + i * (KB / 2) + (colbase / 64) * 32);
                    const uint4 t0 = tv[0], t1 = tv[1];
                    const uint32_t lo[4] = {prmt(t0.x, t0.y, 0x6420u), prmt(t0.z, t0.w, 0x6420u),
                                            prmt(t1.x, t1.y, 0x6420u), prmt(t1.z, t1.w, 0x6420u)};
                    const uint32_t hi[4] = {prmt(t0.x, t0.y, 0x7531u), prmt(t0.z, t0.w, 0x7531u),
                                            prmt(t1.x, t1.y, 0x7531u), prmt(t1.z, t1.w, 0x7531u)};
#pragma unroll
                    for (int c = 0; c < WPT; ++c) {
                        lut16_lookup4(wv[c], lo, hi, v[4 * c], v[4 * c + 1]);
                        lut16_lookup4(wv[c] >> 16, lo, hi, v[4 * c + 2], v[4 * c + 3]);
                    }
                } else {
                    const bool huge = ((sc0 & 0x7FFFu) >= 0x7D80u) || ((sc1 & 0x7FFFu) >= 0x7D80u);
                    const uint32_t s20 = prmt(sc0, 0, 0x1010u), s21 = prmt(sc1, 0, 0x1010u);
                    const uint32_t cs0 = bf16x2_fma(s20, 0x41804180u, 0x80008000u), cn0 = s20 ^ 0x80008000u;
                    const uint32_t cs1 = bf16x2_fma(s21, 0x41804180u, 0x80008000u), cn1 = s21 ^ 0x80008000u;
#pragma unroll
                    for (int c = 0; c < WPT; ++c) {
                        const bool second = SPAN2 && 8 * c >= G;
                        const uint4 r = huge ? dyadic_row8_f32(wv[c], bf16_bits_to_float(second ? sc1 : sc0) * 0.125f)
                                             : dyadic_row8(wv[c], second ? cs1 : cs0, second ? cn1 : cn0);
                        v[4 * c] = r.x; v[4 * c + 1] = r.y; v[4 * c + 2] = r.z; v[4 * c + 3] = r.w;
                    }
                }
                // the previous iteration's store has had this iteration's loads and arithmetic
                // to complete: wait for it now and release that slot to the MMA, then issue
                // this one (one tensor-memory store in flight per warp)
                if (it > 0) {
                    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full_w[a == 0 ? SLOTS - 1 : a - 1]);
                }
                tmem_st_part<4 * WPT>(lane_base + S::ACC_COLS + (uint32_t)(S::SLOT_COLS * a + 4 * WPT * part), v);
                if (++s == STAGES) { s = 0; ph ^= 1; }
                if (++a == SLOTS) { a = 0; aph ^= 1; }
            }
        }
        // release the last slot written (also after an abort: the MMA thread has stopped
        // waiting by then, and an extra arrival on a slot barrier is harmless)
        if (nk > 0) {
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (live && lane == 0) mbar_arrive(&full_w[a == 0 ? SLOTS - 1 : a - 1]);
        }
        // ---- epilogue: TMEM lane 32q + lane holds weight row n, columns = activation rows
        // tcgen05.ld is warp-collective: the decision to drain is taken per warp
        const bool drain = __all_sync(0xFFFFFFFFu, mbar_wait(acc_full, 0)) &&
                           !__any_sync(0xFFFFFFFFu, *(volatile int*)s_abort != 0);
        if (drain) {
            asm volatile("tcgen05.fence::after_thread_sync;");
            // the RW warps of a lane group split the accumulator's columns
            constexpr int CPP = (BN / RW) < 16 ? 16 : BN / RW;
            const int cbeg = part * CPP, cend = min(BN, cbeg + CPP);
#pragma unroll 1
            for (int c0 = cbeg; c0 < cend; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(lane_base + (uint32_t)c0, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m0 + c0 + j;
                        if (m < M) {
                            // LUT16: the activation row was scaled by 2^e; undo it (exact)
                            const float val = LU ? __uint_as_float(v[j]) * reinterpret_cast<const float*>(scale)[m]
                                                 : __uint_as_float(v[j]);
                            if (PARTIAL)                 // [split][tile of the launch][BN][BM]
                                ((float*)out)[(((size_t)blockIdx.y * gridDim.x + blockIdx.x) * BN + c0 + j) * BM +
                                              (n - n0)] = val;
                            else
                                ((uint16_t*)out)[(size_t)m * N + n] = (uint16_t)float_to_bf16_bits(val);
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
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(S::TMEM_COLS));
    }
}

// y[m, n] = bf16(sum over splits of the fp32 partial sums) for the ntl tiles of a partial
// launch starting at tile0; partial sums are laid out [split][tile][bn][BM]. One CTA per
// (tile, activation row): its 128 threads are the tile's 128 weight rows, so every load and
// store of a warp covers 32 consecutive rows, and the split loads are independent.
__global__ void __launch_bounds__(BM)
splitk_reduce_kernel(const float* __restrict__ part, int splits, int ntl, int tile0, int grid_n, int bn,
                     int M, int N, uint16_t* __restrict__ y) {
    const int64_t plane = (int64_t)ntl * bn * BM;
    const int lt = blockIdx.x, c = blockIdx.y, r = threadIdx.x;
    const int lin = tile0 + lt;
    const int n = (lin % grid_n) * BM + r, m = (lin / grid_n) * bn + c;
    if (n >= N || m >= M) return;
    const float* src = part + ((int64_t)lt * bn + c) * BM + r;
    float v = 0.f;
#pragma unroll 4
    for (int sp = 0; sp < splits; ++sp) v += __ldg(src + sp * plane);
    y[(size_t)m * N + n] = (uint16_t)float_to_bf16_bits(v);
}

// Activations for the LUT16 product, one CTA per activation row: the row's largest
// magnitude picks the power of two 2^e that brings it into [2^15, 2^16) (lut_x_exponent),
// the row is written as fp16(x * 2^e), and inv[row] = 2^-e for the epilogue. The row is
// read twice (the second pass mostly from L1/L2). K % 8 == 0.
__global__ void __launch_bounds__(256)
x_to_f16_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ xh, float* __restrict__ inv, int K) {
    __shared__ uint32_t red[8];
    const int64_t row = blockIdx.x;
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * K);
    uint4* hr = reinterpret_cast<uint4*>(xh + row * K);
    const int n8 = K / 8;
    uint32_t mx = 0;
    for (int i = threadIdx.x; i < n8; i += 256) {
        const uint4 v = ldg_v4(xr + i);
        WQ_DCHECK(bf16x8_finite(v), kDbgNonFiniteActivation + 2);
        mx = max(mx, bf16x8_max_mag(v));
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) mx = max(mx, red[w]);
    const int e = lut_x_exponent(mx);
    if (threadIdx.x == 0) inv[row] = pow2_f32(-e);
    const float s1 = pow2_f32(e >> 1), s2 = pow2_f32(e - (e >> 1));
    for (int i = threadIdx.x; i < n8; i += 256) {
        const uint4 v = ldg_v4(xr + i);
        hr[i] = make_uint4(bf16x2_to_f16x2_scaled(v.x, s1, s2), bf16x2_to_f16x2_scaled(v.y, s1, s2),
                           bf16x2_to_f16x2_scaled(v.z, s1, s2), bf16x2_to_f16x2_scaled(v.w, s1, s2));
    }
}

#if WQ_DEBUG
// Debug build only: the finite-activation check for the formats whose activations reach the
// MMA by TMA without passing through a kernel of this library first.
__global__ void __launch_bounds__(256) debug_scan_x_kernel(const uint4* __restrict__ x, int64_t n8) {
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (int64_t)gridDim.x * 256)
        WQ_DCHECK(bf16x8_finite(ldg_v4(x + i)), kDbgNonFiniteActivation + 3);
}
#endif

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
    int bn, kb, splits, kt_per_split, grid_n, grid_m;
    // last-wave split: the first `full` tiles (whole waves) run unsplit; the remaining
    // tiles run as a second launch with K split tail_splits ways (1: no second launch)
    int full, tail_splits, tail_kt_per_split;
};

#ifndef WQ_GEMM_TAIL_WAVES
#define WQ_GEMM_TAIL_WAVES 3           // the last-wave split runs after at most this many whole waves
#endif

#ifndef WQ_GEMM_BN128_MAX
#define WQ_GEMM_BN128_MAX 128
#endif
#ifndef WQ_GEMM_KB128
#define WQ_GEMM_KB128 1
#endif
#ifndef WQ_GEMM_BN384
#define WQ_GEMM_BN384 1
#endif

Plan plan_for(int64_t M, int64_t N, int64_t K, int fmt, size_t tail_cap) {
    Plan p;
    const int sms = sm_count();
    p.kb = 64;
    p.grid_n = (int)((N + BM - 1) / BM);
    // The widest activation tile the MMA takes once m allows it: every activation-row tile
    // reconstructs the same weights again, and reconstruction (not the tensor pipe) is what
    // narrower tiles run out of (measured: BN 128 / 192 at 0.5-0.9x of BN 256 throughput even
    // where they leave fewer SMs idle in the last wave).
    p.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M <= WQ_GEMM_BN128_MAX ? 128 : 256;
    // 384-row activation tiles (two N = 192 MMAs from each reconstructed weight slot) where
    // they need at most 0.7 times the waves of 256-row ones. Each weight is rebuilt once per
    // tile either way, but a 384-row tile takes about 1.35 times as long (4 pipeline stages
    // instead of 6, and shared memory near its bandwidth: the TMA writes plus the MMA's reads
    // of the activation tile), so fewer waves pay only where they are much fewer. Measured:
    // 11008 x 4096 at m = 4096 (7 waves instead of 10) 353 -> 337 us; 4096 x 11008 at
    // m = 4096 (3 instead of 4) 339 -> 344 us and 11008 x 4096 at m = 2048 (4 instead of 5)
    // 179 -> 194 us, which keep 256 rows.
    if (WQ_GEMM_BN384 && p.bn == 256) {
        const int64_t gn = (N + BM - 1) / BM;
        const int64_t w256 = (gn * ((M + 255) / 256) + sms - 1) / sms;
        const int64_t w384 = (gn * ((M + 383) / 384) + sms - 1) / sms;
        if (gn * ((M + 383) / 384) >= sms && 10 * w384 <= 7 * w256) p.bn = 384;
    }
    // 128-column stages for 128-wide activation tiles where K allows: there they halve the
    // per-stage bookkeeping of the reconstruction, which this m is bound by (measured 1.4x at
    // m = 128); the 256-wide tiles keep 64-column stages, whose finer ring overlaps better
    // (measured 1.1x), and LLOYD8S keeps 64 (its level tiles would double too)
    if (WQ_GEMM_KB128 && p.bn == 128 && K % 128 == 0 && fmt != WQ_FMT_LLOYD8S) p.kb = 128;
    p.grid_m = (int)((M + p.bn - 1) / p.bn);
    const int KT = (int)(K / p.kb);
    const int64_t tiles = (int64_t)p.grid_n * p.grid_m;
    const int min_wide = 1024 / p.kb, min_narrow = 512 / p.kb;   // stages per split, at least
    int splits = 1;
    if (p.bn >= 128) {
        // wide tiles (one CTA per SM): split in powers of two while the grid stays within
        // one round and every split keeps >= 1024 columns
        while (tiles * splits * 2 <= sms && KT / (splits * 2) >= min_wide) splits *= 2;
    } else {
        // narrow tiles (256 tensor-memory columns, at most ~100 KB of shared memory) fit two
        // CTAs per SM. A grid of equal CTAs takes ceil(CTAs / slots) rounds of (stages per
        // CTA + a prologue and epilogue of about 256 columns' worth); take the split count
        // with the fewest, keeping >= 512 columns per split
        const int64_t slots = 2 * (int64_t)sms;
        const int64_t fixed = 256 / p.kb;
        int64_t best = -1;
        for (int sp = 1; sp <= 32 && (sp == 1 || KT / sp >= min_narrow); ++sp) {
            const int64_t per = (KT + sp - 1) / sp;
            const int64_t used = (KT + per - 1) / per;           // splits that get work
            const int64_t cost = ((tiles * used + slots - 1) / slots) * (per + fixed);
            if (best < 0 || cost < best) { best = cost; splits = (int)used; }
        }
    }
    p.kt_per_split = (KT + splits - 1) / splits;
    p.splits = (KT + p.kt_per_split - 1) / p.kt_per_split;
    // One to three whole waves of wide tiles plus a tail of at most half a wave: a single pass
    // spends a full wave's time on the tail. Run the whole waves as they are, then the tail
    // tiles with K split s ways (s tail CTAs per tile fit one wave: the tail then takes about
    // 1/s of a wave), each split keeping >= 512 columns, the partial sums within tail_cap.
    // (Measured on 11008 x 4096: m = 512, 1 wave + 24 tiles, 1.25x; with 9 waves + 44 tiles
    // at m = 4096 the second launch and its reduction cost what the tail saves, hence the
    // limit on whole waves.)
    p.full = (int)tiles;
    p.tail_splits = 1;
    p.tail_kt_per_split = KT;
    if (p.bn >= 128 && p.splits == 1) {
        const int64_t full = tiles / sms * sms, tail = tiles - full;
        if (full > 0 && full <= WQ_GEMM_TAIL_WAVES * sms && tail > 0 && 2 * tail <= sms) {
            int64_t sp = sms / tail;
            while (sp > 1 && KT / sp < min_narrow) --sp;
            while (sp > 1 && (size_t)sp * tail * BM * p.bn * sizeof(float) > tail_cap) --sp;
            if (sp > 1) {
                p.tail_kt_per_split = (KT + (int)sp - 1) / (int)sp;
                p.tail_splits = (KT + p.tail_kt_per_split - 1) / p.tail_kt_per_split;
                p.full = (int)full;
            }
        }
    }
    return p;
}

// One launch over tiles [tile0, tile0 + ntl) with K split `splits` ways (partial sums to
// `out` in the [split][tile][BN][BM] layout when partial, bf16 y otherwise).
template <int BN, int G, int F, int KB>
wq_status launch_bn(const Plan& p, bool partial, int tile0, int ntl, int splits, int kt_per_split,
                    const CUtensorMap& tx, const CUtensorMap& tp, const CUtensorMap& tl,
                    const uint16_t* scale, void* out, int M, int N, int K, cudaStream_t s) {
    const int smem = Smem<BN, F, KB>::TOTAL;
    const dim3 grid(ntl, splits, 1);
    // the shared-memory opt-in is set once per kernel variant (a function attribute holds
    // for the process; the flags are per variant and only ever go from false to true)
    static bool raised[2] = {false, false};
    if (partial) {
        auto k = gemm_kernel<BN, G, true, F, KB>;
        if (!raised[1] && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess)
            raised[1] = true;
        k<<<grid, threads_for(BN), smem, s>>>(tx, tp, tl, scale, out, M, N, K, kt_per_split, p.grid_n, tile0);
    } else {
        auto k = gemm_kernel<BN, G, false, F, KB>;
        if (!raised[0] && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess)
            raised[0] = true;
        k<<<grid, threads_for(BN), smem, s>>>(tx, tp, tl, scale, out, M, N, K, kt_per_split, p.grid_n, tile0);
    }
    return check_launch("gemm");
}

// The plan's launches: one (unsplit, or split everywhere) or two (whole waves unsplit, then
// the split tail), each split launch followed by its reduction.
template <int BN, int G, int F, int KB>
wq_status launch_plan(const Plan& p, const CUtensorMap& tx, const CUtensorMap& tp, const CUtensorMap& tl,
                      const uint16_t* scale, uint16_t* y, void* ws, int M, int N, int K, cudaStream_t s) {
    const int tiles = p.grid_n * p.grid_m;
    auto reduce = [&](int splits, int tile0, int ntl) {
        splitk_reduce_kernel<<<dim3(ntl, BN), BM, 0, s>>>((const float*)ws, splits, ntl, tile0, p.grid_n, BN, M, N, y);
        return check_launch("gemm split-k reduce");
    };
    wq_status st;
    if (p.splits > 1) {
        if ((st = launch_bn<BN, G, F, KB>(p, true, 0, tiles, p.splits, p.kt_per_split, tx, tp, tl, scale, ws, M, N,
                                           K, s)))
            return st;
        return reduce(p.splits, 0, tiles);
    }
    if ((st = launch_bn<BN, G, F, KB>(p, false, 0, p.full, 1, K / KB, tx, tp, tl, scale, y, M, N, K, s))) return st;
    if (p.full == tiles) return WQ_OK;
    if ((st = launch_bn<BN, G, F, KB>(p, true, p.full, tiles - p.full, p.tail_splits, p.tail_kt_per_split, tx, tp,
                                       tl, scale, ws, M, N, K, s)))
        return st;
    return reduce(p.tail_splits, p.full, tiles - p.full);
}

}  // namespace

// Up to this many activation rows the product is decode-shaped: the GEMV kernel (weights
// rebuilt in registers, mma.sync, no TMA/TMEM pipeline) runs it faster than the
// tensor-memory pipeline, whose per-stage bookkeeping dominates when BN is this small.
// Measured on 4096x11008 and 11008x4096: at m = 8, 13.3 / 12.0 us against about 23 us; at
// m = 12, 16.6 / 17.9 us against 20.9 / 22.5 us; at m = 16, 17.9 / 19.9 us against 20.8 /
// 23.4 us (with the GEMV's 128-row CTAs in its cluster split). This is the kernel choice by
// batch size of "K-Means量化技术…" §4.1.
#ifndef WQ_GEMM_GEMV_MAX_ROWS
#define WQ_GEMM_GEMV_MAX_ROWS 16
#endif
constexpr int64_t kGemvMaxRows = WQ_GEMM_GEMV_MAX_ROWS;

// Workspace layout: for LUT16 the scaled fp16 copy of the activations [m, k] (rounded up to
// 1 KB) and the per-row factors 2^-e (fp32 [m], rounded up to 1 KB) first, then the fp32
// partial sums of split launches.
size_t lut16_xh_bytes(const wq_weight& w, int64_t m) {
    return ((size_t)m * (size_t)w.k * 2 + 1023) & ~(size_t)1023;
}
size_t lut16_x_bytes(const wq_weight& w, int64_t m) {
    if (w.fmt != WQ_FMT_LUT16) return 0;
    return lut16_xh_bytes(w, m) + (((size_t)m * 4 + 1023) & ~(size_t)1023);
}

size_t gemm_workspace_bytes(const wq_weight& w, int64_t m, size_t tail_cap) {
    if (m <= kGemvMaxRows) return 0;
    const Plan p = plan_for(m, w.n, w.k, w.fmt, tail_cap);
    const size_t tile = (size_t)BM * (size_t)p.bn * sizeof(float);
    const size_t tiles = (size_t)p.grid_n * (size_t)p.grid_m;
    size_t partial = 0;
    if (p.splits > 1) partial = (size_t)p.splits * tiles * tile;
    else if (p.full < (int)tiles) partial = (size_t)p.tail_splits * (tiles - (size_t)p.full) * tile;
    return lut16_x_bytes(w, m) + partial;
}

wq_status launch_gemm(const wq_weight& w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                      size_t ws_bytes, cudaStream_t s, size_t tail_cap) {
    const int M = (int)m, N = (int)w.n, K = (int)w.k;
    if (m <= kGemvMaxRows) {
        const GemvProblem prob{w.packed, w.aux, x, y, N, K};
        return launch_gemv(w.fmt, w.group, &prob, 1, M, s);
    }
    const Plan p = plan_for(M, N, K, w.fmt, tail_cap);
    auto enc = encode_fn();
    if (!enc) return fail(WQ_ECUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    const size_t need = gemm_workspace_bytes(w, m, tail_cap);
    if (need > 0 && (ws == nullptr || ws_bytes < need)) return fail(WQ_EINVAL, "workspace too small");
    const bool lut = w.fmt == WQ_FMT_LUT16;
    const void* xa = x;                    // the activations the MMA reads
    const float* xinv = nullptr;           // LUT16: per activation row, 2^-e
    if (lut) {
        uint16_t* xh = (uint16_t*)ws;
        float* inv = (float*)((uint8_t*)ws + lut16_xh_bytes(w, m));
        x_to_f16_kernel<<<(unsigned)m, 256, 0, s>>>(x, xh, inv, K);
        wq_status cs = check_launch("gemm activations to fp16");
        if (cs) return cs;
        xa = xh;
        xinv = inv;
        ws = (uint8_t*)ws + lut16_x_bytes(w, m);
    }
#if WQ_DEBUG
    if (!lut) {
        const int64_t n8 = m * (int64_t)K / 8;
        debug_scan_x_kernel<<<(unsigned)std::min<int64_t>((n8 + 255) / 256, 4 * (int64_t)sm_count()), 256, 0, s>>>(
            (const uint4*)x, n8);
        wq_status cs = check_launch("gemm debug activation scan");
        if (cs) return cs;
    }
#endif
    CUtensorMap tx, tp;
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        // one 128-byte swizzle row wide, at most 256 rows (a 384-row tile loads two boxes)
        cuuint32_t box[2] = {64, (cuuint32_t)(p.bn > 256 ? p.bn / 2 : p.bn)};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tx, lut ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         (void*)xa, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for x failed (%d)", (int)r);
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K / 2};
        cuuint32_t box[2] = {(cuuint32_t)(p.kb / 2), (cuuint32_t)BM};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)w.packed, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for packed weights failed (%d)", (int)r);
    }
    CUtensorMap tl = tp;                   // unused by DYADIC4 launches
    if (lut) {
        // centroids [N, K/64, 16] fp16 as a 2D [N, K/4] array; a stage's KB/64 groups are
        // KB/4 entries
        cuuint64_t dims[2] = {(cuuint64_t)K / 4, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K / 2};
        cuuint32_t box[2] = {(cuuint32_t)(p.kb / 4), (cuuint32_t)BM};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void*)w.aux, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for LUT16 centroids failed (%d)", (int)r);
    } else if (w.fmt == WQ_FMT_LLOYD8S) {
        // levels [N, K/32, 8] fp32 as a 2D [N, K/4] array; a stage's 2 groups are 16 floats
        cuuint64_t dims[2] = {(cuuint64_t)K / 4, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)K};
        cuuint32_t box[2] = {(cuuint32_t)(p.kb / 4), (cuuint32_t)BM};
        cuuint32_t es[2] = {1, 1};
        CUresult r = enc(&tl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void*)w.aux, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(WQ_ECUDA, "tensor map for LLOYD8S levels failed (%d)", (int)r);
    }
    // the kernel's `scale`: DYADIC4 the bf16 scales; LUT16 the activation rows' factors
    // (the centroids travel through tmap_l); LLOYD8S unused
    const uint16_t* sc = lut ? (const uint16_t*)xinv : (const uint16_t*)w.aux;
    wq_status st;
#define WQ_BN(BNV, KBV)                                                                                   \
    st = (w.fmt == WQ_FMT_LLOYD8S) ? launch_plan<BNV, 32, kFLl, 64>(p, tx, tp, tl, sc, y, ws, M, N, K, s) \
       : lut                     ? launch_plan<BNV, 64, kFLu, KBV>(p, tx, tp, tl, sc, y, ws, M, N, K, s)  \
       : (w.group == 64)         ? launch_plan<BNV, 64, kFDy, KBV>(p, tx, tp, tl, sc, y, ws, M, N, K, s)  \
                                 : launch_plan<BNV, 32, kFDy, KBV>(p, tx, tp, tl, sc, y, ws, M, N, K, s)
    switch (p.bn) {
        case 16: WQ_BN(16, 64); break;
        case 32: WQ_BN(32, 64); break;
        case 64: WQ_BN(64, 64); break;
        case 128:
            if (p.kb == 128) { WQ_BN(128, 128); } else { WQ_BN(128, 64); }
            break;
        case 384: WQ_BN(384, 64); break;
        default: WQ_BN(256, 64); break;
    }
#undef WQ_BN
    return st;
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
