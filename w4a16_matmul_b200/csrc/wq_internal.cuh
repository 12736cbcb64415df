// wq_internal.cuh -- declarations shared by the translation units of libwq (sm_100a).
// Nothing here is part of the public ABI (include/wq.h is).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include <cstddef>

#include "wq.h"

namespace wq {

// ---------------------------------------------------------------------------------------
// Debug build (-DWQ_DEBUG=1, libwq_debug.so): device-side checks of derived indices and of
// the finite-input precondition. A failed check records its code in the translation
// unit's debug word (the first code wins), skips nothing else and never traps; the host
// reads and clears the words through wq_device_error (WQ_EDATA). In the normal build the
// checks compile to nothing and the readers report 0.
// ---------------------------------------------------------------------------------------
#ifndef WQ_DEBUG
#define WQ_DEBUG 0
#endif
enum : int {
    kDbgIndex = 3000,              // + site: a derived index outside its range
    kDbgNonFiniteWeight = 3100,    // + site: a NaN / Inf weight reached a producer
    kDbgNonFiniteActivation = 3200,  // + site: a NaN / Inf activation reached a consumer
    kDbgNonFiniteLatent = 3300,    // + site: a NaN / Inf latent or gradient reached the STE kernels
};
#if WQ_DEBUG
// Defines this translation unit's debug word, debug_fail() and the reader read_debug_<name>.
#define WQ_DEBUG_WORD(name)                                                                   \
    static __device__ int g_debug_word;                                                       \
    __device__ __forceinline__ void debug_fail(int code) { atomicCAS(&g_debug_word, 0, code); } \
    wq_status read_debug_##name(int32_t* code) {                                              \
        int v = 0;                                                                            \
        if (cudaMemcpyFromSymbol(&v, g_debug_word, sizeof v) != cudaSuccess)                  \
            return fail(WQ_ECUDA, "reading the debug word of " #name);                         \
        if (v != 0) {                                                                         \
            const int zero = 0;                                                               \
            cudaMemcpyToSymbol(g_debug_word, &zero, sizeof zero);                             \
        }                                                                                     \
        *code = v;                                                                            \
        return WQ_OK;                                                                         \
    }
#define WQ_DCHECK(cond, code)                 \
    do {                                      \
        if (!(cond)) debug_fail(code);        \
    } while (0)
#else
#define WQ_DEBUG_WORD(name)                          \
    wq_status read_debug_##name(int32_t* code) {     \
        *code = 0;                                   \
        return WQ_OK;                                \
    }
#define WQ_DCHECK(cond, code) \
    do {                      \
    } while (0)
#endif
wq_status read_debug_dyadic(int32_t* code);
wq_status read_debug_gemv(int32_t* code);
wq_status read_debug_gemm(int32_t* code);
wq_status read_debug_lloyd(int32_t* code);
wq_status read_debug_ste(int32_t* code);

// True when none of the eight bf16 values of v is a NaN or an infinity.
__host__ __device__ __forceinline__ bool bf16x8_finite(uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 4; ++i) ok = ok && (w[i] & 0x7F80u) != 0x7F80u && (w[i] & 0x7F800000u) != 0x7F800000u;
    return ok;
}

// True when none of the four fp32 values (bits) of v is a NaN or an infinity.
__host__ __device__ __forceinline__ bool f32x4_finite(uint4 v) {
    return (v.x & 0x7F800000u) != 0x7F800000u && (v.y & 0x7F800000u) != 0x7F800000u &&
           (v.z & 0x7F800000u) != 0x7F800000u && (v.w & 0x7F800000u) != 0x7F800000u;
}

// ---------------------------------------------------------------------------------------
// Host-side status plumbing (wq_api.cu)
// ---------------------------------------------------------------------------------------

// Records a formatted failure message for wq_last_error() and returns `st`.
wq_status fail(wq_status st, const char* fmt, ...);

// Converts the CUDA runtime's last launch error into a status (clears it).
wq_status check_launch(const char* what);

// ---------------------------------------------------------------------------------------
// Kernel launchers (each returns after enqueueing; arguments already validated)
// ---------------------------------------------------------------------------------------

wq_status launch_quantize_dyadic(const uint16_t* w, int64_t n, int64_t k, int group,
                                 uint16_t* scale, uint8_t* codes, uint8_t* packed,
                                 cudaStream_t s);
wq_status launch_pack(const uint8_t* codes, int64_t n, int64_t k, uint8_t* packed, cudaStream_t s);
wq_status launch_fake_quant_ste(const float* z, int64_t n, int64_t k, int group,
                                const uint16_t* scale, float* q, uint8_t* codes, uint8_t* packed,
                                cudaStream_t s);
wq_status launch_gumbel_st_backward(const float* z, int64_t n, int64_t k, int group,
                                    const uint16_t* scale, float tau, const float* gq, float* gz,
                                    float* gscale, cudaStream_t s);
wq_status launch_unpack(const uint8_t* packed, int64_t n, int64_t k, uint8_t* codes, cudaStream_t s);
wq_status launch_dequant(const wq_weight& w, uint16_t* out, cudaStream_t s);

struct GemvProblem {
    const uint8_t* packed;
    const void* aux;
    const uint16_t* x;
    uint16_t* y;
    int32_t n, k;
};
wq_status launch_gemv(int fmt, int group, const GemvProblem* probs, int count, int batch,
                      cudaStream_t s);

// A prepared grouped GEMV (kernel variant, grid and parameters chosen once): built on the
// host heap, launched any number of times, freed by gemv_plan_free.
wq_status gemv_plan_build(int fmt, int group, const GemvProblem* probs, int count, int batch,
                          void** plan);
wq_status gemv_plan_launch(const void* plan, cudaStream_t s);
void gemv_plan_set_overlap(void* plan, bool on);
void gemv_plan_free(void* plan);

wq_status launch_lloyd_g32(const uint16_t* w, int64_t n, int64_t k, int rounds, uint8_t* codes,
                           uint8_t* packed, float* levels, uint8_t* params, float* trace,
                           cudaStream_t s);
wq_status launch_kmeans16(const uint16_t* w, int64_t n, int64_t k, int rounds, uint8_t* codes,
                          uint8_t* packed, uint16_t* lut, float* trace, cudaStream_t s);

// The GEMM's last-wave split may use up to tail_cap bytes of fp32 partial sums (the static
// scratch entry plans with its own, smaller cap).
constexpr size_t kGemmTailScratch = (size_t)64 << 20;
size_t gemm_workspace_bytes(const wq_weight& w, int64_t m, size_t tail_cap = kGemmTailScratch);
wq_status launch_gemm(const wq_weight& w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                      size_t ws_bytes, cudaStream_t s, size_t tail_cap = kGemmTailScratch);
// wq_gemm_w4a16's argument checks and launch, planned with the given tail cap.
wq_status gemm_checked(const wq_weight* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                       size_t ws_bytes, cudaStream_t s, size_t tail_cap);

// Reads and clears the device error word written by expired bounded waits.
wq_status read_device_error(int32_t* code);

// BF16X lossless codec (wq_bf16x.cu)
int64_t bf16x_superblocks(int64_t n, int64_t k);
wq_status launch_bf16x_count(const uint16_t* w, int64_t n, int64_t k, uint32_t* sb_off, cudaStream_t s);
wq_status launch_bf16x_encode(const uint16_t* w, int64_t n, int64_t k, const uint32_t* sb_off,
                              uint8_t* sm, uint64_t* hdr, uint8_t* ovf, int64_t ovf_cap, cudaStream_t s);
wq_status launch_bf16x_decode(const uint8_t* sm, const uint64_t* hdr, const uint32_t* sb_off,
                              const uint8_t* ovf, int64_t ovf_cap, int64_t n, int64_t k,
                              uint16_t* out, cudaStream_t s);
wq_status read_bf16x_error(int32_t* code);

// In-place exclusive scan of count 8-bit values held in the low byte of a[0..count), total
// in a[count], for values written by a pass that also stored, in bits 8..31 of the last
// entry of every tile of kScanTile entries, that tile's total (see wq_bf16x.cu).
constexpr int kScanTile = 256;
wq_status launch_tile_scan_u8(uint32_t* a, int64_t count, cudaStream_t s);

// Water-filling 3/4/5-bit dyadic blocks (wq_wf.cu).
wq_status launch_wf_analyze(const uint16_t* w, int64_t n, int64_t k, double lambda, uint16_t* scale,
                            uint8_t* width, uint32_t* blk_off, double* dist, cudaStream_t s);
wq_status launch_wf_pack(const uint16_t* w, int64_t n, int64_t k, const uint16_t* scale,
                         const uint8_t* width, const uint32_t* blk_off, uint8_t* packed,
                         int64_t packed_bytes, cudaStream_t s);
wq_status launch_wf_dequant(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                            const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                            uint16_t* out, cudaStream_t s);
wq_status launch_wf_gemv(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                         const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                         const uint16_t* x, int batch, uint16_t* y, cudaStream_t s);
wq_status read_wf_error(int32_t* code);

// Number of SMs of the current device (cached per device).
int sm_count();

// ---------------------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) {
    return __uint_as_float(h << 16);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint32_t float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// mbarrier helpers (shared::cta): init, plain arrive, arrive that also announces the bytes
// the asynchronous copies of the phase will deliver, and a bounded wait.
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

constexpr uint64_t kWaitNs = 2000000000ull;   // a device wait longer than 2 s is declared dead
#ifndef WQ_MBAR_SUSPEND_NS
#define WQ_MBAR_SUSPEND_NS 20000
#endif
// Bounded wait for the completion of phase `parity`: gives up after about two seconds of
// wall time and returns false. Each try_wait may suspend the thread for up to
// WQ_MBAR_SUSPEND_NS nanoseconds (it wakes as soon as the phase completes), so a waiting
// warp does not spin on issue slots other warps need.
// `abort` (shared memory) is polled only while the wait spins, so that a CTA whose other
// role gave up stops waiting at once instead of timing out wait by wait.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, const int* abort = nullptr) {
    const uint32_t a = smem_u32(b);
    uint64_t deadline = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
            : "=r"(done) : "r"(a), "r"(parity), "r"((uint32_t)WQ_MBAR_SUSPEND_NS) : "memory");
        if (done) return true;
        if ((i & 7) == 0) {
            if (abort && *(volatile const int*)abort) return false;
            const uint64_t now = global_ns();
            if (deadline == 0) deadline = now + kWaitNs;
            else if (now > deadline) return false;
        }
    }
}

// Asynchronous bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar` (complete_tx). No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Asks the L2 to fetch [p, p + bytes) from memory ahead of use (a hint; p and bytes must be
// multiples of 16 and the range must lie inside one allocation).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Predicated 128-bit load: when `pred` is 0 the registers keep their previous contents
// (no zero fill, no extra moves).
__device__ __forceinline__ void ldg_v4_if(uint4& v, const void* p, uint32_t pred) {
    asm volatile(
        "{ .reg .pred q; setp.ne.b32 q, %5, 0; @q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4]; }"
        : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w) : "l"(p), "r"(pred));
}

// 128-bit store with the streaming (evict-first) cache hint: output written once and not
// read again by this kernel.
__device__ __forceinline__ void stg_cs_v4(void* p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// LLOYD8S lookup of 4 codes (nibbles of the low 16 bits of s; code = level index q in bits
// 0-2, sign in bit 3) in an 8-entry bf16 table of one group held as byte planes: lo[0..1] /
// hi[0..1] hold the low / high bytes of bf16(level[0..7]). The sign bit of each code flips
// the sign bit of the high byte (bf16(-v) = -bf16(v): rounding to nearest even is
// symmetric). Returns the bf16 pairs (code0, code1) and (code2, code3).
__device__ __forceinline__ void lloyd8_lookup4(uint32_t s, const uint32_t* lo, const uint32_t* hi,
                                               uint32_t& p01, uint32_t& p23) {
    const uint32_t s7 = s & 0x7777u;                                     // level index
    // 0xFF where the code's sign bit (bit 3) is set: prmt's sign-replicate selector mode on
    // the byte whose top bit it is (s for codes 1 and 3, s << 4 for codes 0 and 2)
    const uint32_t sg = prmt(s, s << 4, 0x9D8Cu);
    const uint32_t l = prmt(lo[0], lo[1], s7);
    const uint32_t h = prmt(hi[0], hi[1], s7) ^ (sg & 0x80808080u);
    p01 = prmt(l, h, 0x5140u);
    p23 = prmt(l, h, 0x7362u);
}

// LUT16 lookup of 4 codes (nibbles of the low 16 bits of s) in a 16-entry fp16 table held
// as byte planes: lo[q] / hi[q] hold the low / high bytes of entries 4q..4q+3. Returns the
// fp16 pairs (code0, code1) and (code2, code3).
// The byte mask (0xFF where code >= 8) comes from prmt's sign-replicate selector mode: the
// codes' bit 3 is the top bit of a byte of s (codes 1, 3) or of s << 4 (codes 0, 2).
__device__ __forceinline__ void lut16_lookup4(uint32_t s, const uint32_t* lo, const uint32_t* hi,
                                              uint32_t& p01, uint32_t& p23) {
    const uint32_t s7 = s & 0x7777u;                                  // index within 8 entries
    const uint32_t m = prmt(s, s << 4, 0x9D8Cu);                      // byte mask: code >= 8
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

// fp16 activations for the LUT16 products. A bf16 row (or chunk) is converted as x * 2^e,
// with e chosen from its largest magnitude so that this maximum lands in [2^15, 2^16) (all
// of bf16's binades map into fp16 that way, and every magnitude of the row down to 2^-17 *
// 2^-e converts exactly); the fp32 sums are multiplied back by 2^-e. `mag` is the largest
// bf16 magnitude (bits & 0x7FFF); 0 or a non-finite maximum gives e = 0. e lies in
// [-113, 148].
__device__ __forceinline__ int lut_x_exponent(uint32_t mag) {
    if (mag == 0 || mag >= 0x7F80u) return 0;
    const int E = (int)(mag >> 7);                 // biased exponent; 0 for subnormals
    return E ? 142 - E : 117 + __clz(mag & 0x7Fu);
}
// 2^e as an fp32 for e in [-149, 127] (subnormal below -126), exact.
__device__ __forceinline__ float pow2_f32(int e) {
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149));
}
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
// The largest magnitude among the eight (finite) bf16 values of v, as bits.
__device__ __forceinline__ uint32_t bf16x8_max_mag(uint4 v) {
    const uint32_t m = bf16x2_max(bf16x2_max(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                  bf16x2_max(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16);
}
// bf16 pair -> fp16 pair of the values times 2^e for e in [-133, 127] (2^e a bf16 number,
// given as the pair p2 = (2^e, 2^e)): one exact bf16 product (wherever fp16 can hold the
// result), then one rounding to fp16.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_pow2(uint32_t v, uint32_t p2) {
    const uint32_t m = bf16x2_fma(v, p2, 0x80008000u);
    const float lo = __uint_as_float(m << 16), hi = __uint_as_float(m & 0xFFFF0000u);
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// The bf16 bits of 2^e, e in [-133, 127].
__device__ __forceinline__ uint32_t bf16_pow2_bits(int e) {
    return e >= -126 ? (uint32_t)(e + 127) << 7 : 1u << (e + 133);
}
// bf16 pair -> fp16 pair of the values times 2^e, one rounding to nearest even (the fp32
// products by s1 = 2^(e>>1) and s2 = 2^(e - (e>>1)) are exact wherever fp16 can hold the
// result).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t v, float s1, float s2) {
    const float lo = __uint_as_float(v << 16) * s1 * s2, hi = __uint_as_float(v & 0xFFFF0000u) * s1 * s2;
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// The MMAs below have no side effect beyond their outputs, so they are plain (not volatile)
// asm, which leaves the compiler free to schedule them.
// D += A * B on the legacy warp-level tensor-core path, m16n8k16, bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Same with fp16 operands.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t a2, uint32_t a3, uint32_t b0,
                                              uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace wq
