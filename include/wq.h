/*
 * wq.h -- C ABI of libwq: group-wise 4-bit weight coding and W4A16 matmul on B200
 * (sm_100a).
 *
 * Sources cited below:
 *   [DG]  "MiniCPM5-1B 验证: 6× 压缩, ppl 反超 fp, 1.2GB 显存, 50ms Triton 推理"
 *         (DyadicGumbel 4-bit): §2.1 dyadic codebook, §2.2 block layout and
 *         reconstruction, §2.3 hard argmin, §2.5 nibble pack and unpack-to-bf16.
 *   [KM]  "K-Means量化技术：突破LLM低比特部署瓶颈": §1.2 per-block-64 k-means with
 *         16 centroids, §2.2 LUT decoding, §4.1 kernel choice by batch size.
 *   [G32] "int4-g32+warm 裸量化：原理与实验报告": §1.2 112-candidate shape grid,
 *         §1.3 quantisation flow (candidate argmin, 25 Lloyd rounds, sign bit),
 *         §2 storage format, §5.1-5.2 offline quantisation and inference.
 *   [BX]  "同一个 1B 模型，我上了三种压缩方案：无损的、4bit 的、还有没跑通的", section
 *         "第一剑·完美主义：BF16X": the lossless bf16 block codec.
 *
 * Conventions shared by every entry point
 *   - Matrices are row-major. A weight W is [n, k] = (out, in); groups are runs of
 *     `group` consecutive columns of one row. Activations x are [m, k], outputs y [m, n].
 *   - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - Every pointer is a DEVICE pointer (cudaMalloc / torch CUDA memory) of the current
 *     device, 16-byte aligned, unless a parameter says it may be NULL. Host pointers are
 *     rejected with WQ_EINVAL. The caller allocates and owns every buffer; the library
 *     allocates nothing, frees nothing and keeps no pointer after a call returns.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream)
 *     and runs asynchronously: buffers must stay alive until the stream is synchronised.
 *   - Arguments are checked on the host before anything is launched; on any failure
 *     nothing is launched and the status says why (details in wq_last_error()). A launch
 *     failure reported by the CUDA runtime returns WQ_ECUDA.
 *   - Inputs must be finite. NaN or Inf weights or activations give unspecified codes
 *     and outputs (never a fault).
 *   - Entry points are reentrant; concurrent calls on different streams are safe.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* wq_stream;

typedef enum wq_status {
    WQ_OK = 0,
    WQ_EINVAL = 1,        /* bad size, NULL or non-device pointer, bad format field */
    WQ_EALIGN = 2,        /* pointer not 16-byte aligned */
    WQ_EUNSUPPORTED = 3,  /* valid request this library does not implement (e.g. group) */
    WQ_ECUDA = 4,         /* the CUDA runtime reported an error (launch or attribute query) */
    WQ_ETIMEOUT = 5,      /* a bounded device-side wait gave up (reserved) */
    WQ_EDATA = 6          /* a kernel found inconsistent encoded data (wq_device_error) */
} wq_status;

/* Static description of a status code. Never NULL. */
const char* wq_status_string(int32_t status);

/* Detail of the last failure on the calling host thread ("" if none). Thread-local;
 * valid until the next failing call on that thread. */
const char* wq_last_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t wq_version(void);

/* ------------------------------------------------------------------------------------ */
/* Packed weight descriptor                                                              */
/* ------------------------------------------------------------------------------------ */

typedef enum wq_format {
    /* [DG] §2.1-2.2: code idx in 0..15, w = step * (idx - 8), step = scale / 8, one bf16
     * scale (the group's absmax) per group of 64 or 32. aux = bf16 [n, k/group]. */
    WQ_FMT_DYADIC4 = 0,
    /* [G32] §1.3-2: code = q | sign << 3 (q in 0..7 a magnitude level, sign 1 = negative),
     * w = sign ? -level[q] : level[q]; 8 fp32 magnitude levels per group of 32.
     * aux = fp32 [n, k/32, 8]. */
    WQ_FMT_LLOYD8S = 1,
    /* [KM] §1.2, §2.2: code = centroid index 0..15, w = centroid; 16 fp16 centroids per
     * block of 64. aux = fp16 [n, k/64, 16]. */
    WQ_FMT_LUT16 = 2
} wq_format;

typedef struct wq_weight {
    int32_t fmt;            /* wq_format */
    int32_t group;          /* DYADIC4: 64 or 32; LLOYD8S: 32; LUT16: 64 */
    int64_t n;              /* rows (outputs), >= 1 */
    int64_t k;              /* columns (inputs), >= 1, multiple of group */
    const uint8_t* packed;  /* [n, k/2]: byte j of a row = code[2j] | code[2j+1] << 4
                               ([DG] §2.5 "lo | hi << 4": even column in the low nibble) */
    const void* aux;        /* per-group scale / levels / centroids, see wq_format */
} wq_weight;

/* ------------------------------------------------------------------------------------ */
/* Producers                                                                             */
/* ------------------------------------------------------------------------------------ */

/* Dyadic 4-bit quantisation, [DG] §2.1-2.3 and §2.5. For every group of `group`
 * consecutive weights of a row: scale = max |w| (stored as bf16, exact), and for every
 * weight idx = argmin_j |w - (j - 8) * scale / 8| over j = 0..15, the lowest j on a tie.
 *   w       bf16 [n, k], finite.
 *   group   64 or 32; k % group == 0.
 *   scale   out bf16 [n, k/group].
 *   codes   out uint8 [n, k] (one code per byte), may be NULL.
 *   packed  out uint8 [n, k/2] (two codes per byte, see wq_weight), may be NULL.
 * At least one of codes / packed must be non-NULL. An all-zero group gets scale 0 and
 * codes 0 (every code ties). Output is bit-exact (no floating-point freedom). */
wq_status wq_quantize_dyadic(const uint16_t* w, int64_t n, int64_t k, int32_t group,
                             uint16_t* scale, uint8_t* codes, uint8_t* packed,
                             wq_stream stream);

typedef enum wq_lloyd_mode {
    /* [G32] §1.3: per group of 32 magnitudes, the lowest-MSE of the 112 candidate shapes
     * of §1.2 gives 8 initial levels; `rounds` Lloyd rounds (nearest level, lowest index
     * on a tie; level = mean of its members, an empty level keeps its value) and a
     * final nearest assignment; sign kept as bit 3 of the code. codebook = fp32
     * [n, k/32, 8] levels, params = the per-group byte family << 7 | b_rel index << 3 |
     * beta index of [G32] §2, mse_trace = [n, k/32, rounds + 2] (candidate MSE, then the
     * MSE after each assignment). */
    WQ_LLOYD_G32_WARM = 0,
    /* [KM] §1.2: per block of 64 signed weights, 16 centroids initialised at the
     * (4i+2)-th smallest value, `rounds` Lloyd rounds as above, centroids rounded to
     * fp16 and a final nearest assignment against the fp16 centroids. codebook = fp16
     * [n, k/64, 16] (the LUT16 aux), params unused, mse_trace = [n, k/64, rounds + 1]. */
    WQ_LLOYD_KMEANS16 = 1
} wq_lloyd_mode;

typedef struct wq_lloyd_params {
    int32_t mode;    /* wq_lloyd_mode */
    int32_t rounds;  /* Lloyd rounds, 0..64; the pages use 25 */
} wq_lloyd_params;

/* Codebook quantisation (Lloyd / k-means), [G32] §1.3 and §5.1, [KM] §1.2.
 *   w         bf16 [n, k], finite; k % 32 == 0 (G32_WARM) or k % 64 == 0 (KMEANS16).
 *   codes     out uint8 [n, k], may be NULL.
 *   packed    out uint8 [n, k/2], may be NULL (at least one of codes / packed).
 *   codebook  out, see wq_lloyd_mode.
 *   params    out uint8 [n, k/32] (G32_WARM only), may be NULL.
 *   mse_trace out fp32, see wq_lloyd_mode, may be NULL.
 * Both modes take their decisions in double precision. G32_WARM screens the 112
 * candidates in fp32, bounding each candidate's exact MSE from both sides, and evaluates
 * again in double, with the steps of [G32] §1.3 and the squared errors summed in index
 * order, every candidate whose lower bound does not exceed the smallest upper bound; the
 * lowest double MSE wins (lowest candidate on a tie). Lloyd and k-means member sums run in
 * index order, so repeated calls give identical bits. */
wq_status wq_quantize_lloyd(const uint16_t* w, int64_t n, int64_t k, const wq_lloyd_params* p,
                            uint8_t* codes, uint8_t* packed, void* codebook, uint8_t* params,
                            float* mse_trace, wq_stream stream);

/* ------------------------------------------------------------------------------------ */
/* Packing and reconstruction                                                            */
/* ------------------------------------------------------------------------------------ */

/* [DG] §2.5 pack: packed[r, j] = codes[r, 2j] | codes[r, 2j+1] << 4. codes must be in
 * 0..15 (higher bits are dropped). k even, k % 32 == 0. */
wq_status wq_pack(const uint8_t* codes, int64_t n, int64_t k, uint8_t* packed, wq_stream stream);

/* Inverse of wq_pack: codes[r, 2j] = packed & 15, codes[r, 2j+1] = packed >> 4. */
wq_status wq_unpack(const uint8_t* packed, int64_t n, int64_t k, uint8_t* codes, wq_stream stream);

/* Dense reconstruction of a packed weight ([DG] §2.5 unpack; [G32] §5.2; [KM] §2.2):
 *   DYADIC4 -> bf16(step * (idx - 8)), one rounding to nearest even;
 *   LLOYD8S -> bf16(+/- level[q]);
 *   LUT16   -> the fp16 centroid itself (out holds fp16 patterns).
 *   out  [n, k] 16-bit patterns. Bit-exact. */
wq_status wq_dequant(const wq_weight* w, uint16_t* out, wq_stream stream);

/* STE fake quantisation, forward ([DG] §2.3 "STE"): the forward pass of a QAT step on the
 * fp32 latent weights z. q[r, c] = step * (idx - 8) with idx = argmin_j |z - step * (j - 8)|
 * over j = 0..15 (lowest j on a tie, as wq_quantize_dyadic), step = scale / 8 and scale the
 * bf16 scale of the element's group (a trained parameter, so |z| may exceed it: the argmin
 * then picks an end code). q is the code value itself, exact in fp32. The backward pass of
 * the straight-through estimator is the identity (dL/dz = dL/dq) and needs no call.
 *   z       fp32 [n, k]; k % group == 0 and k % 32 == 0.
 *   group   64 or 32.
 *   scale   bf16 [n, k/group], finite and >= 0 (other scales give unspecified codes).
 *   q       out fp32 [n, k].
 *   codes   out uint8 [n, k] (idx), or NULL.
 *   packed  out uint8 [n, k/2] (idx nibbles, as wq_pack), or NULL.
 * Bit-exact (codes, packed bytes and q). */
wq_status wq_fake_quant_ste(const float* z, int64_t n, int64_t k, int32_t group,
                            const uint16_t* scale, float* q, uint8_t* codes, uint8_t* packed,
                            wq_stream stream);

/* Gumbel-ST soft assignment, backward ([DG] §2.3 "Gumbel-ST"), the page's other QAT
 * estimator: soft = softmax(-dist / tau) . codes, hard = codes[argmin dist],
 * q = hard + (soft - soft.detach()), with codes = step * {-8..7}, step = scale / 8 and
 * dist_j = (z - codes_j)^2 (readings: the squared distance, no noise term since the printed
 * softmax has none, lowest index on an argmin tie). The forward value q is hard itself,
 * exactly what wq_fake_quant_ste returns; this call is the backward for an upstream
 * gradient gq:
 *   gz[r, c]     = gq[r, c] * d soft / d z
 *   gscale[r, g] = sum over the group's c of gq[r, c] * (d hard / d scale + d soft / d scale)
 * (the codes depend on the trained scale, so the hard term adds (idx - 8) / 8).
 *   z       fp32 [n, k] latent; k % group == 0 and k % 32 == 0.
 *   group   64 or 32.
 *   scale   bf16 [n, k/group], finite and >= 0.
 *   tau     temperature, a positive normal float (else WQ_EINVAL). scale^2 / tau must stay
 *           below 2^120 (outputs are unspecified beyond it).
 *   gq      fp32 [n, k] upstream gradient dL/dq, finite.
 *   gz      out fp32 [n, k] = dL/dz.
 *   gscale  out fp32 [n, k/group] = dL/dscale, or NULL.
 * fp32 arithmetic: |gz - gz_ref| <= 1e-4 |gz_ref| + 2^-100 |gq| (1 + 2 step^2 / tau) and
 * |gscale - gscale_ref| <= 1e-4 times the group's sum of |terms| of the exact derivative. */
wq_status wq_gumbel_st_backward(const float* z, int64_t n, int64_t k, int32_t group,
                                const uint16_t* scale, float tau, const float* gq, float* gz,
                                float* gscale, wq_stream stream);

/* ------------------------------------------------------------------------------------ */
/* W4A16 consumers                                                                       */
/* ------------------------------------------------------------------------------------ */

/* Decode-side W4A16 GEMV ([DG] §2.5/§3.2 fused unpack; [KM] §2.2, §4.1 small batch):
 * y[b, r] = sum_c Wdeq[r, c] * x[b, c], fp32 accumulation, bf16 output (rounded to
 * nearest even), for b < batch. Wdeq is the reconstruction wq_dequant gives (bf16 for
 * DYADIC4 / LLOYD8S; for LUT16 the fp16 centroid, multiplied by fp16 activations: each
 * batch row's chunk of x that a thread block stages is converted as x * 2^e, with the
 * power of two chosen from the chunk's largest |x| so that it lands in [2^15, 2^16), and
 * the chunk's fp32 sums are multiplied by 2^-e. Every finite bf16 x is in range; an
 * element more than 2^32 below its chunk's largest magnitude may lose low bits, by less
 * than 2^-40 of that magnitude).
 *   w      packed weight (any format).
 *   x      bf16 [batch, k].
 *   batch  1..16.
 *   y      out bf16 [batch, n].
 * Within |y - y_ref| <= 2e-3 * sum_c |Wdeq[r, c]| * |x[b, c]| + half a bf16 ulp of y_ref of
 * the exact product y_ref (the half ulp is the bf16 output rounding itself).
 * Needs no workspace; one kernel launch. */
wq_status wq_gemv_w4a16(const wq_weight* w, const uint16_t* x, int32_t batch, uint16_t* y,
                        wq_stream stream);

/* Several independent GEMVs in ONE launch (e.g. the q/k/v projections of a decoder layer,
 * which share an input, or a whole stack of layers with independent inputs). Problem i
 * computes ys[i] = Wdeq(ws[i]) xs[i] as wq_gemv_w4a16 does. ws, xs, ys are HOST arrays
 * of `count` entries (the pointers they hold are device pointers); all weights must have
 * the same format and group. count in 1..WQ_GEMV_MAX_GROUPED. */
#define WQ_GEMV_MAX_GROUPED 192
wq_status wq_gemv_w4a16_grouped(const wq_weight* ws, const uint16_t* const* xs,
                                uint16_t* const* ys, int32_t count, int32_t batch,
                                wq_stream stream);

/* A prepared grouped GEMV ("plan"), for a launch repeated over the same buffers, such as
 * every decode step of a model. The pages describe no such object; it exists because the
 * argument checks of wq_gemv_w4a16_grouped (one driver query per pointer) cost about as
 * much host time as a decode sweep's kernel takes on the GPU.
 *   - wq_gemv_plan_create checks the arguments exactly as wq_gemv_w4a16_grouped does,
 *     chooses the kernel variant and its grid once, and keeps the device pointers. On
 *     failure *plan is NULL and nothing is kept.
 *   - wq_gemv_plan_launch enqueues that one kernel on `stream`: a few microseconds of host
 *     time, no argument checks, no allocation, allowed during stream capture. It computes
 *     what wq_gemv_w4a16_grouped would with the buffers' contents when the kernel runs.
 *   - The plan is host memory the library allocates: the one exception to "the library
 *     allocates nothing and keeps no pointer". wq_gemv_plan_destroy frees it (NULL is a
 *     no-op). The buffers must stay allocated while the plan is used; launches may come
 *     from several threads, but no launch may run during or after destroy. */
typedef struct wq_gemv_plan_s* wq_gemv_plan;
wq_status wq_gemv_plan_create(const wq_weight* ws, const uint16_t* const* xs,
                              uint16_t* const* ys, int32_t count, int32_t batch,
                              wq_gemv_plan* plan);
wq_status wq_gemv_plan_launch(wq_gemv_plan plan, wq_stream stream);
void wq_gemv_plan_destroy(wq_gemv_plan plan);

/* Lets each later launch of the plan overlap the kernel before it in the stream
 * (programmatic dependent launch), for decode loops where back-to-back launches would
 * otherwise leave the GPU idle between kernels and during each kernel's last wave. With
 * enable = 1, a launch's thread blocks may start, and load the plan's weights (packed codes
 * and per-group scales, levels or centroids), while the previous kernel's last blocks are
 * still running; they read the activations and write the outputs only after that kernel
 * has completed and its writes are visible. Enable it only when the kernel launched just
 * before the plan does not write the plan's weights (a previous launch of the plan, or any
 * kernel that only produces its activations, is fine). enable = 0 (the default) restores
 * plain stream order. Returns WQ_EINVAL for a NULL plan or another value. Host only; takes
 * effect at the next wq_gemv_plan_launch. The pages describe no such mode. */
wq_status wq_gemv_plan_set_overlap(wq_gemv_plan plan, int32_t enable);

/* Bytes of device workspace wq_gemm_w4a16 needs for this weight and m (0 if none): fp32
 * partial sums where K is split across CTAs (small m, or a last wave of at most half the
 * SMs after up to three whole waves, its partial sums up to 64 MiB), plus LUT16's converted
 * activations. */
size_t wq_gemm_workspace_bytes(const wq_weight* w, int64_t m);

/* Prefill-side W4A16 GEMM on the tcgen05 tensor cores ([KM] §4.1 large batch; [DG] §3.2
 * "materialized" bf16 path fused): y[i, r] = sum_c Wdeq[r, c] * x[i, c] for i < m, fp32
 * accumulation in tensor memory, bf16 output. Formats DYADIC4 (group 64 or 32), LLOYD8S
 * (the 8-level codebook plus sign of [G32] §5.2, rebuilt per stage from the group's levels)
 * and LUT16 (the per-block-64 centroid table of [KM] §2.2, looked up per stage; the product
 * runs in fp16 on the activations converted into the workspace as x * 2^e per activation
 * row, the power of two chosen from the row's largest |x| as in wq_gemv_w4a16, and the
 * epilogue multiplies the row's sums by 2^-e). For m <= 16 the decode-shaped case runs on the
 * GEMV kernel of wq_gemv_w4a16 (the kernel choice by batch size of [KM] §4.1), with the same
 * tolerance and no workspace.
 *   x      bf16 [m, k]; m >= 1; k % 64 == 0.
 *   y      out bf16 [m, n].
 *   ws     device workspace of at least wq_gemm_workspace_bytes(w, m) bytes (NULL if 0);
 *          for LUT16 it includes 2*m*k bytes for the scaled fp16 activations and 4*m for
 *          the rows' factors 2^-e (each rounded up to 1 KB).
 * Same tolerance as wq_gemv_w4a16. */
wq_status wq_gemm_w4a16(const wq_weight* w, const uint16_t* x, int64_t m, uint16_t* y,
                        void* ws, size_t ws_bytes, wq_stream stream);

/* Reads and clears the library's device-side error words. Kernels that wait on the GPU
 * (the GEMM pipeline's mbarrier waits, the water-filled GEMV's waits for its staged bytes)
 * give up after a bounded time instead of hanging and record a nonzero code (the GEMV's
 * is 2100); the BF16X kernels record one when an overflow-table index would pass
 * ovf_bytes, and the water-filling kernels one when a block's width is outside 3..5 or its
 * bytes do not fit packed_bytes (2000 dequant, 2001 pack, 2002 GEMV; the access is skipped
 * in every case). *code receives the code (0 = none). Synchronous (copies three ints from
 * the device). Returns WQ_ETIMEOUT if a wait had expired, WQ_EDATA for inconsistent BF16X
 * or water-filling data, WQ_OK otherwise.
 * The debug build of the library (libwq_debug.so, compiled with -DWQ_DEBUG=1) also checks
 * on the device what the normal build takes as preconditions, records the first failed
 * check of each kernel family and reports it here with WQ_EDATA (the kernels never trap):
 *   3001 / 3010 / 3011 / 3020 / 3030 / 3031  a derived index out of range (dequant scale
 *        index; GEMV problem and tile, staged chunk; GEMM tile and K range; Lloyd candidate;
 *        k-means rank);
 *   3101 / 3102 / 3103  a NaN or Inf weight given to wq_quantize_dyadic / the G32_WARM /
 *        the KMEANS16 producer;
 *   3201 / 3202 / 3203  a NaN or Inf activation given to the GEMV / the LUT16 GEMM / the
 *        other GEMMs;
 *   3301 / 3302 / 3303  a NaN or Inf latent (wq_fake_quant_ste / wq_gumbel_st_backward) or
 *        upstream gradient (wq_gumbel_st_backward).
 * The normal build skips these checks and never reports these codes. */
wq_status wq_device_error(int32_t* code);

/* ------------------------------------------------------------------------------------ */
/* BF16X lossless block codec ([BX] "第一剑·完美主义：BF16X")                              */
/* ------------------------------------------------------------------------------------ */
/* Blocks of 16 consecutive bf16 weights (flat row-major order) share their largest
 * exponent field E; each weight keeps a 3-bit field, E - e when that is at most 6, else 7
 * (escaped: its exponent field goes to an overflow table); sign and mantissa are kept
 * verbatim, so decoding gives back every bit pattern, Inf and NaN included (the one
 * exception to "inputs must be finite"). The page fixes neither bit layout nor the mantissa
 * storage; this library's layout, for a matrix of n*k weights (k % 32 == 0, n*k < 2^32):
 *   sm      uint8 [n, k]: sign << 7 | mantissa, one byte per weight.
 *   hdr     uint64 [n, k/16]: bit 16p + j = bit p of weight j's field (p = 0, 1, 2);
 *           bits 48..55 = E; bits 56..63 = escapes in the earlier blocks of the block's
 *           superblock (16 consecutive blocks).
 *   sb_off  uint32 [S + 1], S = wq_bf16x_superblocks(n, k): escapes before superblock t;
 *           sb_off[S] = total escapes.
 *   ovf     uint8 [total]: exponent fields of the escaped weights in flat order
 *           (ovf_bytes = its allocated size; at least 16 bytes are allocated even if empty).
 * Storage is 12 bits per weight plus 4 bytes per 256 weights plus one byte per escape. */

/* S for an [n, k] matrix, or -1 if k is not a multiple of 16 or n, k < 1. */
int64_t wq_bf16x_superblocks(int64_t n, int64_t k);

/* First encoding pass: sb_off[0..S] = the exclusive escape offsets and the total. The caller
 * reads sb_off[S] back to size ovf, then calls wq_bf16x_encode with the same w and sb_off. */
wq_status wq_bf16x_count(const uint16_t* w, int64_t n, int64_t k, uint32_t* sb_off, wq_stream stream);

/* Second pass: writes sm, hdr and ovf. An escape index at or past ovf_bytes (an sb_off not
 * produced by wq_bf16x_count for this w) is skipped and flagged for wq_device_error. */
wq_status wq_bf16x_encode(const uint16_t* w, int64_t n, int64_t k, const uint32_t* sb_off,
                          uint8_t* sm, uint64_t* hdr, uint8_t* ovf, int64_t ovf_bytes,
                          wq_stream stream);

/* out = the bf16 [n, k] matrix the encoding holds (bit-exact). Overflow reads at or past
 * ovf_bytes are skipped (exponent 0 is used) and flagged for wq_device_error. */
wq_status wq_bf16x_decode(const uint8_t* sm, const uint64_t* hdr, const uint32_t* sb_off,
                          const uint8_t* ovf, int64_t ovf_bytes, int64_t n, int64_t k,
                          uint16_t* out, wq_stream stream);

/* ------------------------------------------------------------------------------------ */
/* Water-filling: 3/4/5-bit dyadic blocks in one level index space ([DG] §2.1, §6)       */
/* ------------------------------------------------------------------------------------ */
/* [DG] §2.1: with half = 2^(b-1) and step = scale / half the b-bit codebook is
 * step * {-half .. half-1}; the 3/4/5-bit codebooks line up, so a block's precision can
 * change without rebuilding the codebook: code idx_b of a b-bit block is code
 * idx_5 = idx_b << (5 - b) of the 5-bit codebook, reconstructed as bf16((scale / 16) *
 * (idx_5 - 16)). [DG] §6 leaves the allocation disabled; this library's reading of it:
 *   block   64 consecutive weights of a row; scale = max |w| (bf16, exact).
 *   codes   idx_b = argmin_j |w - (j - half) * step| over j = 0 .. 2^b - 1, lowest j on a tie.
 *   D_b     the block's squared error sum (w - code)^2 at b bits (each term exact in double,
 *           summed over the block's weights in order, in double).
 *   width   the smallest b in {3, 4, 5} with D_b <= 64 * lambda (the water level lambda, a
 *           squared error per weight), else 5. A bit budget is met by the choice of lambda
 *           (dist lets the caller pick it).
 *   layout  scale bf16 [n, k/64]; width uint8 [n, k/64]; packed: the blocks' bit streams back
 *           to back in row-major block order, block i taking 8 * width_i bytes, code j in
 *           bits [b j, b j + b) counted from bit 0 of the block's first byte (b = 4 gives the
 *           nibble layout of wq_pack); blk_off uint32 [n k/64 + 1]: each block's byte offset,
 *           and the total byte count at the end.
 * k must be a multiple of 64 and n * k / 64 * 40 below 2^32. Results are bit-exact. */

/* Pass 1: scale, width and blk_off for water level lambda (>= 0; +inf gives 3 bits
 * everywhere); dist (may be NULL) receives D_3, D_4, D_5 as fp64 [n, k/64, 3]. The caller
 * reads blk_off[n k/64] back to size packed. */
wq_status wq_quantize_wf_analyze(const uint16_t* w, int64_t n, int64_t k, double lambda,
                                 uint16_t* scale, uint8_t* width, uint32_t* blk_off, double* dist,
                                 wq_stream stream);

/* Pass 2: the codes at each block's width into packed (packed_bytes allocated, at least
 * blk_off[n k/64]). A block that does not fit, or a width outside 3..5, is skipped and
 * flagged for wq_device_error. */
wq_status wq_quantize_wf_pack(const uint16_t* w, int64_t n, int64_t k, const uint16_t* scale,
                              const uint8_t* width, const uint32_t* blk_off, uint8_t* packed,
                              int64_t packed_bytes, wq_stream stream);

/* out = bf16 [n, k] reconstruction through the 5-bit index space (bit-exact). A block
 * outside packed_bytes, or a width outside 3..5, gives zeros and is flagged for
 * wq_device_error. */
wq_status wq_dequant_wf(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                        const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                        uint16_t* out, wq_stream stream);

/* y[i, r] = sum_c Wdeq[r, c] * x[i, c] for i < batch on water-filled weights, Wdeq the
 * reconstruction of wq_dequant_wf (bf16, bit-exact), fp32 products and accumulation, bf16
 * output: the decode-side consumer of the format. The pages give the format (one index
 * space for the 3/4/5-bit codebooks, [DG] §2.1, §6) but no kernel that consumes it; this
 * is the dyadic GEMV's contract on it.
 *   x      bf16 [batch, k]; batch 1 .. 16.
 *   y      out bf16 [batch, n].
 * Same tolerance as wq_gemv_w4a16. A block outside packed_bytes, or a width outside 3..5,
 * contributes nothing and is flagged for wq_device_error (WQ_EDATA). For batches 1 to 4
 * each row's blocks are read in runs of 32: a run whose first or end offset is not a
 * multiple of 8, or that does not lie inside packed_bytes, is not read at all (all of its
 * blocks count as flagged); inside a run, a block is decoded only when the next block's
 * offset (or the run's end) lies exactly 8 * width bytes past its own. */
wq_status wq_gemv_wf(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                     const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                     const uint16_t* x, int32_t batch, uint16_t* y, wq_stream stream);

/* The GEMM above without a caller workspace, for callers that cannot allocate device
 * memory: e.g. an inference server whose caching allocator owns the whole device memory
 * budget and forbids any other cudaMalloc, a plugin that may only use the buffers its host
 * framework hands it, or a latency-critical path that must not pay cudaMalloc's implicit
 * device synchronisation. The pages describe no such entry point; it exists only for them.
 * When m is small and K is split across CTAs, the fp32 partial sums go to a scratch array
 * that the library allocates statically (a file-scope device array of
 * WQ_GEMM_STATIC_SCRATCH_BYTES); every GPU that loads libwq holds that array until the
 * process exits. This entry point itself allocates and frees nothing.
 *   - Same arguments, layout, tolerance and results as wq_gemm_w4a16. A last wave is split
 *     only as far as its partial sums fit the array, so the launches may differ from
 *     wq_gemm_w4a16's where that one would use more.
 *   - A problem whose scratch need still exceeds WQ_GEMM_STATIC_SCRATCH_BYTES (e.g. the
 *     split-K partial sums of a small m) is rejected with WQ_EINVAL; use wq_gemm_w4a16 with
 *     a workspace for it.
 *   - All calls share the one array, which keeps the last call's contents (every call
 *     writes all the scratch it reads, so nothing has to start at zero). Calls whose GPU
 *     work overlaps (e.g. on two streams) race on it: serialise them.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) once and caches it; make that first call before any stream
 *     capture. The cache remembers the context it was filled in: after cudaDeviceReset
 *     the next call on that device looks the address up again (make it, too, outside a
 *     capture). LUT16 also keeps its scaled fp16 activations in the array. */
#define WQ_GEMM_STATIC_SCRATCH_BYTES (16u << 20)
wq_status wq_gemm_w4a16_static(const wq_weight* w, const uint16_t* x, int64_t m, uint16_t* y,
                               wq_stream stream);

/* ------------------------------------------------------------------------------------ */
/* Failure injection (host side only)                                                    */
/* ------------------------------------------------------------------------------------ */

/* Make the next `count` entry points that would launch work fail with WQ_ECUDA before
 * launching anything (for testing callers' error paths without a GPU fault). 0 clears.
 * Process-wide. */
void wq_debug_fail_next_launches(int32_t count);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
