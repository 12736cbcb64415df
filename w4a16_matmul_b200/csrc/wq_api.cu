// wq_api.cu -- the extern "C" entry points of libwq: argument checks on the host, then one
// launcher call. Nothing is launched when a check fails.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "wq_internal.cuh"

namespace wq {

namespace {
thread_local char g_last_error[512] = "";
std::atomic<int32_t> g_fail_next{0};
}  // namespace

wq_status fail(wq_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

wq_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(WQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
    return WQ_OK;
}

int sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            v = 148;
        }
        cache[dev] = v;
    }
    return cache[dev];
}

namespace {

// A device pointer of the current device (or managed memory), 16-byte aligned.
wq_status check_ptr(const void* p, const char* name, bool nullable) {
    if (p == nullptr) {
        if (nullable) return WQ_OK;
        return fail(WQ_EINVAL, "%s is NULL", name);
    }
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0)
        return fail(WQ_EALIGN, "%s (%p) is not 16-byte aligned", name, p);
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(WQ_EINVAL, "%s (%p): cudaPointerGetAttributes failed: %s", name, p,
                    cudaGetErrorString(e));
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
        return fail(WQ_EINVAL, "%s (%p) is not device memory", name, p);
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && a.type == cudaMemoryTypeDevice && a.device != dev)
        return fail(WQ_EINVAL, "%s (%p) lives on device %d, current device is %d", name, p,
                    a.device, dev);
    return WQ_OK;
}

wq_status check_injected() {
    int32_t v = g_fail_next.load();
    while (v > 0) {
        if (g_fail_next.compare_exchange_weak(v, v - 1))
            return fail(WQ_ECUDA, "injected launch failure (wq_debug_fail_next_launches)");
    }
    return WQ_OK;
}

// Sizes shared by every matrix argument: n, k >= 1, k a multiple of 32 (so that every
// packed row starts on a 16-byte boundary) and of the group; 32-bit addressable rows.
wq_status check_shape(int64_t n, int64_t k, int64_t group) {
    if (n < 1 || k < 1) return fail(WQ_EINVAL, "n=%lld and k=%lld must be >= 1", (long long)n, (long long)k);
    if (n > (1LL << 31) - 1 || k > (1LL << 31) - 1)
        return fail(WQ_EINVAL, "n=%lld or k=%lld exceeds 2^31-1", (long long)n, (long long)k);
    if (k % 32 != 0) return fail(WQ_EINVAL, "k=%lld must be a multiple of 32", (long long)k);
    if (group > 0 && k % group != 0)
        return fail(WQ_EINVAL, "k=%lld is not a multiple of group %lld", (long long)k, (long long)group);
    return WQ_OK;
}

wq_status check_weight(const wq_weight* w) {
    if (!w) return fail(WQ_EINVAL, "weight descriptor is NULL");
    if (w->fmt == WQ_FMT_DYADIC4) {
        if (w->group != 64 && w->group != 32)
            return fail(WQ_EUNSUPPORTED, "DYADIC4 group must be 64 or 32 (got %d)", w->group);
    } else if (w->fmt == WQ_FMT_LLOYD8S) {
        if (w->group != 32) return fail(WQ_EUNSUPPORTED, "LLOYD8S group must be 32 (got %d)", w->group);
    } else if (w->fmt == WQ_FMT_LUT16) {
        if (w->group != 64) return fail(WQ_EUNSUPPORTED, "LUT16 group must be 64 (got %d)", w->group);
    } else {
        return fail(WQ_EINVAL, "unknown weight format %d", w->fmt);
    }
    wq_status st = check_shape(w->n, w->k, w->group);
    if (st) return st;
    if ((st = check_ptr(w->packed, "weight.packed", false))) return st;
    if ((st = check_ptr(w->aux, "weight.aux", false))) return st;
    return WQ_OK;
}

// BF16X sizes: the usual matrix checks, and every escape index below 2^32 (sb_off is uint32)
wq_status check_bf16x_shape(int64_t n, int64_t k) {
    wq_status st = check_shape(n, k, 0);
    if (st) return st;
    if (n * k >= (1LL << 32))
        return fail(WQ_EINVAL, "n*k=%lld must be below 2^32 (32-bit escape offsets)", (long long)(n * k));
    return WQ_OK;
}

}  // namespace
wq_status gemm_checked(const wq_weight* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                       size_t ws_bytes, cudaStream_t stream, size_t tail_cap) {
    g_last_error[0] = 0;
    wq_status st = check_weight(w);
    if (st) return st;
    if (w->k % 64 != 0) return fail(WQ_EINVAL, "GEMM needs k %% 64 == 0 (k=%lld)", (long long)w->k);
    if (m < 1 || m > (1LL << 31) - 1) return fail(WQ_EINVAL, "m=%lld outside 1..2^31-1", (long long)m);
    if ((st = check_ptr(x, "x", false))) return st;
    if ((st = check_ptr(y, "y", false))) return st;
    size_t need = gemm_workspace_bytes(*w, m, tail_cap);
    if (need > 0) {
        if ((st = check_ptr(ws, "ws", false))) return st;
        if (ws_bytes < need)
            return fail(WQ_EINVAL, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
    }
    if ((st = check_injected())) return st;
    return launch_gemm(*w, x, m, y, ws, ws_bytes, stream, tail_cap);
}

}  // namespace wq

using namespace wq;

extern "C" {

const char* wq_status_string(int32_t s) {
    switch (s) {
        case WQ_OK: return "WQ_OK";
        case WQ_EINVAL: return "WQ_EINVAL: invalid argument";
        case WQ_EALIGN: return "WQ_EALIGN: pointer not 16-byte aligned";
        case WQ_EUNSUPPORTED: return "WQ_EUNSUPPORTED: valid request not implemented";
        case WQ_ECUDA: return "WQ_ECUDA: CUDA runtime error";
        case WQ_ETIMEOUT: return "WQ_ETIMEOUT: bounded device wait expired";
        case WQ_EDATA: return "WQ_EDATA: the device found inconsistent encoded data";
        default: return "unknown wq_status";
    }
}

const char* wq_last_error(void) { return g_last_error; }

int32_t wq_version(void) { return 100; }

void wq_debug_fail_next_launches(int32_t count) { g_fail_next.store(count > 0 ? count : 0); }

wq_status wq_device_error(int32_t* code) {
    g_last_error[0] = 0;
    if (!code) return fail(WQ_EINVAL, "code is NULL");
    wq_status st = read_device_error(code);
    if (st) return st;
    int32_t data = 0, wf = 0;
    if ((st = read_bf16x_error(&data))) return st;
    if ((st = read_wf_error(&wf))) return st;
    if (*code != 0) return fail(WQ_ETIMEOUT, "a bounded device wait expired (code %d)", *code);
    if (data != 0) {
        *code = data;
        return fail(WQ_EDATA, "BF16X overflow index past ovf_bytes (code %d)", data);
    }
    if (wf >= 2100) {
        *code = wf;
        return fail(WQ_ETIMEOUT, "a water-filled GEMV's wait for its staged bytes expired (code %d)", wf);
    }
    if (wf != 0) {
        *code = wf;
        return fail(WQ_EDATA, "water-filling block outside packed_bytes or bad width (code %d)", wf);
    }
    // debug build: the first failed device-side check of each kernel family
    wq_status (*readers[])(int32_t*) = {read_debug_dyadic, read_debug_gemv, read_debug_gemm,
                                        read_debug_lloyd, read_debug_ste};
    int32_t first = 0;
    for (auto rd : readers) {
        int32_t v = 0;
        if ((st = rd(&v))) return st;
        if (first == 0) first = v;
    }
    if (first != 0) {
        *code = first;
        return fail(WQ_EDATA, "a device-side debug check failed (code %d)", first);
    }
    return WQ_OK;
}

// Water-filling sizes: the usual matrix checks, k a multiple of 64, and every block offset
// (at most 40 bytes per block) below 2^32.
static wq_status check_wf_shape(int64_t n, int64_t k) {
    wq_status st = check_shape(n, k, 64);
    if (st) return st;
    if (n * (k / 64) * 40 >= (1LL << 32))
        return fail(WQ_EINVAL, "n * k / 64 * 40 bytes must stay below 2^32 (n=%lld, k=%lld)",
                    (long long)n, (long long)k);
    return WQ_OK;
}

wq_status wq_quantize_wf_analyze(const uint16_t* w, int64_t n, int64_t k, double lambda,
                                 uint16_t* scale, uint8_t* width, uint32_t* blk_off, double* dist,
                                 wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_wf_shape(n, k);
    if (st) return st;
    if (!(lambda >= 0.0)) return fail(WQ_EINVAL, "lambda must be >= 0 (got %g)", lambda);
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(width, "width", false))) return st;
    if ((st = check_ptr(blk_off, "blk_off", false))) return st;
    if ((st = check_ptr(dist, "dist", true))) return st;
    if ((st = check_injected())) return st;
    return launch_wf_analyze(w, n, k, lambda, scale, width, blk_off, dist, (cudaStream_t)stream);
}

wq_status wq_quantize_wf_pack(const uint16_t* w, int64_t n, int64_t k, const uint16_t* scale,
                              const uint8_t* width, const uint32_t* blk_off, uint8_t* packed,
                              int64_t packed_bytes, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_wf_shape(n, k);
    if (st) return st;
    if (packed_bytes < 0) return fail(WQ_EINVAL, "packed_bytes must be >= 0");
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(width, "width", false))) return st;
    if ((st = check_ptr(blk_off, "blk_off", false))) return st;
    if ((st = check_ptr(packed, "packed", false))) return st;
    if ((st = check_injected())) return st;
    return launch_wf_pack(w, n, k, scale, width, blk_off, packed, packed_bytes, (cudaStream_t)stream);
}

wq_status wq_dequant_wf(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                        const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                        uint16_t* out, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_wf_shape(n, k);
    if (st) return st;
    if (packed_bytes < 0) return fail(WQ_EINVAL, "packed_bytes must be >= 0");
    if ((st = check_ptr(packed, "packed", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(width, "width", false))) return st;
    if ((st = check_ptr(blk_off, "blk_off", false))) return st;
    if ((st = check_ptr(out, "out", false))) return st;
    if ((st = check_injected())) return st;
    return launch_wf_dequant(packed, packed_bytes, scale, width, blk_off, n, k, out, (cudaStream_t)stream);
}

wq_status wq_gemv_wf(const uint8_t* packed, int64_t packed_bytes, const uint16_t* scale,
                     const uint8_t* width, const uint32_t* blk_off, int64_t n, int64_t k,
                     const uint16_t* x, int32_t batch, uint16_t* y, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_wf_shape(n, k);
    if (st) return st;
    if (packed_bytes < 0) return fail(WQ_EINVAL, "packed_bytes must be >= 0");
    if (batch < 1 || batch > 16) return fail(WQ_EINVAL, "batch=%d outside 1..16", batch);
    if ((st = check_ptr(packed, "packed", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(width, "width", false))) return st;
    if ((st = check_ptr(blk_off, "blk_off", false))) return st;
    if ((st = check_ptr(x, "x", false))) return st;
    if ((st = check_ptr(y, "y", false))) return st;
    if ((st = check_injected())) return st;
    return launch_wf_gemv(packed, packed_bytes, scale, width, blk_off, n, k, x, batch, y, (cudaStream_t)stream);
}

int64_t wq_bf16x_superblocks(int64_t n, int64_t k) {
    if (n < 1 || k < 1 || k % 16 != 0) return -1;
    return bf16x_superblocks(n, k);
}

wq_status wq_bf16x_count(const uint16_t* w, int64_t n, int64_t k, uint32_t* sb_off, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_bf16x_shape(n, k);
    if (st) return st;
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(sb_off, "sb_off", false))) return st;
    if ((st = check_injected())) return st;
    return launch_bf16x_count(w, n, k, sb_off, (cudaStream_t)stream);
}

wq_status wq_bf16x_encode(const uint16_t* w, int64_t n, int64_t k, const uint32_t* sb_off,
                          uint8_t* sm, uint64_t* hdr, uint8_t* ovf, int64_t ovf_bytes,
                          wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_bf16x_shape(n, k);
    if (st) return st;
    if (ovf_bytes < 0) return fail(WQ_EINVAL, "ovf_bytes=%lld is negative", (long long)ovf_bytes);
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(sb_off, "sb_off", false))) return st;
    if ((st = check_ptr(sm, "sm", false))) return st;
    if ((st = check_ptr(hdr, "hdr", false))) return st;
    if ((st = check_ptr(ovf, "ovf", false))) return st;
    if ((st = check_injected())) return st;
    return launch_bf16x_encode(w, n, k, sb_off, sm, hdr, ovf, ovf_bytes, (cudaStream_t)stream);
}

wq_status wq_bf16x_decode(const uint8_t* sm, const uint64_t* hdr, const uint32_t* sb_off,
                          const uint8_t* ovf, int64_t ovf_bytes, int64_t n, int64_t k,
                          uint16_t* out, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_bf16x_shape(n, k);
    if (st) return st;
    if (ovf_bytes < 0) return fail(WQ_EINVAL, "ovf_bytes=%lld is negative", (long long)ovf_bytes);
    if ((st = check_ptr(sm, "sm", false))) return st;
    if ((st = check_ptr(hdr, "hdr", false))) return st;
    if ((st = check_ptr(sb_off, "sb_off", false))) return st;
    if ((st = check_ptr(ovf, "ovf", false))) return st;
    if ((st = check_ptr(out, "out", false))) return st;
    if ((st = check_injected())) return st;
    return launch_bf16x_decode(sm, hdr, sb_off, ovf, ovf_bytes, n, k, out, (cudaStream_t)stream);
}

wq_status wq_quantize_dyadic(const uint16_t* w, int64_t n, int64_t k, int32_t group,
                             uint16_t* scale, uint8_t* codes, uint8_t* packed, wq_stream stream) {
    g_last_error[0] = 0;
    if (group != 64 && group != 32)
        return fail(WQ_EUNSUPPORTED, "dyadic group must be 64 or 32 (got %d)", group);
    wq_status st = check_shape(n, k, group);
    if (st) return st;
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(codes, "codes", true))) return st;
    if ((st = check_ptr(packed, "packed", true))) return st;
    if (!codes && !packed) return fail(WQ_EINVAL, "codes and packed are both NULL");
    if ((st = check_injected())) return st;
    return launch_quantize_dyadic(w, n, k, group, scale, codes, packed, (cudaStream_t)stream);
}

wq_status wq_quantize_lloyd(const uint16_t* w, int64_t n, int64_t k, const wq_lloyd_params* p,
                            uint8_t* codes, uint8_t* packed, void* codebook, uint8_t* params,
                            float* mse_trace, wq_stream stream) {
    g_last_error[0] = 0;
    if (!p) return fail(WQ_EINVAL, "params is NULL");
    if (p->rounds < 0 || p->rounds > 64) return fail(WQ_EINVAL, "rounds=%d outside 0..64", p->rounds);
    int group;
    if (p->mode == WQ_LLOYD_G32_WARM) group = 32;
    else if (p->mode == WQ_LLOYD_KMEANS16) group = 64;
    else return fail(WQ_EINVAL, "unknown lloyd mode %d", p->mode);
    wq_status st = check_shape(n, k, group);
    if (st) return st;
    if ((st = check_ptr(w, "w", false))) return st;
    if ((st = check_ptr(codes, "codes", true))) return st;
    if ((st = check_ptr(packed, "packed", true))) return st;
    if ((st = check_ptr(codebook, "codebook", false))) return st;
    if ((st = check_ptr(params, "params", true))) return st;
    if ((st = check_ptr(mse_trace, "mse_trace", true))) return st;
    if (!codes && !packed) return fail(WQ_EINVAL, "codes and packed are both NULL");
    if ((st = check_injected())) return st;
    if (p->mode == WQ_LLOYD_G32_WARM)
        return launch_lloyd_g32(w, n, k, p->rounds, codes, packed, (float*)codebook, params,
                                mse_trace, (cudaStream_t)stream);
    return launch_kmeans16(w, n, k, p->rounds, codes, packed, (uint16_t*)codebook, mse_trace,
                           (cudaStream_t)stream);
}

wq_status wq_pack(const uint8_t* codes, int64_t n, int64_t k, uint8_t* packed, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_shape(n, k, 0);
    if (st) return st;
    if ((st = check_ptr(codes, "codes", false))) return st;
    if ((st = check_ptr(packed, "packed", false))) return st;
    if ((st = check_injected())) return st;
    return launch_pack(codes, n, k, packed, (cudaStream_t)stream);
}

wq_status wq_unpack(const uint8_t* packed, int64_t n, int64_t k, uint8_t* codes, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_shape(n, k, 0);
    if (st) return st;
    if ((st = check_ptr(packed, "packed", false))) return st;
    if ((st = check_ptr(codes, "codes", false))) return st;
    if ((st = check_injected())) return st;
    return launch_unpack(packed, n, k, codes, (cudaStream_t)stream);
}

wq_status wq_dequant(const wq_weight* w, uint16_t* out, wq_stream stream) {
    g_last_error[0] = 0;
    wq_status st = check_weight(w);
    if (st) return st;
    if ((st = check_ptr(out, "out", false))) return st;
    if ((st = check_injected())) return st;
    return launch_dequant(*w, out, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

// The checks of a grouped GEMV call; fills probs[0..count).
wq_status check_grouped(const wq_weight* ws, const uint16_t* const* xs, uint16_t* const* ys,
                        int32_t count, int32_t batch, GemvProblem* probs) {
    if (!ws || !xs || !ys) return fail(WQ_EINVAL, "ws, xs and ys must be non-NULL host arrays");
    if (count < 1 || count > WQ_GEMV_MAX_GROUPED)
        return fail(WQ_EINVAL, "count=%d outside 1..%d", count, WQ_GEMV_MAX_GROUPED);
    if (batch < 1 || batch > 16) return fail(WQ_EINVAL, "batch=%d outside 1..16", batch);
    for (int i = 0; i < count; ++i) {
        wq_status st = check_weight(&ws[i]);
        if (st) return st;
        if (ws[i].fmt != ws[0].fmt || ws[i].group != ws[0].group)
            return fail(WQ_EINVAL, "problem %d: all grouped weights must share format and group", i);
        if ((st = check_ptr(xs[i], "x", false))) return st;
        if ((st = check_ptr(ys[i], "y", false))) return st;
        probs[i] = GemvProblem{ws[i].packed, ws[i].aux, xs[i], ys[i], (int32_t)ws[i].n, (int32_t)ws[i].k};
    }
    return WQ_OK;
}

}  // namespace

extern "C" {

wq_status wq_fake_quant_ste(const float* z, int64_t n, int64_t k, int32_t group,
                            const uint16_t* scale, float* q, uint8_t* codes, uint8_t* packed,
                            wq_stream stream) {
    g_last_error[0] = 0;
    if (group != 64 && group != 32)
        return fail(WQ_EUNSUPPORTED, "fake quantisation group must be 64 or 32 (got %d)", group);
    wq_status st = check_shape(n, k, group);
    if (st) return st;
    if ((st = check_ptr(z, "z", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(q, "q", false))) return st;
    if ((st = check_ptr(codes, "codes", true))) return st;
    if ((st = check_ptr(packed, "packed", true))) return st;
    if ((st = check_injected())) return st;
    return launch_fake_quant_ste(z, n, k, group, scale, q, codes, packed, (cudaStream_t)stream);
}

wq_status wq_gumbel_st_backward(const float* z, int64_t n, int64_t k, int32_t group,
                                const uint16_t* scale, float tau, const float* gq, float* gz,
                                float* gscale, wq_stream stream) {
    g_last_error[0] = 0;
    if (group != 64 && group != 32)
        return fail(WQ_EUNSUPPORTED, "Gumbel-ST group must be 64 or 32 (got %d)", group);
    if (!(tau > 0.0f) || !(tau <= 3.0e38f) || tau < 1.17549435e-38f)
        return fail(WQ_EINVAL, "tau must be a positive normal finite float (got %g)", (double)tau);
    wq_status st = check_shape(n, k, group);
    if (st) return st;
    if ((st = check_ptr(z, "z", false))) return st;
    if ((st = check_ptr(scale, "scale", false))) return st;
    if ((st = check_ptr(gq, "gq", false))) return st;
    if ((st = check_ptr(gz, "gz", false))) return st;
    if ((st = check_ptr(gscale, "gscale", true))) return st;
    if ((st = check_injected())) return st;
    return launch_gumbel_st_backward(z, n, k, group, scale, tau, gq, gz, gscale, (cudaStream_t)stream);
}

wq_status wq_gemv_plan_create(const wq_weight* ws, const uint16_t* const* xs, uint16_t* const* ys,
                              int32_t count, int32_t batch, wq_gemv_plan* plan) {
    g_last_error[0] = 0;
    if (!plan) return fail(WQ_EINVAL, "plan must be a non-NULL host pointer");
    *plan = nullptr;
    GemvProblem probs[WQ_GEMV_MAX_GROUPED];
    wq_status st = check_grouped(ws, xs, ys, count, batch, probs);
    if (st) return st;
    void* p = nullptr;
    if ((st = gemv_plan_build(ws[0].fmt, ws[0].group, probs, count, batch, &p))) return st;
    *plan = reinterpret_cast<wq_gemv_plan>(p);
    return WQ_OK;
}

wq_status wq_gemv_plan_launch(wq_gemv_plan plan, wq_stream stream) {
    g_last_error[0] = 0;
    if (!plan) return fail(WQ_EINVAL, "plan is NULL");
    wq_status st = check_injected();
    if (st) return st;
    return gemv_plan_launch(plan, (cudaStream_t)stream);
}

wq_status wq_gemv_plan_set_overlap(wq_gemv_plan plan, int32_t enable) {
    g_last_error[0] = 0;
    if (!plan) return fail(WQ_EINVAL, "plan is NULL");
    if (enable != 0 && enable != 1) return fail(WQ_EINVAL, "enable must be 0 or 1, got %d", enable);
    gemv_plan_set_overlap(plan, enable == 1);
    return WQ_OK;
}

void wq_gemv_plan_destroy(wq_gemv_plan plan) {
    if (plan) gemv_plan_free(plan);
}

wq_status wq_gemv_w4a16_grouped(const wq_weight* ws, const uint16_t* const* xs,
                                uint16_t* const* ys, int32_t count, int32_t batch,
                                wq_stream stream) {
    g_last_error[0] = 0;
    GemvProblem probs[WQ_GEMV_MAX_GROUPED];
    wq_status st = check_grouped(ws, xs, ys, count, batch, probs);
    if (st) return st;
    if ((st = check_injected())) return st;
    return launch_gemv(ws[0].fmt, ws[0].group, probs, count, batch, (cudaStream_t)stream);
}

wq_status wq_gemv_w4a16(const wq_weight* w, const uint16_t* x, int32_t batch, uint16_t* y,
                        wq_stream stream) {
    if (!w) { g_last_error[0] = 0; return fail(WQ_EINVAL, "weight descriptor is NULL"); }
    return wq_gemv_w4a16_grouped(w, &x, &y, 1, batch, stream);
}

size_t wq_gemm_workspace_bytes(const wq_weight* w, int64_t m) {
    if (!w || m < 1) return 0;
    return gemm_workspace_bytes(*w, m);
}


wq_status wq_gemm_w4a16(const wq_weight* w, const uint16_t* x, int64_t m, uint16_t* y, void* ws,
                        size_t ws_bytes, wq_stream stream) {
    return gemm_checked(w, x, m, y, ws, ws_bytes, (cudaStream_t)stream, kGemmTailScratch);
}

}  // extern "C"
