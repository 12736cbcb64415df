// wq_gemm_static.cu -- wq_gemm_w4a16_static: the W4A16 GEMM with its split-K scratch in a
// statically allocated device array, for callers that cannot allocate device memory.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes, present on every
// GPU that loads this library until the process exits. Host code cannot use the array's
// name as a device address (it names a host-side shadow), so the device address is looked
// up with cudaGetSymbolAddress, with the device current, on the first call on a device, and
// cached. The cache entry remembers the CUDA context it was resolved in: after
// cudaDeviceReset the device's next context loads the module again, possibly elsewhere,
// and the next call resolves the address anew.
#include <cuda.h>

#include <mutex>
#include <vector>

#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr size_t kStaticScratchBytes = WQ_GEMM_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_gemm_scratch[kStaticScratchBytes];

// The unique ID of the calling thread's current context (0 if the driver cannot tell).
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = (GetCurrent)p;
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = (GetId)p;
        cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS)
        return id;
    return 0;
}

// Device address of g_gemm_scratch on the current device, resolved on the first use in
// each context of the device.
wq_status scratch_address(void** out) {
    struct Entry {
        void* addr;
        unsigned long long ctx;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(WQ_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    // (0 when no context is current yet: then the lookup, which creates it, runs again)
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, Entry{nullptr, 0});
    if (cache[dev].addr == nullptr || cache[dev].ctx != ctx || ctx == 0) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gemm_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(WQ_ECUDA, "cudaGetSymbolAddress(static GEMM scratch): %s", cudaGetErrorString(e));
        cache[dev] = Entry{p, ctx};
    }
    *out = cache[dev].addr;
    return WQ_OK;
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemm_w4a16_static(const wq_weight* w, const uint16_t* x, int64_t m,
                                          uint16_t* y, wq_stream stream) {
    using namespace wq;
    if (!w) return fail(WQ_EINVAL, "weight descriptor is NULL");
    // planned so that a last-wave split stays within the static scratch
    const size_t need = m < 1 ? 0 : gemm_workspace_bytes(*w, m, kStaticScratchBytes);
    if (need > kStaticScratchBytes)
        return fail(WQ_EINVAL,
                    "this GEMM (n=%lld, k=%lld, m=%lld) needs %zu bytes of scratch; the static scratch "
                    "holds %zu: call wq_gemm_w4a16 with a caller workspace instead",
                    (long long)w->n, (long long)w->k, (long long)m, need, kStaticScratchBytes);
    void* scratch = nullptr;
    if (need > 0) {
        wq_status st = scratch_address(&scratch);
        if (st) return st;
    }
    return gemm_checked(w, x, m, y, scratch, need > 0 ? kStaticScratchBytes : 0, (cudaStream_t)stream,
                        kStaticScratchBytes);
}
