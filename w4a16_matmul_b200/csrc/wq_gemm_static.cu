// wq_gemm_static.cu -- wq_gemm_w4a16_static: the W4A16 GEMM with its split-K scratch in a
// statically allocated device array, for callers that cannot allocate device memory.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes, present on every
// GPU that loads this library until the process exits. Host code cannot use the array's
// name as a device address (it names a host-side shadow), so the device address is looked
// up once per device with cudaGetSymbolAddress and cached.
#include <mutex>
#include <vector>

#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr size_t kStaticScratchBytes = WQ_GEMM_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_gemm_scratch[kStaticScratchBytes];

// Device address of g_gemm_scratch on the current device, resolved on first use.
wq_status scratch_address(void** out) {
    static std::mutex mu;
    static std::vector<void*> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(WQ_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    std::lock_guard<std::mutex> lock(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1, nullptr);
    if (cache[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_gemm_scratch);
        if (e != cudaSuccess || p == nullptr)
            return fail(WQ_ECUDA, "cudaGetSymbolAddress(static GEMM scratch): %s", cudaGetErrorString(e));
        cache[dev] = p;
    }
    *out = cache[dev];
    return WQ_OK;
}

}  // namespace
}  // namespace wq

extern "C" wq_status wq_gemm_w4a16_static(const wq_weight* w, const uint16_t* x, int64_t m,
                                          uint16_t* y, wq_stream stream) {
    using namespace wq;
    if (!w) return fail(WQ_EINVAL, "weight descriptor is NULL");
    const size_t need = wq_gemm_workspace_bytes(w, m);
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
    return wq_gemm_w4a16(w, x, m, y, scratch, need > 0 ? kStaticScratchBytes : 0, stream);
}
