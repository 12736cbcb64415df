// wq_gemm.cu -- W4A16 GEMM on tcgen05 (placeholder until the kernel lands).
#include "wq_internal.cuh"

namespace wq {

size_t gemm_workspace_bytes(const wq_weight&, int64_t) { return 0; }

wq_status launch_gemm(const wq_weight&, const uint16_t*, int64_t, uint16_t*, void*, size_t,
                      cudaStream_t) {
    return fail(WQ_EUNSUPPORTED, "wq_gemm_w4a16 is not built yet");
}

}  // namespace wq
