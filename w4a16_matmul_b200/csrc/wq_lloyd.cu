// wq_lloyd.cu -- codebook producers (placeholder until the kernels land).
#include "wq_internal.cuh"

namespace wq {

wq_status launch_lloyd_g32(const uint16_t*, int64_t, int64_t, int, uint8_t*, uint8_t*, float*,
                           uint8_t*, float*, cudaStream_t) {
    return fail(WQ_EUNSUPPORTED, "wq_quantize_lloyd(G32_WARM) is not built yet");
}

wq_status launch_kmeans16(const uint16_t*, int64_t, int64_t, int, uint8_t*, uint8_t*, uint16_t*,
                          float*, cudaStream_t) {
    return fail(WQ_EUNSUPPORTED, "wq_quantize_lloyd(KMEANS16) is not built yet");
}

}  // namespace wq
