// Fused decode step (placeholder until the persistent kernel lands): reports
// "not supported" so that hata_decode_step runs the granular chain.
#include "hata_kernels.cuh"

namespace hata {

bool fused_step_applies(const hata_dims_t&, int) { return false; }

size_t fused_step_ws_bytes(const hata_dims_t&, int) { return 0; }

cudaError_t launch_fused_step(const hata_dims_t&, const WsLayout&, const void*, const void*, const void*,
                              const float*, uint32_t*, const int32_t*, int, float, void*, uint32_t*, int32_t*, char*,
                              cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace hata
