// End-to-end decode-step loop through libhata's public C ABI, for the benchmark's
// end-to-end figure.  Every step:
//   1. one host-to-device copy of the step's inputs from pinned host memory into a
//      device staging buffer: the queries, then the new token's K rows and V rows;
//   2. hata_append_kv: the new rows go to slot L_b - 1 of the K and V caches;
//   3. hata_decode_step on the staged queries, its output written straight into
//      the pinned host output buffer (mapped into the device's address space, so
//      the result crosses to the host inside the step, with no separate copy);
//   4. a stream synchronize, after which the host holds the step's output.
// Native code, so that the loop measures the library and the transfers rather
// than an interpreter.
#include <cuda_runtime.h>

#include <chrono>
#include <cstdint>

#include "hata.h"

extern "C" {

// Runs `steps` end-to-end steps over R layers' buffers (layer i % R at step i).
//   in_host   pinned [B*Hq + 2*B*Hkv][d] (dims->dtype): q [B][Hq][d], then the new
//             K rows [B][Hkv][d], then the new V rows [B][Hkv][d]
//   out_host  pinned [B][Hq][d] (dims->dtype), device-accessible (mapped)
//   stage[R]  device buffers shaped like in_host, 16-byte aligned
//   K, V, W, codes, lens: each layer's caches, W_H, code cache and seq_lens
// Writes the device-side elapsed milliseconds (CUDA events around the loop, on
// `stream`) and the host wall-clock milliseconds.  Returns a hata_status_t, or
// HATA_ERR_CUDA when a copy, an event or the output mapping fails.
HATA_API int hata_e2e_run(const hata_dims_t* dims, int k, int steps, int R, const void* in_host, void* out_host,
                          void* const* stage, void* const* K, void* const* V, const float* const* W,
                          uint32_t* const* codes, const int32_t* const* lens, void* ws, size_t ws_bytes,
                          void* stream, float* device_ms, float* host_ms) {
  if (!dims || steps < 1 || R < 1 || !in_host || !out_host || !stage || !device_ms || !host_ms)
    return HATA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t esz = dims->dtype == HATA_BF16 ? 2 : 4;
  const size_t row = (size_t)dims->head_dim * esz;
  const size_t q_bytes = (size_t)dims->batch * dims->n_q_heads * row;
  const size_t kv_half = (size_t)dims->batch * dims->n_kv_heads * row;
  const size_t in_bytes = q_bytes + 2 * kv_half;
  void* out_dev = nullptr;
  if (cudaHostGetDevicePointer(&out_dev, out_host, 0) != cudaSuccess) {
    (void)cudaGetLastError();
    return HATA_ERR_CUDA;
  }
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return HATA_ERR_CUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return HATA_ERR_CUDA;
  }
  int status = HATA_OK;
  const auto t0 = std::chrono::steady_clock::now();
  cudaEventRecord(e0, st);
  for (int i = 0; i < steps && status == HATA_OK; ++i) {
    const int l = i % R;
    char* sg = static_cast<char*>(stage[l]);
    if (cudaMemcpyAsync(sg, in_host, in_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
      status = HATA_ERR_CUDA;
      break;
    }
    status = hata_append_kv(dims, sg + q_bytes, sg + q_bytes + kv_half, K[l], V[l], lens[l], stream);
    if (status != HATA_OK) break;
    status = hata_decode_step(dims, sg, K[l], V[l], W[l], codes[l], lens[l], k, 0.f, out_dev, nullptr, nullptr, ws,
                              ws_bytes, stream);
    if (status != HATA_OK) break;
    if (cudaStreamSynchronize(st) != cudaSuccess) status = HATA_ERR_CUDA;
  }
  cudaEventRecord(e1, st);
  if (cudaEventSynchronize(e1) != cudaSuccess) status = HATA_ERR_CUDA;
  const auto t1 = std::chrono::steady_clock::now();
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  *device_ms = ms;
  *host_ms = std::chrono::duration<float, std::milli>(t1 - t0).count();
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return status;
}

}  // extern "C"
