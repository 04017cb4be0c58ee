// hata_topk_noalloc: the top-k select of hata_topk for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain scratch memory: code that a host engine
// runs with only its input and output buffers, code recorded into a CUDA graph
// where an allocation is not allowed, or latency-critical code where an
// allocation could block or synchronise the device.  This entry point takes the
// same inputs and outputs as hata_topk but keeps its scratch (per-chunk
// histograms, per-chunk offsets, thresholds, arrival counters and a status
// word) in one fixed array of device memory that belongs to the library.
//
// Facts a caller must know:
//   * the array holds kNoAllocScratchBytes (8 MiB) on every GPU that loads the
//     library, for the life of the process;
//   * problems whose scratch would not fit are rejected with
//     HATA_ERR_WORKSPACE before anything is launched;
//   * the first call on a device looks up the array's device address (with
//     that device current); make that first call before any stream capture;
//   * every call on a device shares the array: two calls whose work overlaps
//     on the GPU (different streams without ordering) corrupt each other;
//   * the counters that must start at zero are cleared by each call (an
//     enqueued memset), so a previous call that stopped early cannot leave
//     them dirty.
#include <mutex>

#include "hata_kernels.cuh"

namespace hata {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

// Scratch of hata_topk_noalloc.  In host code this name is only a handle for
// cudaGetSymbolAddress, never a device address.
static __device__ __align__(256) unsigned char g_topk_scratch[kNoAllocScratchBytes];

// Regions of the top-k scratch (the same regions hata_topk uses in a workspace).
WsLayout topk_layout(const hata_dims_t& d) {
  WsLayout L{};
  const size_t B = d.batch, Hkv = d.n_kv_heads, G = d.n_q_heads / d.n_kv_heads;
  L.nchunk = (int)((d.max_seq + kTopkChunk - 1) / kTopkChunk);
  L.nbins = (int)(G * d.hash_bits + 1);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.status = take(kAlign);
  L.topk_count = take(B * Hkv * 4);  // next to the status word: one memset clears both
  L.topk_hist = take(B * Hkv * (size_t)L.nchunk * L.nbins * 4);
  L.topk_chunk = take(B * Hkv * (size_t)L.nchunk * 2 * 4);
  L.topk_thr = take(B * Hkv * 2 * 4);
  L.total = off;
  return L;
}

// Device address of the scratch array for the current device, looked up once.
cudaError_t scratch_ptr(char** out) {
  static std::mutex mu;
  static char* ptrs[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = static_cast<char*>(p);
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace hata

using namespace hata;

extern "C" hata_status_t hata_topk_noalloc(const hata_dims_t* dims, const int32_t* scores, const int32_t* seq_lens,
                                           int k, int32_t* idx, int32_t* n_sel, void* stream) {
  const hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!scores || !seq_lens || !idx || k < 1) return HATA_ERR_INVALID_ARG;
  const WsLayout L = topk_layout(*dims);
  if (L.total > kNoAllocScratchBytes) return HATA_ERR_WORKSPACE;  // too large for the built-in scratch
  char* ws = nullptr;
  if (scratch_ptr(&ws) != cudaSuccess) return HATA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // status word and arrival counters start at zero
  if (cudaMemsetAsync(ws + L.status, 0, L.topk_hist - L.status, st) != cudaSuccess) return HATA_ERR_CUDA;
  if (launch_topk(*dims, L, scores, seq_lens, k, idx, n_sel, ws, st) != cudaSuccess) return HATA_ERR_CUDA;
  return HATA_OK;
}
