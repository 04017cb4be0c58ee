// extern "C" entry points of libhata: argument validation, workspace carving,
// launches.  Nothing here allocates device memory or synchronises (except
// hata_read_device_status).
#include <algorithm>
#include <cmath>
#include <cstdio>

#include "hata_kernels.cuh"

using namespace hata;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hata_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HATA_OK;
  return HATA_ERR_CUDA;
}

WsLayout layout_for(const hata_dims_t& d, int k) {
  return make_layout(d, k, std::max(fused_step_ws_bytes(d, k), split_step_ws_bytes(d, k)));
}

// The fused form of a decode step (both give the same results).  Measured on B200 at
// the benchmark workloads: the single-launch cluster form is faster while the units
// are few (8 units at 32K-128K, one unit, 32 units of r = 32 codes), the all-SM form
// with many units (128 ragged units) and on a paged cache (its per-segment copies are
// issued from several lanes at once).
bool use_all_sm(const hata_dims_t& d, int k, bool paged) {
  if (!split_step_applies(d, k)) return false;
  if (d.flags & (HATA_FLAG_ALL_SM_SCAN | HATA_FLAG_TEST_EXPIRE_WAIT)) return true;
  // Measured on B200: the cluster form wins while units are few and each selects little (8
  // units of k = 512: 18.9 against 19.5 us); the all-SM form from 64 units, and from 32 units
  // when the selection is large (32 units of k = 2048: 44.4 against 47.8 us), where its tail
  // runs the attention on tensor-core tiles.
  const long long units = (long long)d.batch * d.n_kv_heads;
  const long long rows = units * std::min<long long>(k, d.max_seq);
  return paged || units >= 64 || (units >= 32 && rows >= 32768) || !fused_step_applies(d, k);
}

hata_status_t check_ws(const hata_dims_t& d, int k, const void* ws, size_t bytes, WsLayout* L) {
  *L = layout_for(d, k);
  if (!ws || !aligned16(ws)) return HATA_ERR_WORKSPACE;
  if (bytes < L->total) return HATA_ERR_WORKSPACE;
  return HATA_OK;
}

}  // namespace

extern "C" {

int hata_version(void) { return 100; }

const char* hata_status_string(hata_status_t s) {
  switch (s) {
    case HATA_OK: return "ok";
    case HATA_ERR_INVALID_ARG: return "invalid argument";
    case HATA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case HATA_ERR_CUDA: return "CUDA error";
    case HATA_ERR_TIMEOUT: return "device-side wait timed out";
    case HATA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

hata_status_t hata_workspace_size(const hata_dims_t* dims, int k, size_t* bytes) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (k < 1 || !bytes) return HATA_ERR_INVALID_ARG;
  *bytes = layout_for(*dims, k).total;
  return HATA_OK;
}

hata_status_t hata_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || bytes == 0) return HATA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_encode_append(const hata_dims_t* dims, const void* x, int x_heads, int x_len, int n_tok,
                                 const int32_t* seq_end, const float* W_H, uint32_t* codes, int codes_len,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!x || !W_H || !codes || !aligned16(x) || !aligned16(W_H) || !aligned16(codes)) return HATA_ERR_INVALID_ARG;
  if (x_heads < 1 || x_heads % dims->n_kv_heads || x_len < 1 || codes_len < 1 || n_tok < 0)
    return HATA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < kStatusBytes) return HATA_ERR_WORKSPACE;
  if (n_tok == 0) return HATA_OK;
  return cuda_status(launch_encode(*dims, x, x_heads, x_len, n_tok, seq_end, W_H, codes, codes_len,
                                   static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_prefill_workspace_size(const hata_dims_t* dims, size_t* bytes) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!bytes) return HATA_ERR_INVALID_ARG;
  *bytes = prefill_ws_bytes(*dims);
  return HATA_OK;
}

hata_status_t hata_prefill_attention(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                     const float* W_H, void* codes, const int32_t* seq_lens, float scale, void* out,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  const hata_dims_t& d = *dims;
  if (d.dtype != HATA_BF16) return HATA_ERR_UNSUPPORTED;
  if (codes && d.hash_bits > 128) return HATA_ERR_UNSUPPORTED;
  if (!q || !K || !V || !seq_lens || !out || (codes && !W_H)) return HATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || (codes && !aligned16(codes)))
    return HATA_ERR_INVALID_ARG;
  if (!(scale >= 0.f) || scale == INFINITY) return HATA_ERR_INVALID_ARG;
  if ((long long)d.batch * d.n_q_heads * d.max_seq + 128 > 0x7fffffffLL) return HATA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) || workspace_bytes < prefill_ws_bytes(d)) return HATA_ERR_WORKSPACE;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf((float)d.head_dim);
  cudaError_t e = launch_prefill(d, q, K, V, W_H, codes, seq_lens, sc, out, static_cast<char*>(workspace),
                                 static_cast<cudaStream_t>(stream));
  return e == cudaErrorNotSupported ? HATA_ERR_UNSUPPORTED : cuda_status(e);
}

hata_status_t hata_append_kv(const hata_dims_t* dims, const void* new_k, const void* new_v, void* K, void* V,
                             const int32_t* seq_lens, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!new_k || !new_v || !K || !V || !seq_lens) return HATA_ERR_INVALID_ARG;
  if (!aligned16(new_k) || !aligned16(new_v) || !aligned16(K) || !aligned16(V)) return HATA_ERR_INVALID_ARG;
  return cuda_status(
      launch_append_kv(*dims, new_k, new_v, K, V, seq_lens, nullptr, static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_append_kv_paged(const hata_dims_t* dims, const void* new_k, const void* new_v, void* K_pool,
                                   void* V_pool, const int32_t* block_table, int block_size, int n_blocks,
                                   const int32_t* seq_lens, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!new_k || !new_v || !K_pool || !V_pool || !block_table || !seq_lens) return HATA_ERR_INVALID_ARG;
  if (!aligned16(new_k) || !aligned16(new_v) || !aligned16(K_pool) || !aligned16(V_pool)) return HATA_ERR_INVALID_ARG;
  if (block_size < 16 || block_size > 65536 || (block_size & (block_size - 1)) || n_blocks < 1)
    return HATA_ERR_INVALID_ARG;
  PagedCache pg;
  pg.block_table = block_table;
  pg.block_shift = 0;
  while ((1 << pg.block_shift) < block_size) ++pg.block_shift;
  pg.n_blocks = n_blocks;
  pg.max_blocks = (dims->max_seq + block_size - 1) / block_size;
  return cuda_status(
      launch_append_kv(*dims, new_k, new_v, K_pool, V_pool, seq_lens, &pg, static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_hamming_scores(const hata_dims_t* dims, const uint32_t* qcode, const uint32_t* codes,
                                  const int32_t* seq_lens, int32_t* scores, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!qcode || !codes || !seq_lens || !scores || !aligned16(codes)) return HATA_ERR_INVALID_ARG;
  return cuda_status(launch_hamming(*dims, qcode, codes, seq_lens, scores, static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_topk(const hata_dims_t* dims, const int32_t* scores, const int32_t* seq_lens, int k,
                        int32_t* idx, int32_t* n_sel, void* workspace, size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!scores || !seq_lens || !idx || k < 1) return HATA_ERR_INVALID_ARG;
  WsLayout L;
  if ((s = check_ws(*dims, k, workspace, workspace_bytes, &L)) != HATA_OK) return s;
  return cuda_status(launch_topk(*dims, L, scores, seq_lens, k, idx, n_sel, static_cast<char*>(workspace),
                                 static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_sparse_decode(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                 const int32_t* idx, int k, float scale, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!q || !K || !V || !idx || !out || k < 1) return HATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return HATA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return HATA_ERR_INVALID_ARG;
  WsLayout L;
  if ((s = check_ws(*dims, k, workspace, workspace_bytes, &L)) != HATA_OK) return s;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)dims->head_dim);
  return cuda_status(launch_sparse_decode(*dims, L, q, K, V, idx, k, scale, out, static_cast<char*>(workspace),
                                          static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_dense_workspace_size(const hata_dims_t* dims, size_t* bytes) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!bytes) return HATA_ERR_INVALID_ARG;
  *bytes = dense_ws_bytes(*dims);
  return HATA_OK;
}

hata_status_t hata_dense_decode(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                const int32_t* seq_lens, float scale, void* out, void* workspace,
                                size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (dims->dtype != HATA_BF16 || dims->n_q_heads / dims->n_kv_heads > 8) return HATA_ERR_UNSUPPORTED;
  if (!q || !K || !V || !out) return HATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return HATA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return HATA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < dense_ws_bytes(*dims)) return HATA_ERR_WORKSPACE;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)dims->head_dim);
  return cuda_status(launch_dense_decode(*dims, q, K, V, seq_lens, scale, out, static_cast<char*>(workspace),
                                         static_cast<cudaStream_t>(stream)));
}

hata_status_t hata_decode_step_qk(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                  const float* W_q, const float* W_k, uint32_t* codes, const int32_t* seq_lens, int k,
                                  float scale, void* out, uint32_t* qcode_out, int32_t* idx_out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!q || !K || !V || !W_q || !W_k || !codes || !seq_lens || !out || k < 1) return HATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(W_q) || !aligned16(W_k) || !aligned16(codes) ||
      !aligned16(out))
    return HATA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return HATA_ERR_INVALID_ARG;
  WsLayout L;
  if ((s = check_ws(*dims, k, workspace, workspace_bytes, &L)) != HATA_OK) return s;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)dims->head_dim);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);

  cudaError_t e = cudaErrorNotSupported;
  if (use_all_sm(*dims, k, false))
    e = launch_split_step(*dims, L, q, K, V, W_q, W_k, codes, seq_lens, k, scale, out, qcode_out, idx_out, nullptr,
                          ws, st);
  else if (!(dims->flags & HATA_FLAG_TEST_EXPIRE_WAIT))  // the test hook exists in the all-SM form only
    e = launch_fused_step(*dims, L, q, K, V, W_q, W_k, codes, seq_lens, k, scale, out, qcode_out, idx_out, nullptr,
                          ws, st);
  if (e != cudaErrorNotSupported) return cuda_status(e);
  if (dims->flags & HATA_FLAG_TEST_EXPIRE_WAIT) return HATA_ERR_UNSUPPORTED;

  // Chain of the granular kernels (shapes the fused kernel does not cover).
  const hata_dims_t& d = *dims;
  uint32_t* qc = qcode_out ? qcode_out : reinterpret_cast<uint32_t*>(ws + L.qcode);
  int32_t* ix = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  int32_t* sc = reinterpret_cast<int32_t*>(ws + L.scores);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  if ((e = launch_encode(d, q, d.n_q_heads, 1, 1, nullptr, W_q, qc, 1, status, st)) != cudaSuccess)
    return cuda_status(e);
  if ((e = launch_encode(d, K, d.n_kv_heads, d.max_seq, 1, seq_lens, W_k, codes, d.max_seq, status, st)) !=
      cudaSuccess)
    return cuda_status(e);
  if ((e = launch_hamming(d, qc, codes, seq_lens, sc, st)) != cudaSuccess) return cuda_status(e);
  if ((e = launch_topk(d, L, sc, seq_lens, k, ix, nullptr, ws, st)) != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_sparse_decode(d, L, q, K, V, ix, k, scale, out, ws, st));
}

hata_status_t hata_decode_step(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                               const float* W_H, uint32_t* codes, const int32_t* seq_lens, int k, float scale,
                               void* out, uint32_t* qcode_out, int32_t* idx_out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return hata_decode_step_qk(dims, q, K, V, W_H, W_H, codes, seq_lens, k, scale, out, qcode_out, idx_out, workspace,
                             workspace_bytes, stream);
}

hata_status_t hata_decode_step_paged(const hata_dims_t* dims, const void* q, const void* K_pool, const void* V_pool,
                                     const float* W_q, const float* W_k, uint32_t* codes_pool,
                                     const int32_t* block_table, int block_size, int n_blocks,
                                     const int32_t* seq_lens, int k, float scale, void* out, uint32_t* qcode_out,
                                     int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream) {
  hata_status_t s = check_dims(dims);
  if (s != HATA_OK) return s;
  if (!q || !K_pool || !V_pool || !W_q || !W_k || !codes_pool || !block_table || !seq_lens || !out || k < 1)
    return HATA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(K_pool) || !aligned16(V_pool) || !aligned16(W_q) || !aligned16(W_k) ||
      !aligned16(codes_pool) || !aligned16(out))
    return HATA_ERR_INVALID_ARG;
  if (block_size < 16 || block_size > 65536 || (block_size & (block_size - 1)) || n_blocks < 1)
    return HATA_ERR_INVALID_ARG;
  if ((long long)n_blocks * dims->n_kv_heads * block_size > 0x7fffffffLL) return HATA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return HATA_ERR_INVALID_ARG;
  WsLayout L;
  if ((s = check_ws(*dims, k, workspace, workspace_bytes, &L)) != HATA_OK) return s;
  if (scale <= 0.f) scale = 1.0f / std::sqrt((float)dims->head_dim);
  PagedCache pg;
  pg.block_table = block_table;
  pg.block_shift = 0;
  while ((1 << pg.block_shift) < block_size) ++pg.block_shift;
  pg.n_blocks = n_blocks;
  pg.max_blocks = (dims->max_seq + block_size - 1) / block_size;
  cudaError_t e = cudaErrorNotSupported;
  if (use_all_sm(*dims, k, true))
    e = launch_split_step(*dims, L, q, K_pool, V_pool, W_q, W_k, codes_pool, seq_lens, k, scale, out, qcode_out,
                          idx_out, &pg, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream));
  if (e != cudaErrorNotSupported) return cuda_status(e);
  if (dims->flags & HATA_FLAG_TEST_EXPIRE_WAIT) return HATA_ERR_UNSUPPORTED;
  e = launch_fused_step(*dims, L, q, K_pool, V_pool, W_q, W_k, codes_pool, seq_lens, k, scale, out, qcode_out, idx_out,
                        &pg, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream));
  return e == cudaErrorNotSupported ? HATA_ERR_UNSUPPORTED : cuda_status(e);
}

int hata_decode_step_kernel_count(const hata_dims_t* dims, int k) {
  if (check_dims(dims) != HATA_OK || k < 1) return -1;
  if (use_all_sm(*dims, k, false)) return 3;
  return fused_step_applies(*dims, k) ? 1 : 6;
}

hata_status_t hata_read_device_status(void* workspace, void* stream, int* device_status) {
  if (!workspace || !device_status) return HATA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return HATA_ERR_CUDA;
  *device_status = (int)v;
  return HATA_OK;
}

}  // extern "C"
