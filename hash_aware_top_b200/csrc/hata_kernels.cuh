// Internal launchers of libhata's kernels (host side).  Arguments are already
// validated by hata_api.cu; every launcher returns cudaGetLastError().
#pragma once

#include "hata_common.cuh"

namespace hata {

// status: the caller's device status word (a bounded wait that runs out is recorded there)
cudaError_t launch_encode(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                          const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len, uint32_t* status,
                          cudaStream_t stream);

size_t prefill_ws_bytes(const hata_dims_t& d);
cudaError_t launch_prefill(const hata_dims_t& d, const void* q, const void* K, const void* V, const float* W,
                           void* codes, const int32_t* seq_lens, float scale, void* out, char* ws,
                           cudaStream_t stream);
cudaError_t launch_hamming(const hata_dims_t& d, const uint32_t* qcode, const uint32_t* codes,
                           const int32_t* seq_lens, int32_t* scores, cudaStream_t stream);

cudaError_t launch_topk(const hata_dims_t& d, const WsLayout& L, const int32_t* scores, const int32_t* seq_lens,
                        int k, int32_t* idx, int32_t* n_sel, char* ws, cudaStream_t stream);

cudaError_t launch_sparse_decode(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K,
                                 const void* V, const int32_t* idx, int k, float scale, void* out, char* ws,
                                 cudaStream_t stream);

// Whether the fused decode-step kernel covers these dims and budget.
bool fused_step_applies(const hata_dims_t& d, int k);
// Fused decode step: bytes of workspace its plan needs (0 if it does not apply)
size_t fused_step_ws_bytes(const hata_dims_t& d, int k);
cudaError_t launch_encode_mma(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                              const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len,
                              cudaStream_t stream);
// Prefill encode on tcgen05 tensor cores (bf16 keys, r <= 128; else cudaErrorNotSupported).
cudaError_t launch_encode_tc(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                             const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len,
                             uint32_t* status, cudaStream_t stream);
size_t dense_ws_bytes(const hata_dims_t& d);
cudaError_t launch_dense_decode(const hata_dims_t& d, const void* q, const void* K, const void* V,
                                const int32_t* seq_lens, float scale, void* out, char* ws, cudaStream_t stream);
// Returns cudaErrorNotSupported when the fused kernel does not apply to these dims.
// Paged cache: K, V and codes are pools [n_blocks][Hkv][1 << block_shift][...] and
// block_table [B][max_blocks] maps each sequence's logical blocks to pool blocks.
struct PagedCache {
  const int32_t* block_table;
  int block_shift, n_blocks, max_blocks;
};

// pg: paged pools (the layout of the paged step), or null for [B][Hkv][max_seq][d] caches
cudaError_t launch_append_kv(const hata_dims_t& d, const void* new_k, const void* new_v, void* K, void* V,
                             const int32_t* seq_lens, const PagedCache* pg, cudaStream_t stream);

// Wk: separate key encoder, or equal to W (one encoder for queries and keys).
// pg: paged cache, or null for [B][Hkv][max_seq][...] slabs.
cudaError_t launch_fused_step(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K,
                              const void* V, const float* W, const float* Wk, uint32_t* codes,
                              const int32_t* seq_lens, int k, float scale, void* out, uint32_t* qcode_out,
                              int32_t* idx_out, const PagedCache* pg, char* ws, cudaStream_t stream);

// Decode step as a scan kernel over all SMs plus a per-unit tail kernel (hata_fused.cu).
bool split_step_applies(const hata_dims_t& d, int k);
size_t split_step_ws_bytes(const hata_dims_t& d, int k);
cudaError_t launch_split_step(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K,
                              const void* V, const float* W, const float* Wk, uint32_t* codes,
                              const int32_t* seq_lens, int k, float scale, void* out, uint32_t* qcode_out,
                              int32_t* idx_out, const PagedCache* pg, char* ws, cudaStream_t stream);

}  // namespace hata
