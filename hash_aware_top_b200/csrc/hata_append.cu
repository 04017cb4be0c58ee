// KV cache update of a decode step ("HATA" paper notes, Decode 阶段算法: the new
// token's key and value join the cache before the step scores it): the new rows
// K_new[b][g][:] and V_new[b][g][:] are written to slot L_b - 1 of their slabs.
// A plain row copy, one 16-byte vector per thread: both rows of a (b, g) pair are
// d * sizeof(T) bytes (256 or 512), so every vector is aligned when the bases are.
// The paged form writes the slot the block table gives (the layout of the paged step).
#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kAppThreads = 256;

// Paged form: the slot of logical token t of sequence b, KV head g is slot t mod bs of pool
// block block_table[b][t / bs] ([n_blocks][Hkv][bs] rows); a block number outside the pool
// is skipped (no write).
template <bool PAGED>
__global__ void __launch_bounds__(kAppThreads)
    append_kv_kernel(const uint4* __restrict__ new_k, const uint4* __restrict__ new_v, uint4* __restrict__ K,
                     uint4* __restrict__ V, const int32_t* __restrict__ seq_lens, int hkv, int max_seq,
                     int vec_per_row, long long n_vec, const int32_t* __restrict__ block_table, int block_shift,
                     int max_blocks, int n_blocks) {
  const long long e = (long long)blockIdx.x * kAppThreads + threadIdx.x;
  if (e >= n_vec) return;
  const long long half = n_vec / 2;  // vectors of all K rows, then of all V rows
  const bool is_v = e >= half;
  const long long ev = is_v ? e - half : e;
  const long long row = ev / vec_per_row;  // (b, g) pair
  const int c = (int)(ev % vec_per_row);
  const int b = (int)(row / hkv), g = (int)(row % hkv);
  const int L = seq_lens[b];
  if (L < 1 || L > max_seq) return;  // no slot to write
  size_t slot;
  if constexpr (PAGED) {
    const int t = L - 1;
    const int blk = block_table[(size_t)b * max_blocks + (t >> block_shift)];
    if (blk < 0 || blk >= n_blocks) return;
    slot = (((size_t)blk * hkv + g) << block_shift) + (size_t)(t & ((1 << block_shift) - 1));
  } else {
    slot = (size_t)row * max_seq + (L - 1);
  }
  const size_t dst = slot * vec_per_row + c;
  if (is_v) V[dst] = new_v[ev];
  else K[dst] = new_k[ev];
}

}  // namespace

cudaError_t launch_append_kv(const hata_dims_t& d, const void* new_k, const void* new_v, void* K, void* V,
                             const int32_t* seq_lens, const PagedCache* pg, cudaStream_t st) {
  const int esize = d.dtype == HATA_BF16 ? 2 : 4;
  const int vec_per_row = d.head_dim * esize / 16;
  const long long n_vec = 2LL * d.batch * d.n_kv_heads * vec_per_row;
  const long long blocks = (n_vec + kAppThreads - 1) / kAppThreads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const uint4 *nk = static_cast<const uint4*>(new_k), *nv = static_cast<const uint4*>(new_v);
  uint4 *Kc = static_cast<uint4*>(K), *Vc = static_cast<uint4*>(V);
  if (pg)
    append_kv_kernel<true><<<(unsigned)blocks, kAppThreads, 0, st>>>(nk, nv, Kc, Vc, seq_lens, d.n_kv_heads, d.max_seq,
                                                                     vec_per_row, n_vec, pg->block_table,
                                                                     pg->block_shift, pg->max_blocks, pg->n_blocks);
  else
    append_kv_kernel<false><<<(unsigned)blocks, kAppThreads, 0, st>>>(nk, nv, Kc, Vc, seq_lens, d.n_kv_heads,
                                                                      d.max_seq, vec_per_row, n_vec, nullptr, 0, 0, 0);
  return cudaGetLastError();
}

}  // namespace hata
