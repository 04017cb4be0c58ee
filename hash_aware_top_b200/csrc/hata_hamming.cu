// Hamming scan with the GQA sum ("HATA" paper notes, Decode 阶段算法: Hamming
// distance bitcount(xor(Q_H, K_H_cache)), scores of query heads sharing a KV
// cache aggregated; 硬件高效优化: XOR + popc with coalesced access).
//
// Each thread scores one token per step; a warp reads 32 consecutive codes
// (32 * r/8 contiguous bytes, one 128-bit load per lane for r = 128), and every
// thread keeps 8 tokens' loads in flight before computing.  The query side of a
// group is folded into per-word constants (hata_common.cuh, QuadWord) so that a
// G = 4 group costs 2 popc per code word instead of 4.
#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kHamThreads = 256;
constexpr int kHamTPT = 8;  // tokens per thread

// H16: 16-bit codes, one uint16 per token (the word holds it zero-extended, NW = 1)
template <int NW, int G, bool H16>
__global__ void __launch_bounds__(kHamThreads)
    hamming_kernel(const uint32_t* __restrict__ qcode, const uint32_t* __restrict__ codes,
                   const int32_t* __restrict__ seq_lens, int32_t* __restrict__ scores, int max_seq, int hkv,
                   int g_rt) {
  extern __shared__ uint32_t qs[];  // [G][NW]
  const int b = blockIdx.z, g = blockIdx.y;
  const int L = clamp_len(seq_lens, b, max_seq, nullptr);
  const int t0 = blockIdx.x * kHamThreads * kHamTPT;
  if (t0 >= L) return;
  const int Gn = G ? G : g_rt;
  const size_t q0 = ((size_t)b * hkv * Gn + (size_t)g * Gn) * NW;
  for (int e = threadIdx.x; e < Gn * NW; e += kHamThreads)
    qs[e] = H16 ? (uint32_t)reinterpret_cast<const uint16_t*>(qcode)[q0 + e] : qcode[q0 + e];
  __syncthreads();
  GroupQuery<NW, G> gq;
  gq.init(qs);

  const size_t slab = (size_t)b * hkv + g;
  const uint32_t* cb = codes + slab * max_seq * NW;
  const uint16_t* cb16 = reinterpret_cast<const uint16_t*>(codes) + slab * max_seq;
  int32_t* out = scores + slab * max_seq;
  uint32_t kw[kHamTPT][NW];
#pragma unroll
  for (int u = 0; u < kHamTPT; ++u) {
    const int t = t0 + u * kHamThreads + threadIdx.x;
    if (t < L) {
      if constexpr (H16) kw[u][0] = (uint32_t)__ldg(cb16 + t);
      else load_code<NW>(cb + (size_t)t * NW, kw[u]);
    }
  }
#pragma unroll
  for (int u = 0; u < kHamTPT; ++u) {
    const int t = t0 + u * kHamThreads + threadIdx.x;
    if (t < L) out[t] = gq.score(kw[u], qs, Gn);
  }
}

template <int NW, bool H16 = false>
cudaError_t launch_nw(const hata_dims_t& d, const uint32_t* qcode, const uint32_t* codes, const int32_t* seq_lens,
                      int32_t* scores, cudaStream_t st) {
  const int G = d.n_q_heads / d.n_kv_heads;
  dim3 grid((d.max_seq + kHamThreads * kHamTPT - 1) / (kHamThreads * kHamTPT), d.n_kv_heads, d.batch);
  const size_t smem = (size_t)G * NW * 4;
  switch (G) {
    case 1: hamming_kernel<NW, 1, H16><<<grid, kHamThreads, smem, st>>>(qcode, codes, seq_lens, scores, d.max_seq, d.n_kv_heads, G); break;
    case 2: hamming_kernel<NW, 2, H16><<<grid, kHamThreads, smem, st>>>(qcode, codes, seq_lens, scores, d.max_seq, d.n_kv_heads, G); break;
    case 4: hamming_kernel<NW, 4, H16><<<grid, kHamThreads, smem, st>>>(qcode, codes, seq_lens, scores, d.max_seq, d.n_kv_heads, G); break;
    case 8: hamming_kernel<NW, 8, H16><<<grid, kHamThreads, smem, st>>>(qcode, codes, seq_lens, scores, d.max_seq, d.n_kv_heads, G); break;
    default: hamming_kernel<NW, 0, H16><<<grid, kHamThreads, smem, st>>>(qcode, codes, seq_lens, scores, d.max_seq, d.n_kv_heads, G); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_hamming(const hata_dims_t& d, const uint32_t* qcode, const uint32_t* codes,
                           const int32_t* seq_lens, int32_t* scores, cudaStream_t stream) {
  switch (d.hash_bits) {
    case 16: return launch_nw<1, true>(d, qcode, codes, seq_lens, scores, stream);
    case 32: return launch_nw<1>(d, qcode, codes, seq_lens, scores, stream);
    case 64: return launch_nw<2>(d, qcode, codes, seq_lens, scores, stream);
    case 128: return launch_nw<4>(d, qcode, codes, seq_lens, scores, stream);
    case 256: return launch_nw<8>(d, qcode, codes, seq_lens, scores, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hata
