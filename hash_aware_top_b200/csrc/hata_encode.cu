// HashEncode + cache update: y = x . W_H (fp32), bit = [y > 0], LSB-first pack,
// written straight into the code cache ("HATA" paper notes, 硬件高效优化:
// projection -> sign -> bitpack -> cache update fused in one kernel).
//
// Three forms, chosen by the number of tokens per sequence and the key type:
//   * decode form (n_tok <= kDecodeTok): the few rows of a call (G query heads,
//     or one new key per KV head) are latency-bound, so the work is spread over
//     one CTA per (32-column word, KV group, batch).  Each CTA stages its rows
//     and its 32 columns of W_H (transposed) in shared memory and every (row,
//     column) projection is one warp_dot128 -- the same arithmetic as the fused
//     decode step, so both paths produce identical codes.
//   * prefill form, bf16 keys and r <= 128: the tcgen05 tensor-core kernel of
//     hata_encode_tc.cu (W_H split in three bf16 parts, fp32 accumulation), or
//     the mma.sync kernel of hata_encode_mma.cu when no TMA tensor map can be made;
//   * prefill form otherwise: each CTA owns one (batch, KV group) and a tile of 32 rows;
//     thread (slice s, column j) accumulates y_j for rows s, s + NS, ... with
//     fp32 FMAs in ascending i, reading W_H[g][i][j] coalesced along j; the sign
//     bits of 32 consecutive columns are one warp ballot, i.e. one packed word.
// The forms round differently, so a key encoded by two of them can differ only in
// bits whose projection is within fp32 rounding of zero.
#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kEncThreads = 256;
constexpr int kEncRows = 32;
constexpr int kDecodeTok = 4;     // decode form up to this many tokens per sequence
constexpr int kDecRows = 16;      // rows per decode-form CTA

template <typename T>
__global__ void __launch_bounds__(kEncThreads)
    encode_decode_kernel(const T* __restrict__ x, int x_heads, int x_len, int n_tok,
                         const int32_t* __restrict__ seq_end, const float* __restrict__ W,
                         uint32_t* __restrict__ codes, int codes_len, int hpg, int R) {
  constexpr int D = kHeadDim;
  __shared__ float xs[kDecRows][D];
  __shared__ float ws[32][D];
  __shared__ uint32_t words[kDecRows];
  const int w = blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nbz = (hpg * n_tok + kDecRows - 1) / kDecRows;
  const int bb = b / nbz, row0 = (b % nbz) * kDecRows;
  const int rows_total = hpg * n_tok;
  const int end = seq_end ? seq_end[bb] : x_len;
  const int t_lo = end - n_tok;
  const int lim = min(x_len, codes_len);
  for (int e = tid; e < kDecRows * D; e += kEncThreads) {
    const int rr = e / D, i = e % D, rho = row0 + rr;
    float v = 0.f;
    if (rho < rows_total) {
      const int h = g * hpg + rho / n_tok, t = t_lo + rho % n_tok;
      if (t >= 0 && t < lim) v = to_f32(x[(((size_t)bb * x_heads + h) * x_len + t) * D + i]);
    }
    xs[rr][i] = v;
  }
  const int CW = R < 32 ? R : 32;  // columns of this code word (16 for 16-bit codes)
  const float* Wg = W + (size_t)g * D * R + 32 * w;
  for (int e = tid; e < 32 * D; e += kEncThreads) {
    const int i = e / 32, c = e % 32;
    ws[c][i] = c < CW ? __ldg(Wg + (size_t)i * R + c) : 0.f;
  }
  if (tid < kDecRows) words[tid] = 0u;
  __syncthreads();
  const int nrows = min(kDecRows, rows_total - row0);
  for (int pr = warp; pr < nrows * CW; pr += kEncThreads / 32) {
    const int rr = pr / CW, c = pr % CW;
    const float y = warp_dot128(xs[rr], ws[c], lane);
    if (lane == 0 && y > 0.f) atomicOr(&words[rr], 1u << c);
  }
  __syncthreads();
  if (tid < nrows) {
    const int rho = row0 + tid;
    const int h = g * hpg + rho / n_tok, t = t_lo + rho % n_tok;
    const size_t slot = ((size_t)bb * x_heads + h) * codes_len + t;
    if (t >= 0 && t < lim) {
      if (R == 16) reinterpret_cast<uint16_t*>(codes)[slot] = (uint16_t)words[tid];
      else codes[slot * (R / 32) + w] = words[tid];
    }
  }
}

template <typename T, int R>
__global__ void __launch_bounds__(kEncThreads)
    encode_kernel(const T* __restrict__ x, int x_heads, int x_len, int n_tok, const int32_t* __restrict__ seq_end,
                  const float* __restrict__ W, uint32_t* __restrict__ codes, int codes_len, int hpg) {
  constexpr int D = kHeadDim;
  constexpr int NS = kEncThreads / R;  // row slices
  constexpr int RPT = kEncRows / NS;   // rows per thread
  constexpr int NW = R / 32;
  __shared__ float xs[kEncRows][D];

  const int b = blockIdx.z, g = blockIdx.y;
  const int rows_total = hpg * n_tok;
  const int row0 = blockIdx.x * kEncRows;
  const int end = seq_end ? seq_end[b] : x_len;
  const int t_lo = end - n_tok;
  const int lim = min(x_len, codes_len);

  for (int e = threadIdx.x; e < kEncRows * D; e += kEncThreads) {
    const int rr = e / D, i = e % D, rho = row0 + rr;
    float v = 0.f;
    if (rho < rows_total) {
      const int h = g * hpg + rho / n_tok, t = t_lo + rho % n_tok;
      if (t >= 0 && t < lim) v = to_f32(x[(((size_t)b * x_heads + h) * x_len + t) * D + i]);
    }
    xs[rr][i] = v;
  }
  __syncthreads();

  const int j = threadIdx.x % R, s = threadIdx.x / R;
  float acc[RPT];
#pragma unroll
  for (int q = 0; q < RPT; ++q) acc[q] = 0.f;
  const float* Wg = W + (size_t)g * D * R + j;
#pragma unroll 4
  for (int i = 0; i < D; ++i) {
    const float w = __ldg(Wg + (size_t)i * R);
#pragma unroll
    for (int q = 0; q < RPT; ++q) acc[q] = fmaf(xs[s + q * NS][i], w, acc[q]);
  }

  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int q = 0; q < RPT; ++q) {
    const unsigned word = __ballot_sync(0xffffffffu, acc[q] > 0.f);
    const int rho = row0 + s + q * NS;
    // 16-bit codes: a warp holds two rows' codes, lanes 0 and 16 each write one half
    if ((R == 16 ? (lane & 15) : lane) == 0 && rho < rows_total) {
      const int h = g * hpg + rho / n_tok, t = t_lo + rho % n_tok;
      const size_t slot = ((size_t)b * x_heads + h) * codes_len + t;
      if (t >= 0 && t < lim) {
        if constexpr (R == 16) reinterpret_cast<uint16_t*>(codes)[slot] = (uint16_t)(word >> (lane & 16));
        else codes[slot * NW + j / 32] = word;
      }
    }
  }
}

template <typename T>
cudaError_t launch_t(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok, const int32_t* seq_end,
                     const float* W, uint32_t* codes, int codes_len, uint32_t* status, cudaStream_t st) {
  const int hpg = x_heads / d.n_kv_heads;
  if (n_tok <= kDecodeTok) {
    const int nbz = (hpg * n_tok + kDecRows - 1) / kDecRows;
    dim3 grid((d.hash_bits + 31) / 32, d.n_kv_heads, d.batch * nbz);
    encode_decode_kernel<T><<<grid, kEncThreads, 0, st>>>(static_cast<const T*>(x), x_heads, x_len, n_tok, seq_end,
                                                          W, codes, codes_len, hpg, d.hash_bits);
    return cudaGetLastError();
  }
  if constexpr (sizeof(T) == 2) {  // bf16 keys: tensor-core prefill (r <= 128), tcgen05 first, then mma.sync
    cudaError_t e = launch_encode_tc(d, x, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, status, st);
    if (e == cudaErrorNotSupported) e = launch_encode_mma(d, x, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, st);
    if (e != cudaErrorNotSupported) return e;
  }
  const long long rows = (long long)hpg * n_tok;
  dim3 grid((unsigned)((rows + kEncRows - 1) / kEncRows), d.n_kv_heads, d.batch);
  const T* xp = static_cast<const T*>(x);
  switch (d.hash_bits) {
    case 16: encode_kernel<T, 16><<<grid, kEncThreads, 0, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 32: encode_kernel<T, 32><<<grid, kEncThreads, 0, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 64: encode_kernel<T, 64><<<grid, kEncThreads, 0, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 128: encode_kernel<T, 128><<<grid, kEncThreads, 0, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 256: encode_kernel<T, 256><<<grid, kEncThreads, 0, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                          const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len, uint32_t* status,
                          cudaStream_t stream) {
  if (d.dtype == HATA_BF16)
    return launch_t<__nv_bfloat16>(d, x, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, status, stream);
  return launch_t<float>(d, x, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, status, stream);
}

}  // namespace hata
