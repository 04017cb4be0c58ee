// Shared device helpers and the workspace layout of libhata (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "hata.h"

namespace hata {

constexpr int kHeadDim = 128;        // d supported by this version
constexpr int kTopkChunk = 4096;     // tokens per top-k chunk in the granular path
constexpr int kSparseRows = 32;      // gathered rows per CTA in the granular sparse decode
constexpr int kMaxBins = 8193;       // G * r + 1 histogram bins supported
constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 16;  // smallest buffer that can hold a device status word

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Validation of the problem shape shared by every entry point (host side).
inline hata_status_t check_dims(const hata_dims_t* d) {
  if (!d) return HATA_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1 || d->max_seq < 1 || d->head_dim < 1 ||
      d->hash_bits < 1)
    return HATA_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads) return HATA_ERR_INVALID_ARG;
  if (d->dtype != HATA_F32 && d->dtype != HATA_BF16) return HATA_ERR_INVALID_ARG;
  if (d->flags & ~(HATA_FLAG_EARLY_PREFETCH | HATA_FLAG_TEST_EXPIRE_WAIT | HATA_FLAG_ALL_SM_SCAN))
    return HATA_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return HATA_ERR_UNSUPPORTED;
  if (d->hash_bits != 16 && d->hash_bits != 32 && d->hash_bits != 64 && d->hash_bits != 128 && d->hash_bits != 256)
    return HATA_ERR_UNSUPPORTED;
  if (d->hash_bits == 16 && (d->max_seq & 1)) return HATA_ERR_INVALID_ARG;  // 16-bit codes: whole 32-bit pairs
  const long long G = d->n_q_heads / d->n_kv_heads;
  if (G > 16 || G * d->hash_bits + 1 > kMaxBins) return HATA_ERR_UNSUPPORTED;
  return HATA_OK;
}

// Workspace regions (byte offsets).  One layout serves every call for given dims and k.
struct WsLayout {
  size_t status;         // uint32 device status word (+ padding)
  size_t qcode;          // [B][Hq][W] uint32 (decode step without qcode_out)
  size_t scores;         // [B][Hkv][Lmax] int32 (decode step chain)
  size_t idx;            // [B][Hkv][k] int32 (decode step without idx_out)
  size_t topk_hist;      // [B][Hkv][nchunk][nbins] int32
  size_t topk_chunk;     // [B][Hkv][nchunk][2] int32: selected-before, ties-before
  size_t topk_thr;       // [B][Hkv][2] int32: threshold T, tie quota m
  size_t topk_count;     // [B][Hkv] uint32 arrival counters
  size_t sp_part;        // [B][Hkv][nsplit][G][d + 2] float partials (m, l, o)
  size_t sp_count;       // [B][Hkv] uint32 arrival counters
  size_t fused;          // fused decode-step region
  size_t fused_bytes;
  size_t total;
  int nchunk, nbins, nsplit;
};

struct FusedPlan;  // defined in hata_step.cu

inline WsLayout make_layout(const hata_dims_t& d, int k, size_t fused_bytes) {
  WsLayout L{};
  const size_t B = d.batch, Hq = d.n_q_heads, Hkv = d.n_kv_heads, Lm = d.max_seq;
  const size_t CB = (size_t)d.hash_bits / 8, G = Hq / Hkv;  // bytes per code
  L.nchunk = (int)((Lm + kTopkChunk - 1) / kTopkChunk);
  L.nbins = (int)(G * d.hash_bits + 1);
  L.nsplit = (k + kSparseRows - 1) / kSparseRows;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.status = take(kAlign);
  L.qcode = take(B * Hq * CB);
  L.scores = take(B * Hkv * Lm * 4);
  L.idx = take(B * Hkv * (size_t)k * 4);
  L.topk_hist = take(B * Hkv * (size_t)L.nchunk * L.nbins * 4);
  L.topk_chunk = take(B * Hkv * (size_t)L.nchunk * 2 * 4);
  L.topk_thr = take(B * Hkv * 2 * 4);
  L.topk_count = take(B * Hkv * 4);
  L.sp_part = take(B * Hkv * (size_t)L.nsplit * G * (kHeadDim + 2) * 4);
  L.sp_count = take(B * Hkv * 4);
  L.fused = take(fused_bytes);
  L.fused_bytes = fused_bytes;
  L.total = off;
  return L;
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t code) {
  if (status) atomicCAS(status, 0u, code);
}

__device__ __forceinline__ int clamp_len(const int32_t* seq_lens, int b, int max_seq, uint32_t* status) {
  int L = seq_lens ? seq_lens[b] : max_seq;
  if (L > max_seq) {
    set_status(status, HATA_ERR_INVALID_ARG);
    L = max_seq;
  }
  return L < 0 ? 0 : L;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Sum of the G per-head Hamming distances for one 32-bit word of a key code.
// Heads are taken four at a time: with a_h = q_h ^ k, the three-way sum
// a0 + a1 + a2 = xor3 + 2 * maj3, and both xor3 and maj3 of (q_h ^ k) equal the
// same function of the q_h, xor'ed with k (they are self-dual).  Adding a3:
//   a0 + a1 + a2 + a3 = popc(Q ^ q3) + 2 popc(M ^ k) + 2 popc((Q ^ k) & (q3 ^ k))
// with Q = q0 ^ q1 ^ q2 and M = maj(q0, q1, q2) precomputed per query group.
// The first term does not depend on k and is added once per token.  This halves
// the popc count of the plain sum for G = 4.
struct QuadWord {
  uint32_t Q, M, q3;
};

__device__ __forceinline__ QuadWord make_quad(uint32_t q0, uint32_t q1, uint32_t q2, uint32_t q3) {
  QuadWord w;
  w.Q = q0 ^ q1 ^ q2;
  w.M = (q0 & q1) | (q0 & q2) | (q1 & q2);
  w.q3 = q3;
  return w;
}

__device__ __forceinline__ int quad_word_var(const QuadWord& w, uint32_t k) {
  return 2 * (__popc(w.M ^ k) + __popc((w.Q ^ k) & (w.q3 ^ k)));
}

__device__ __forceinline__ int quad_word_const(const QuadWord& w) { return __popc(w.Q ^ w.q3); }

template <int NW>
__device__ __forceinline__ void load_code(const uint32_t* p, uint32_t (&w)[NW]) {
  if constexpr (NW == 1) {
    w[0] = __ldg(p);
  } else if constexpr (NW == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < NW / 4; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
}

// Sum of popcounts of N words.  Groups of three words go through a carry-save
// adder first (x0 + x1 + x2 = xor3 + 2 * maj3, two LOP3 each), which trades
// one popc (16 per clock per SM) for two logic ops (64 per clock per SM); three
// adders per eight words balance the two pipes.
template <int N>
__device__ __forceinline__ int popc_sum(const uint32_t (&x)[N]) {
  if constexpr (N == 1) {
    return __popc(x[0]);
  } else if constexpr (N == 2) {
    return __popc(x[0]) + __popc(x[1]);
  } else if constexpr (N == 4) {
    const uint32_t s = x[0] ^ x[1] ^ x[2], c = (x[0] & x[1]) | (x[2] & (x[0] ^ x[1]));
    return __popc(s) + __popc(x[3]) + 2 * __popc(c);
  } else if constexpr (N == 8) {
    const uint32_t s1 = x[0] ^ x[1] ^ x[2], c1 = (x[0] & x[1]) | (x[2] & (x[0] ^ x[1]));
    const uint32_t s2 = x[3] ^ x[4] ^ x[5], c2 = (x[3] & x[4]) | (x[5] & (x[3] ^ x[4]));
    const uint32_t s3 = s1 ^ s2 ^ x[6], c3 = (s1 & s2) | (x[6] & (s1 ^ s2));
    return __popc(s3) + __popc(x[7]) + 2 * (__popc(c1) + __popc(c2) + __popc(c3));
  } else {
    static_assert(N % 8 == 0, "popc_sum: N must be 1, 2, 4 or a multiple of 8");
    int s = 0;
#pragma unroll
    for (int i = 0; i < N; i += 8) {
      const uint32_t y[8] = {x[i], x[i + 1], x[i + 2], x[i + 3], x[i + 4], x[i + 5], x[i + 6], x[i + 7]};
      s += popc_sum<8>(y);
    }
    return s;
  }
}

// Query-side state of one KV group for the per-token score D = sum_h popc(q_h ^ k).
//   G % 4 == 0 : G/4 quads, each 2 weight-2 words per code word (QuadWord)
//   G == 2     : popc(q0 ^ q1) + 2 popc((q0 ^ k) & (q1 ^ k))
//   G == 1     : popc(q0 ^ k)
//   G == 0     : runtime group size, plain sum over heads (codes in shared memory)
// The per-token words are summed with popc_sum (carry-save, see above).
template <int NW, int G>
struct GroupQuery {
  static constexpr int NQ = G >= 4 ? G / 4 : 1;
  QuadWord quad[NQ][NW];
  uint32_t a[NW], c[NW];
  int cst;

  __device__ __forceinline__ void init(const uint32_t* qg /* [G][NW] */) {
    cst = 0;
    if constexpr (G % 4 == 0 && G > 0) {
#pragma unroll
      for (int u = 0; u < NQ; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          quad[u][w] = make_quad(qg[(4 * u) * NW + w], qg[(4 * u + 1) * NW + w], qg[(4 * u + 2) * NW + w],
                                 qg[(4 * u + 3) * NW + w]);
          cst += quad_word_const(quad[u][w]);
        }
    } else if constexpr (G == 2) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        a[w] = qg[w];
        c[w] = qg[NW + w];
        cst += __popc(a[w] ^ c[w]);
      }
    } else if constexpr (G == 1) {
#pragma unroll
      for (int w = 0; w < NW; ++w) a[w] = qg[w];
    }
  }

  __device__ __forceinline__ int score(const uint32_t (&k)[NW], const uint32_t* qg, int g_rt) const {
    if constexpr (G % 4 == 0 && G > 0) {
      uint32_t x[2 * NQ * NW];
#pragma unroll
      for (int u = 0; u < NQ; ++u)
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          x[2 * (u * NW + w)] = quad[u][w].M ^ k[w];
          x[2 * (u * NW + w) + 1] = (quad[u][w].Q ^ k[w]) & (quad[u][w].q3 ^ k[w]);
        }
      return cst + 2 * popc_sum<2 * NQ * NW>(x);
    } else if constexpr (G == 2) {
      uint32_t x[NW];
#pragma unroll
      for (int w = 0; w < NW; ++w) x[w] = (a[w] ^ k[w]) & (c[w] ^ k[w]);
      return cst + 2 * popc_sum<NW>(x);
    } else if constexpr (G == 1) {
      uint32_t x[NW];
#pragma unroll
      for (int w = 0; w < NW; ++w) x[w] = a[w] ^ k[w];
      return popc_sum<NW>(x);
    } else {
      int s = 0;
      for (int h = 0; h < g_rt; ++h)
#pragma unroll
        for (int w = 0; w < NW; ++w) s += __popc(qg[h * NW + w] ^ k[w]);
      return s;
    }
  }
};

// y = sum_{i < 128} x[i] * w[i] computed by one warp in a fixed order: lane l
// accumulates x[l + 32u] * w[l + 32u] for u = 0..3 with fp32 FMAs (u
// ascending, starting from the u = 0 product), then the 32 partial sums are
// combined by a xor butterfly over offsets 16, 8, 4, 2, 1 (every lane ends with
// the same value, since each step adds two equal operand pairs).  Every kernel
// that encodes a decode-time vector uses this function, so query and key codes
// are bit-identical across the granular and the fused paths.
__device__ __forceinline__ float warp_dot128(const float* x, const float* w, int lane) {
  float p = x[lane] * w[lane];
  p = fmaf(x[lane + 32], w[lane + 32], p);
  p = fmaf(x[lane + 64], w[lane + 64], p);
  p = fmaf(x[lane + 96], w[lane + 96], p);
#pragma unroll
  for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
  return p;
}

// warp_dot128 for N (x, w) pairs at once: the same operations per pair, in
// the same order, interleaved so that the shuffle chains overlap.
template <int N>
__device__ __forceinline__ void warp_dot128_multi(const float* const (&x)[N], const float* const (&w)[N], int lane,
                                                  float (&y)[N]) {
#pragma unroll
  for (int j = 0; j < N; ++j) {
    float p = x[j][lane] * w[j][lane];
    p = fmaf(x[j][lane + 32], w[j][lane + 32], p);
    p = fmaf(x[j][lane + 64], w[j][lane + 64], p);
    p = fmaf(x[j][lane + 96], w[j][lane + 96], p);
    y[j] = p;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int j = 0; j < N; ++j) y[j] += __shfl_xor_sync(0xffffffffu, y[j], o);
}

// Block-wide exclusive prefix sum over NT threads (NT a multiple of 32).
// `warp_sums` is shared scratch of NT / 32 ints.  Returns this thread's
// exclusive prefix and writes the block total to *total.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) warp_sums[lane] = w;  // inclusive warp prefix
  }
  __syncthreads();
  const int before = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[NT / 32 - 1];
  __syncthreads();
  return before + x - v;
}

}  // namespace hata
