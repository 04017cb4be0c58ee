// Prefill HashEncode on the 5th-generation tensor cores: y = x . W_H for every
// cached key, bit = [y > 0], LSB-first pack, written into the code cache ("HATA"
// paper notes, 硬件高效优化: projection -> sign -> bitpack -> cache update in one
// kernel; this is the one genuinely dense contraction of the method,
// [L x 128] x [128 x r]).
//
// fp32 accuracy from bf16 operands: the keys are bf16 already (exact), and W_H is
// split once per CTA into three bf16 parts w1 + w2 + w3 (w1 = bf16(w),
// w2 = bf16(w - w1), w3 = bf16(w - w1 - w2)), which carry its 24-bit mantissa;
// every product is exact in fp32 and the three parts accumulate into the same
// fp32 accumulator.  Only the summation order differs from a scalar fp32 dot
// product, so a code bit can differ from the exact sign only where |y| is within
// fp32 rounding of zero.
//
// One CTA of five warps per SM, persistent over the 128-key tiles of one
// (batch, head):
//   * W_H^T (three parts, r x 128 each) sits in shared memory in the K-major
//     core-matrix layout the tensor core reads without swizzling: 8 rows x 16
//     bytes per core matrix (128 contiguous bytes), the 16 core matrices along K
//     of an 8-row group next to each other (128 bytes apart), 8-row groups 2048
//     bytes apart;
//   * key tiles arrive by TMA (two 2-D boxes of 128 keys x 64 elements, 128-byte
//     swizzle: the K-major layout with 1024-byte 8-row groups that the tensor
//     core reads directly), S tiles in flight, each completing on its stage's
//     mbarrier;
//   * warp 4 (one lane) issues the tile's MMAs (M = 128 keys, K = 16 each,
//     kind::f16 with bf16 inputs and fp32 accumulation; for r <= 64 one MMA of
//     N = 3r per K step over the three stacked parts, for r = 128 three of N = r)
//     into one of two TMEM accumulators, commits them to an mbarrier, and refills
//     a stage as soon as the MMAs reading it are done;
//   * warps 0-3 read each finished accumulator (warp w owns TMEM lanes
//     32w .. 32w + 31, i.e. keys), add the parts, turn 32 columns at a time into
//     a code word, store each key's code as one vector and release the
//     accumulator on a 128-thread mbarrier.  No CTA-wide barrier inside the loop.
// Every wait is bounded: on expiry the kernel records HATA_ERR_TIMEOUT in the
// caller's status word (the workspace passed to hata_encode_append), stops
// issuing work, waits (bounded) for the MMAs it issued, frees its TMEM and
// returns.
#include <algorithm>
#include <map>
#include <mutex>

#include "hata_kernels.cuh"
#include "hata_tc.cuh"

namespace hata {

namespace {

constexpr int kTcThreads = 160;  // warps 0-3: epilogue (TMEM lanes 32w..); warp 4: TMA + MMA issue
constexpr int kTcEpi = 128;
constexpr int kTcTile = 128;                          // keys per tile (the MMA's M)
constexpr int kTcTileBytes = kTcTile * kHeadDim * 2;  // 32 KB of bf16 keys
constexpr int kTcSmemBudget = 200 * 1024;
constexpr uint32_t kTcWaitTries = 1u << 22;

__host__ __device__ constexpr int tc_w_bytes(int R) { return 3 * R * kHeadDim * 2; }
__host__ __device__ constexpr int tc_stages(int R) {
  return (kTcSmemBudget - tc_w_bytes(R)) / kTcTileBytes > 5 ? 5 : (kTcSmemBudget - tc_w_bytes(R)) / kTcTileBytes;
}
// + 1 KB to align the key stages to the 1024 bytes of the 128-byte swizzle
__host__ __device__ constexpr int tc_smem(int R) { return tc_w_bytes(R) + tc_stages(R) * kTcTileBytes + 1024; }

// byte offset of the 16-byte chunk (row, k .. k + 7) in the core-matrix layout
__device__ __forceinline__ uint32_t cm_off(int row, int k) {
  return (uint32_t)((((row >> 3) * (kHeadDim / 8) + (k >> 3)) << 7) + ((row & 7) << 4));
}

// r <= 64: the three W_H^T parts, stacked, are one B operand of N = 3r (each key
// slice is read from shared memory once per K step); the epilogue adds the three
// column groups.  r = 128: three accumulating MMAs of N = r per K step.
__host__ __device__ constexpr bool tc_cat(int R) { return 3 * R <= 256; }
__host__ __device__ constexpr int tc_acc_cols(int R) { return tc_cat(R) ? 3 * R : R; }  // per accumulator
__host__ __device__ constexpr int tc_tmem_cols(int R) {  // two accumulators, rounded to a power of two
  return 2 * tc_acc_cols(R) <= 64 ? 64 : 2 * tc_acc_cols(R) <= 128 ? 128 : 2 * tc_acc_cols(R) <= 256 ? 256 : 512;
}

// bounded wait for the phase of the given parity (false: not complete after the limit)
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity) { return tc::mbar_wait(bar, parity, kTcWaitTries); }

template <int R>
__global__ void __launch_bounds__(kTcThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap xmap, int x_heads, int x_len, int n_tok,
                     const int32_t* __restrict__ seq_end, const float* __restrict__ W, uint32_t* __restrict__ codes,
                     int codes_len, int hpg, uint32_t* status) {
  constexpr int D = kHeadDim;
  constexpr int NWd = R / 32;
  constexpr int S = tc_stages(R);
  constexpr int WPART = R * D * 2;  // bytes of one W_H^T part
  static_assert(S >= 2, "shared memory for at least two key tiles");
  static_assert(R % 32 == 0 && R >= 32 && R <= 128, "N = r in {32, 64, 128}");
  constexpr bool CAT = tc_cat(R);
  constexpr int AC = tc_acc_cols(R);
  constexpr int TCOLS = tc_tmem_cols(R);
  static_assert(2 * AC <= TCOLS && TCOLS <= 512, "two accumulators in TMEM");
  extern __shared__ __align__(1024) unsigned char sm[];  // [3 W_H^T parts][pad][S key tiles]
  __shared__ __align__(8) uint64_t full[S];               // key tile landed in stage s
  __shared__ __align__(8) uint64_t mma_done[2];           // MMAs into accumulator a complete
  __shared__ __align__(8) uint64_t acc_free[2];           // accumulator a read by all 128 threads
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s, loaded_s, issued_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y, b = bh / x_heads, h = bh % x_heads, g = h / hpg;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
  const uint32_t xbase = (sbase + 3 * WPART + 1023u) & ~1023u;  // key stages, 1024-byte aligned

  const int end = seq_end ? seq_end[b] : x_len;
  const int lim = min(x_len, codes_len);
  const int ts = max(end - n_tok, 0), te = min(end, lim);  // keys of this (batch, head) to encode
  const int ntile = te > ts ? (te - ts + kTcTile - 1) / kTcTile : 0;
  const int nmine = ntile > (int)blockIdx.x ? (ntile - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const int row_base = (b * x_heads + h) * x_len + ts;  // tensor-map row of this slab's first key to encode
  uint32_t* cb = codes + ((size_t)b * x_heads + h) * codes_len * NWd;

  if (warp == 0) {  // two fp32 accumulators of R columns each
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(&tmem_base_s)),
                 "r"(TCOLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // the i-th tile of this CTA (tile blockIdx.x + i * gridDim.x) into stage i % S
  auto issue_load = [&](int i) {
    const int tile = (int)blockIdx.x + i * (int)gridDim.x;
    const uint32_t dst = xbase + (uint32_t)(i % S) * kTcTileBytes;
    tc::mbar_expect(&full[i % S], (uint32_t)kTcTileBytes);
    tc::tma_load_2d(dst, &xmap, 0, row_base + tile * kTcTile, &full[i % S]);
    tc::tma_load_2d(dst + kTcTileBytes / 2, &xmap, 64, row_base + tile * kTcTile, &full[i % S]);
    loaded_s = i + 1;
  };
  if (tid == 0) {
    for (int s_ = 0; s_ < S; ++s_)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"((uint32_t)__cvta_generic_to_shared(&full[s_])));
    for (int a_ = 0; a_ < 2; ++a_) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"((uint32_t)__cvta_generic_to_shared(&mma_done[a_])));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"((uint32_t)__cvta_generic_to_shared(&acc_free[a_])),
                   "r"(kTcEpi));
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    abort_s = 0;
    loaded_s = 0;
    issued_s = 0;
    for (int i = 0; i < min(S, nmine); ++i) issue_load(i);  // keys stream in while W_H is split below
  }

  // W_H^T split into three bf16 parts, one (column n, 8 consecutive k) chunk per step
  {
    const float* Wg = W + (size_t)g * D * R;
    for (int it = tid; it < R * (D / 8); it += kTcThreads) {
      const int n = it % R, k0 = (it / R) * 8;
      __align__(16) __nv_bfloat16 p1[8], p2[8], p3[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float w = __ldg(Wg + (size_t)(k0 + e) * R + n);
        p1[e] = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(p1[e]);
        p2[e] = __float2bfloat16_rn(r1);
        p3[e] = __float2bfloat16_rn(r1 - __bfloat162float(p2[e]));
      }
      const uint32_t off = cm_off(n, k0);
      *reinterpret_cast<uint4*>(sm + off) = *reinterpret_cast<const uint4*>(p1);
      *reinterpret_cast<uint4*>(sm + WPART + off) = *reinterpret_cast<const uint4*>(p2);
      *reinterpret_cast<uint4*>(sm + 2 * WPART + off) = *reinterpret_cast<const uint4*>(p3);
    }
  }
  tc::fence_async_smem();  // the W_H parts (generic stores) before the tensor core reads them
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t idesc = tc::idesc_bf16(kTcTile, CAT ? 3 * R : R, false);
  const uint64_t bd0 = tc::desc_kmajor_cm(sbase);  // W_H^T part 0, first K step

  // bounded wait; on expiry record the timeout once and stop issuing work
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) {
    if (abort_s) return false;
    if (tc_wait(bar, parity)) return true;
    if (!abort_s) set_status(status, HATA_ERR_TIMEOUT);
    abort_s = 1;
    return false;
  };
  // codes of this CTA's tile i (accumulator i & 1): warp w holds keys 32w .. 32w + 31
  auto epilogue = [&](int i) {
    const int r0 = ts + ((int)blockIdx.x + i * (int)gridDim.x) * kTcTile, key = 32 * warp + lane;
    uint32_t word[NWd];
#pragma unroll
    for (int c = 0; c < NWd; ++c) {
      const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)((i & 1) * AC + 32 * c);
      uint32_t v[32];
      tc::ld32(ta, v);
      if constexpr (CAT) {  // y = (x.w1 + x.w2) + x.w3
        uint32_t v2[32], v3[32];
        tc::ld32(ta + R, v2);
        tc::ld32(ta + 2 * R, v3);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = __float_as_uint((__uint_as_float(v[j]) + __uint_as_float(v2[j])) + __uint_as_float(v3[j]));
      }
      uint32_t bits = 0u;
#pragma unroll
      for (int j = 0; j < 32; ++j) bits |= (__uint_as_float(v[j]) > 0.f ? 1u : 0u) << j;
      word[c] = bits;
    }
    if (r0 + key < te) {
      uint32_t* dst = cb + (size_t)(r0 + key) * NWd;
      if constexpr (NWd == 4) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(word[0], word[1], word[2], word[3]);
      } else if constexpr (NWd == 2) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(word[0], word[1]);
      } else {
        dst[0] = word[0];
      }
    }
  };

  if (warp == 4) {
    if (lane == 0) {  // producer: the MMAs of tile i, then the refill of the stage tile i - 1 used
      for (int i = 0; i < nmine; ++i) {
        bool ok = wait_or_abort(&full[i % S], (uint32_t)((i / S) & 1));
        if (ok && i >= 2) ok = wait_or_abort(&acc_free[i & 1], (uint32_t)(((i - 2) >> 1) & 1));
        if (!ok) break;
        tc::fence_after();
        // descriptors advance by adding (byte offset >> 4) to the start-address field
        // (every address stays below 256 KB, so the field never carries)
        const uint64_t ad0 = tc::desc_kmajor_sw128(xbase + (uint32_t)(i % S) * kTcTileBytes);
        const uint32_t d = tmem + (uint32_t)((i & 1) * AC);
#pragma unroll
        for (int p = 0; p < (CAT ? 1 : 3); ++p)
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc::mma(d, ad0 + (uint64_t)(((ks >> 2) * (kTcTileBytes / 2) + (ks & 3) * 32) >> 4),
                   bd0 + (uint64_t)((p * WPART + ks * 256) >> 4), idesc, (p | ks) ? 1u : 0u);
        tc::commit(&mma_done[i & 1]);
        issued_s = i + 1;
        if (i >= 1 && i - 1 + S < nmine) {  // tile i - 1's MMAs done: its stage takes tile i - 1 + S
          if (!wait_or_abort(&mma_done[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1))) break;
          issue_load(i - 1 + S);
        }
      }
    }
  } else {  // epilogue warps: tile j's codes once its MMAs are done, then free its accumulator
    for (int j = 0; j < nmine; ++j) {
      const bool ok = wait_or_abort(&mma_done[j & 1], (uint32_t)((j >> 1) & 1));
      tc::fence_after();
      if (ok) epilogue(j);
      tc::fence_before();
      tc::mbar_arrive(&acc_free[j & 1]);
      if (!ok) break;
    }
  }
  __syncthreads();
  if (warp == 0) {
    if (abort_s && lane == 0) {  // let the copies and MMAs already issued finish (bounded) before leaving
      for (int j = max(0, loaded_s - S); j < loaded_s; ++j) tc_wait(&full[j % S], (uint32_t)((j / S) & 1));
      if (issued_s > 0) tc_wait(&mma_done[(issued_s - 1) & 1], (uint32_t)(((issued_s - 1) >> 1) & 1));
    }
    __syncwarp();
    tc::fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(TCOLS) : "memory");
  }
}

// Per device: the SM count and the shared-memory attributes of the three
// instantiations, set once under a mutex.  A failed attribute call is returned
// (the caller then uses another encode kernel).
cudaError_t tc_device_setup(int* sms_out) {
  static std::mutex mu;
  static std::map<int, std::pair<cudaError_t, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(dev);
  if (it == done.end()) {
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(encode_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem(32));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(encode_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem(64));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(encode_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc_smem(128));
    if (e != cudaSuccess) (void)cudaGetLastError();
    it = done.emplace(dev, std::make_pair(e, std::max(sms, 1))).first;
  }
  *sms_out = it->second.second;
  return it->second.first;
}

}  // namespace

cudaError_t launch_encode_tc(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                             const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len,
                             uint32_t* status, cudaStream_t st) {
  if (d.dtype != HATA_BF16 || d.hash_bits > 128 || d.hash_bits < 32) return cudaErrorNotSupported;
  int sms = 0;
  if (tc_device_setup(&sms) != cudaSuccess) return cudaErrorNotSupported;
  const int hpg = x_heads / d.n_kv_heads;
  const long long heads = (long long)d.batch * x_heads;
  const long long tiles = (n_tok + kTcTile - 1) / kTcTile;
  const long long rows = heads * x_len;
  if (rows + kTcTile >= 0x7fffffffLL) return cudaErrorNotSupported;
  // x as a 2-D tensor [rows][128] bf16; boxes of 128 rows x 64 elements, 128-byte swizzle
  CUtensorMap xmap;
  if (!make_bf16_rows_map(&xmap, x, rows, kTcTile)) return cudaErrorNotSupported;
  // Few (batch, head) pairs: one wave, one CTA per SM split evenly over the pairs.  Many
  // pairs (per-sequence lengths are only known on the device, and may differ widely): about
  // four waves of CTAs, several per pair striding over its tiles, so that the block
  // scheduler evens out long and short sequences.
  long long per = sms / heads;
  if (per < 4) per = (4LL * sms + heads - 1) / heads;
  const unsigned per_head = (unsigned)std::max<long long>(1, std::min<long long>(tiles, per));
  dim3 grid(per_head, (unsigned)heads);
  switch (d.hash_bits) {
    case 32:
      encode_tc_kernel<32><<<grid, kTcThreads, tc_smem(32), st>>>(xmap, x_heads, x_len, n_tok, seq_end, W, codes,
                                                                  codes_len, hpg, status);
      break;
    case 64:
      encode_tc_kernel<64><<<grid, kTcThreads, tc_smem(64), st>>>(xmap, x_heads, x_len, n_tok, seq_end, W, codes,
                                                                  codes_len, hpg, status);
      break;
    case 128:
      encode_tc_kernel<128><<<grid, kTcThreads, tc_smem(128), st>>>(xmap, x_heads, x_len, n_tok, seq_end, W, codes,
                                                                    codes_len, hpg, status);
      break;
    default:
      return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace hata
