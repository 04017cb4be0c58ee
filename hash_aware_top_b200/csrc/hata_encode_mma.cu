// Prefill HashEncode on the legacy tensor-core path (mma.sync), the fallback of
// the tcgen05 kernel in hata_encode_tc.cu when no TMA tensor map can be made:
// y = x . W_H for every cached key,
// bit = [y > 0], LSB-first pack, written into the code cache ("HATA" paper notes,
// 硬件高效优化: projection -> sign -> bitpack -> cache update in one kernel; this
// is the one genuinely dense contraction of the method, [L x 128] x [128 x r]).
//
// fp32 accuracy from bf16 tiles: the keys are bf16 already (exact), and W_H is
// split once per CTA into three bf16 parts w1 + w2 + w3 (w1 = bf16(w),
// w2 = bf16(w - w1), w3 = bf16(w - w1 - w2)), which carry its 24-bit mantissa;
// every product is exact in fp32 and the three parts accumulate into the same
// fp32 tile.  Only the summation order differs from a scalar fp32 dot product,
// so a code bit can differ from the exact sign only where |y| is within fp32
// rounding of zero.
//
// Layout of the work: W_H^T is the A operand (rows = 16 output columns, held in
// registers for the whole kernel: 8 k-steps x 3 parts x 4 registers), the keys
// are B (8 keys per n-tile, read from a padded shared-memory tile of 64 keys
// filled by cp.async, four tiles in flight), y^T accumulates in fp32.  Warp w owns
// 16 columns and a share of the tile's keys; the sign bits of a (key, 16
// columns) pair are gathered with four ballots and written as one u16, and the
// tile's codes leave as whole words.  CTAs are persistent per (batch, head).
#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kEmThreads = 256;
constexpr int kEmTile = 64;                  // keys per tile
constexpr int kEmRowB = kHeadDim * 2 + 16;   // bytes per staged key row (padded)
constexpr int kEmStages = 4;                 // key tiles in flight per CTA
constexpr int kEmSmem = kEmStages * kEmTile * kEmRowB;

__device__ __forceinline__ void em_cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"((unsigned)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void em_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void em_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
// D += A * B, m16n8k16, bf16 in, fp32 accumulate (PTX fragment layout, g = lane/4, c = lane%4):
//   a0 = A[g][2c..2c+1], a1 = A[g+8][2c..], a2 = A[g][2c+8..], a3 = A[g+8][2c+8..]
//   b0 = B[2c..2c+1][g], b1 = B[2c+8..][g]; d0 = D[g][2c], d1 = D[g][2c+1], d2 = D[g+8][2c], d3 = D[g+8][2c+1]
__device__ __forceinline__ void em_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t em_pack(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}
// bits 0, 4, ..., 28 of x -> bits 0..7
__device__ __forceinline__ uint32_t em_compress8(uint32_t x) {
  x &= 0x11111111u;
  x = (x | (x >> 3)) & 0x03030303u;
  x = (x | (x >> 6)) & 0x000f000fu;
  return (x | (x >> 12)) & 0xffu;
}

template <int R>
__global__ void __launch_bounds__(kEmThreads, 2)
    encode_mma_kernel(const __nv_bfloat16* __restrict__ x, int x_heads, int x_len, int n_tok,
                      const int32_t* __restrict__ seq_end, const float* __restrict__ W, uint32_t* __restrict__ codes,
                      int codes_len, int hpg) {
  constexpr int D = kHeadDim;
  constexpr int NCT = R / 16;         // column tiles (one per warp)
  constexpr int KG = 8 / NCT;         // warps sharing a column tile split the tile's keys
  constexpr int CPW = kEmTile / 8 / KG;  // 8-key chunks per warp per tile
  constexpr int NWd = R / 32;
  static_assert(NCT <= 8 && 8 % NCT == 0, "r in {16..128}");
  extern __shared__ __align__(128) unsigned char xsm[];  // kEmStages tiles of kEmTile padded key rows
  __shared__ uint16_t cs[kEmTile][NCT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2, cq = lane & 3;
  const int ct = warp % NCT, kg = warp / NCT;
  const int bh = blockIdx.y, b = bh / x_heads, h = bh % x_heads, g = h / hpg;

  // A operand: W_H^T rows 16 ct .. 16 ct + 15 (output columns), split in three bf16 parts
  uint32_t A[3][D / 16][4];
  {
    const float* Wg = W + (size_t)g * D * R + 16 * ct + gq;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
      for (int rg = 0; rg < 4; ++rg) {
        const int col = (rg & 1) * 8, kk = 16 * ks + 2 * cq + (rg >> 1) * 8;
        const float w0 = __ldg(Wg + (size_t)kk * R + col), w1 = __ldg(Wg + (size_t)(kk + 1) * R + col);
        const __nv_bfloat16 a1 = __float2bfloat16_rn(w0), b1 = __float2bfloat16_rn(w1);
        const float r0 = w0 - __bfloat162float(a1), r1 = w1 - __bfloat162float(b1);
        const __nv_bfloat16 a2 = __float2bfloat16_rn(r0), b2 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 a3 = __float2bfloat16_rn(r0 - __bfloat162float(a2));
        const __nv_bfloat16 b3 = __float2bfloat16_rn(r1 - __bfloat162float(b2));
        A[0][ks][rg] = em_pack(a1, b1);
        A[1][ks][rg] = em_pack(a2, b2);
        A[2][ks][rg] = em_pack(a3, b3);
      }
  }

  const int end = seq_end ? seq_end[b] : x_len;
  const int lim = min(x_len, codes_len);
  const int ts = max(end - n_tok, 0), te = min(end, lim);  // keys of this (batch, head) to encode
  const int ntile = te > ts ? (te - ts + kEmTile - 1) / kEmTile : 0;
  const __nv_bfloat16* xb = x + ((size_t)b * x_heads + h) * x_len * D;
  uint32_t* cb = codes + ((size_t)b * x_heads + h) * codes_len * NWd;

  auto load = [&](int tile, int st) {  // rows past the end are zeroed (finite; their codes are not written)
    const int r0 = ts + tile * kEmTile, nr = min(kEmTile, te - r0);
    for (int e = tid; e < kEmTile * 16; e += kEmThreads) {
      const int row = e >> 4, pc = e & 15;
      unsigned char* dst = xsm + st * (kEmTile * kEmRowB) + row * kEmRowB + pc * 16;
      if (row < nr) em_cp_async16(dst, xb + (size_t)(r0 + row) * D + pc * 8);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    em_commit();
  };
  // the CTA's tiles are blockIdx.x + i * gridDim.x; tile i goes to stage i % kEmStages,
  // with kEmStages - 1 tiles in flight ahead of the one being encoded (one cp.async
  // group per tile; empty groups past the end keep the count uniform)
#pragma unroll
  for (int i = 0; i < kEmStages - 1; ++i) {
    const int tl = blockIdx.x + i * gridDim.x;
    if (tl < ntile) load(tl, i);
    else em_commit();
  }
  int i = 0;
  for (int tile = blockIdx.x; tile < ntile; tile += gridDim.x, ++i) {
    const int ahead = tile + (kEmStages - 1) * gridDim.x;
    if (ahead < ntile) load(ahead, (i + kEmStages - 1) % kEmStages);
    else em_commit();
    em_wait<kEmStages - 1>();
    __syncthreads();  // this tile's keys have landed; cs is free
    const unsigned char* xt = xsm + (i % kEmStages) * (kEmTile * kEmRowB);
#pragma unroll
    for (int ch = 0; ch < CPW; ++ch) {
      const int n0 = (kg * CPW + ch) * 8;
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      const unsigned char* xrow = xt + (n0 + gq) * kEmRowB + 4 * cq;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xrow + 32 * ks);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(xrow + 32 * ks + 16);
        em_mma(c, A[0][ks], b0, b1);
        em_mma(c, A[1][ks], b0, b1);
        em_mma(c, A[2][ks], b0, b1);
      }
      // c0: (column gq, key 2cq), c1: (gq, 2cq + 1), c2: (gq + 8, 2cq), c3: (gq + 8, 2cq + 1)
      const uint32_t s0 = __ballot_sync(0xffffffffu, c[0] > 0.f), s1 = __ballot_sync(0xffffffffu, c[1] > 0.f);
      const uint32_t s2 = __ballot_sync(0xffffffffu, c[2] > 0.f), s3 = __ballot_sync(0xffffffffu, c[3] > 0.f);
      if (lane < 8) {  // lane n: key n0 + n, columns 16 ct .. 16 ct + 15
        const int kc = lane >> 1;
        const uint32_t lo = em_compress8(((lane & 1) ? s1 : s0) >> kc);
        const uint32_t hi = em_compress8(((lane & 1) ? s3 : s2) >> kc);
        cs[n0 + lane][ct] = (uint16_t)(lo | (hi << 8));
      }
    }
    __syncthreads();
    const int r0 = ts + tile * kEmTile, nr = min(kEmTile, te - r0);
    for (int e = tid; e < nr * NWd; e += kEmThreads) {
      const int key = e / NWd, w = e % NWd;
      cb[(size_t)(r0 + key) * NWd + w] = (uint32_t)cs[key][2 * w] | ((uint32_t)cs[key][2 * w + 1] << 16);
    }
  }
}

}  // namespace

cudaError_t launch_encode_mma(const hata_dims_t& d, const void* x, int x_heads, int x_len, int n_tok,
                              const int32_t* seq_end, const float* W, uint32_t* codes, int codes_len,
                              cudaStream_t st) {
  if (d.dtype != HATA_BF16 || d.hash_bits > 128 || d.hash_bits < 32) return cudaErrorNotSupported;
  // Per device, once under a mutex: the SM count and the shared-memory attributes of the
  // three instantiations.  A failed attribute call makes this form unavailable on that
  // device (cudaErrorNotSupported: the caller uses the SIMT encode).
  static std::mutex mu;
  static std::map<int, std::pair<bool, int>> setup;
  int dev = 0;
  const cudaError_t de = cudaGetDevice(&dev);
  if (de != cudaSuccess) return de;
  int sms = 1;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = setup.find(dev);
    if (it == setup.end()) {
      int n = 0;
      cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(encode_mma_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, kEmSmem);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(encode_mma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kEmSmem);
      if (e == cudaSuccess) e = cudaFuncSetAttribute(encode_mma_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kEmSmem);
      if (e != cudaSuccess) (void)cudaGetLastError();
      it = setup.emplace(dev, std::make_pair(e == cudaSuccess, std::max(n, 1))).first;
    }
    if (!it->second.first) return cudaErrorNotSupported;
    sms = it->second.second;
  }
  const int hpg = x_heads / d.n_kv_heads;
  const long long heads = (long long)d.batch * x_heads;
  const long long tiles = (n_tok + kEmTile - 1) / kEmTile;
  // one wave: two CTAs per SM (registers), split evenly over the (batch, head) pairs
  const unsigned per_head = (unsigned)std::max<long long>(1, std::min<long long>(tiles, (2LL * sms) / heads));
  dim3 grid(per_head, (unsigned)heads);
  const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
  switch (d.hash_bits) {
    case 32: encode_mma_kernel<32><<<grid, kEmThreads, kEmSmem, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 64: encode_mma_kernel<64><<<grid, kEmThreads, kEmSmem, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    case 128: encode_mma_kernel<128><<<grid, kEmThreads, kEmSmem, st>>>(xp, x_heads, x_len, n_tok, seq_end, W, codes, codes_len, hpg); break;
    default: return cudaErrorNotSupported;
  }
  return cudaGetLastError();
}

}  // namespace hata
