// Dense flash-decode over every cached token: exact softmax attention of the G
// query heads of a (batch, KV head) against all L cached K/V rows.  This is the
// dense-attention baseline the "HATA" paper notes measure their decode speed-ups
// against (实验 section: up to 7.2x over dense attention at 128K context); it
// shares the cache layout and inputs of hata_decode_step so the two can be timed
// side by side.
//
// Grid = (splits, B * Hkv), with one wave of CTAs over the GPU's SMs.  Each CTA streams its split in
// tiles of 64 tokens through a two-stage shared-memory buffer (16-byte cp.async
// pieces into rows padded to 272 bytes, so the tensor-core fragment loads hit
// distinct banks), and keeps an online softmax per query head:
//   * logits: one m16n8k16 bf16 tile per warp (rows = query heads, columns = 8
//     tokens, 8 k-steps over the 128 dimensions), fp32 accumulate;
//   * one warp per head takes the tile maximum, rescales, writes the
//     probabilities as bf16 and adds their sum (fixed order);
//   * P.V: each warp owns 16 output columns (two n8 tiles) and accumulates over
//     the tile's 64 rows with ldmatrix.trans V fragments.
// Partials (max, sum, weighted V) go to the workspace; the last CTA of each
// (batch, KV head) to arrive merges them (log-sum-exp) and resets the counter.
#include <algorithm>
#include <map>
#include <mutex>

#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kDnThreads = 256;
constexpr int kDnTile = 64;                      // tokens per tile
constexpr int kDnRowB = kHeadDim * 2 + 16;       // bytes per staged bf16 row (padded)
constexpr int kDnStageB = 2 * kDnTile * kDnRowB;  // K and V tiles of one stage

struct DenseParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int32_t* seq_lens;
  __nv_bfloat16* out;
  float* part;
  uint32_t* count;
  uint32_t* status;
  int Hq, Hkv, max_seq, nsplit, split;  // split: tokens per CTA, a multiple of kDnTile
  float scale_log2;
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
// D += A * B for a 16x16 bf16 A (row), a 16x8 bf16 B (col) and fp32 D, in the
// fragment layout of mma.m16n8k16 (g = lane / 4, c = lane % 4):
//   a0 = A[g][2c..2c+1], a1 = A[g+8][2c..], a2 = A[g][2c+8..], a3 = A[g+8][2c+8..]
//   b0 = B[2c..2c+1][g], b1 = B[2c+8..2c+9][g]; d0 = D[g][2c], d1 = D[g][2c+1], d2, d3 rows g+8
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// Two transposed 8x8 b16 tiles; lanes 0-7 address tile 0's rows, lanes 8-15 tile 1's.
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"((unsigned)__cvta_generic_to_shared(row))
               : "memory");
}

template <int G>
__global__ void __launch_bounds__(kDnThreads, 2) dense_decode_kernel(const DenseParams p) {
  static_assert(G >= 1 && G <= 8, "query heads per KV head: the mma rows 0..7");
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int D = kHeadDim;
  unsigned char* stage = smem;                                                  // [2][K tile, V tile]
  float* lg = reinterpret_cast<float*>(smem + 2 * kDnStageB);                   // [G][kDnTile] logits
  __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(lg + G * kDnTile);      // [G][kDnTile] probabilities
  __shared__ float mrun[G], lrun[G], alph[G];
  __shared__ float wsp[G], Ms[G];
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2, cq = lane & 3;
  const int sp = blockIdx.x, u = blockIdx.y;
  const int b = u / p.Hkv, g = u % p.Hkv;
  int L = p.seq_lens ? p.seq_lens[b] : p.max_seq;
  if (L > p.max_seq) {
    set_status(p.status, HATA_ERR_INVALID_ARG);
    L = p.max_seq;
  }
  L = max(L, 0);
  const int tb = sp * p.split, te = min(L, tb + p.split);
  const int ntile = te > tb ? (te - tb + kDnTile - 1) / kDnTile : 0;
  const __nv_bfloat16* Kb = p.K + (size_t)u * p.max_seq * D;
  const __nv_bfloat16* Vb = p.V + (size_t)u * p.max_seq * D;

  // query fragments (rows = heads; rows >= G are zero), all 8 k-steps
  uint32_t qa0[D / 16], qa2[D / 16];
  {
    const __nv_bfloat16* qh = p.q + ((size_t)b * p.Hq + (size_t)g * G + min(gq, G - 1)) * D + 2 * cq;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa0[ks] = gq < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * ks) : 0u;
      qa2[ks] = gq < G ? *reinterpret_cast<const uint32_t*>(qh + 16 * ks + 8) : 0u;
    }
  }
  if (tid < G) {
    mrun[tid] = -INFINITY;
    lrun[tid] = 0.f;
  }
  // tile t -> stage st: 32 pieces of 16 bytes per token (16 of K, 16 of V); rows
  // past the end of the split are zeroed so they stay finite
  auto load_tile = [&](int t, int st) {
    const int r0 = tb + kDnTile * t, nr = min(kDnTile, te - r0);
    unsigned char* kt = stage + st * kDnStageB;
    unsigned char* vt = kt + kDnTile * kDnRowB;
    for (int e = tid; e < kDnTile * 32; e += kDnThreads) {
      const int row = e >> 5, w = e & 31;
      unsigned char* dst = (w < 16 ? kt : vt) + row * kDnRowB + (w & 15) * 16;
      if (row < nr) {
        const __nv_bfloat16* src = (w < 16 ? Kb : Vb) + (size_t)(r0 + row) * D + (w & 15) * 8;
        cp_async16(dst, src);
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
  };
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // output columns 16 warp + 8 nt + 2c, +1
  if (ntile > 0) load_tile(0, 0);
  for (int t = 0; t < ntile; ++t) {
    const int st = t & 1;
    if (t + 1 < ntile) {
      load_tile(t + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // tile t has landed
    const unsigned char* kt = stage + st * kDnStageB;
    const unsigned char* vt = kt + kDnTile * kDnRowB;
    const int nr = min(kDnTile, te - (tb + kDnTile * t));
    {  // logits of tokens 8 warp .. 8 warp + 7
      float c4[4] = {0.f, 0.f, 0.f, 0.f};
      const unsigned char* krow = kt + (8 * warp + gq) * kDnRowB + 4 * cq;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(krow + 32 * ks);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(krow + 32 * ks + 16);
        mma_16816(c4, qa0[ks], qa2[ks], b0, b1);
      }
      if (gq < G)
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          const int i = 8 * warp + 2 * cq + tt;
          lg[gq * kDnTile + i] = i < nr ? c4[tt] * p.scale_log2 : -INFINITY;
        }
    }
    __syncthreads();
    if (warp < G) {  // online softmax of head `warp` over this tile (64 = 2 x 32 tokens)
      const int h = warp;
      const float v0 = lg[h * kDnTile + lane], v1 = lg[h * kDnTile + 32 + lane];
      float mx = fmaxf(v0, v1);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = mrun[h];
      const float m_new = fmaxf(m_old, mx);  // finite: the tile has at least one token
      const float p0 = exp2f(v0 - m_new), p1 = exp2f(v1 - m_new);  // exp2(-inf) = 0
      pb[h * kDnTile + lane] = __float2bfloat16_rn(p0);
      pb[h * kDnTile + 32 + lane] = __float2bfloat16_rn(p1);
      float sm = p0 + p1;
#pragma unroll
      for (int o = 16; o; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
      __syncwarp();
      if (lane == 0) {
        const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
        alph[h] = alpha;
        lrun[h] = lrun[h] * alpha + sm;
        mrun[h] = m_new;
      }
    }
    __syncthreads();
    {  // P.V into output columns 16 warp .. 16 warp + 15
      const float al = gq < G ? alph[gq] : 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        acc[nt][0] *= al;
        acc[nt][1] *= al;
      }
      const __nv_bfloat16* ph = pb + min(gq, G - 1) * kDnTile + 2 * cq;
#pragma unroll
      for (int ks = 0; ks < kDnTile / 16; ++ks) {
        const uint32_t a0 = gq < G ? *reinterpret_cast<const uint32_t*>(ph + 16 * ks) : 0u;
        const uint32_t a2 = gq < G ? *reinterpret_cast<const uint32_t*>(ph + 16 * ks + 8) : 0u;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t b0, b1;
          ldmatrix_x2_trans(b0, b1, vt + (16 * ks + (lane & 15)) * kDnRowB + (16 * warp + 8 * nt) * 2);
          mma_16816(acc[nt], a0, a2, b0, b1);
        }
      }
    }
    __syncthreads();  // the stage is free for tile t + 2
  }

  // this split's partial: (max, sum) per head, then its weighted V
  float* pp = p.part + ((size_t)u * p.nsplit + sp) * G * (D + 2);
  if (gq < G)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int d0 = 16 * warp + 8 * nt + 2 * cq;
      pp[gq * (D + 2) + 2 + d0] = acc[nt][0];
      pp[gq * (D + 2) + 3 + d0] = acc[nt][1];
    }
  if (tid < G) {
    pp[tid * (D + 2)] = mrun[tid];
    pp[tid * (D + 2) + 1] = lrun[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&p.count[u], 1u) == (unsigned)(p.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // merge: per head the maximum and the weights of the splits, then every column
  const float* pu = p.part + (size_t)u * p.nsplit * G * (D + 2);
  if (warp < G) {
    const int h = warp;
    float M = -INFINITY;
    for (int s2 = lane; s2 < p.nsplit; s2 += 32) M = fmaxf(M, __ldcg(pu + ((size_t)s2 * G + h) * (D + 2)));
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float l = 0.f;
    if (M != -INFINITY)
      for (int s2 = lane; s2 < p.nsplit; s2 += 32) {
        const float* src = pu + ((size_t)s2 * G + h) * (D + 2);
        const float ms2 = __ldcg(src);
        if (ms2 != -INFINITY) l = fmaf(__ldcg(src + 1), exp2f(ms2 - M), l);
      }
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      Ms[h] = M;
      wsp[h] = l;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kDnThreads) {
    const int h = e / D, d = e % D;
    const float M = Ms[h];
    float o = 0.f;
    if (M != -INFINITY) {
#pragma unroll 8
      for (int s2 = 0; s2 < p.nsplit; ++s2) {
        const float* src = pu + ((size_t)s2 * G + h) * (D + 2);
        const float ms2 = __ldcg(src);
        o = fmaf(__ldcg(src + 2 + d), ms2 == -INFINITY ? 0.f : exp2f(ms2 - M), o);
      }
    }
    const float l = wsp[h];
    p.out[((size_t)b * p.Hq + (size_t)g * G + h) * D + d] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
  }
  if (tid == 0) p.count[u] = 0u;
}

// Per device: the shared-memory attribute of dense_decode_kernel<G>, set once under a
// mutex; a failed attribute call is returned on every later launch on that device.
template <int G>
cudaError_t dense_attr_g() {
  static std::mutex mu;
  static std::map<int, cudaError_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(dev);
  if (it == done.end()) {
    e = cudaFuncSetAttribute(dense_decode_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(2 * kDnStageB + 8 * kDnTile * 6));
    if (e != cudaSuccess) (void)cudaGetLastError();
    it = done.emplace(dev, e).first;
  }
  return it->second;
}

template <int G>
cudaError_t launch_dense_g(const DenseParams& prm, int units, size_t smem, cudaStream_t st) {
  const cudaError_t attr = dense_attr_g<G>();
  if (attr != cudaSuccess) return attr;
  dense_decode_kernel<G><<<dim3((unsigned)prm.nsplit, (unsigned)units), kDnThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace

// Tokens per CTA: the splits of all units fill the CTAs that fit on the device
// at once (one wave), rounded to whole tiles.
// CTAs of one wave on the current device (SMs x resident CTAs), found once per device
// under a mutex.
int dense_slots() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    dev = -1;
  }
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    int sms = 0, per_sm = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) sms = 1;
    const size_t smem = 2 * kDnStageB + (size_t)8 * kDnTile * 6;
    if (dev < 0 ||
        cudaFuncSetAttribute(dense_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dense_decode_kernel<8>, kDnThreads, smem) !=
            cudaSuccess)
      per_sm = 1;
    (void)cudaGetLastError();
    it = cache.emplace(dev, std::max(1, std::max(1, sms) * std::max(1, per_sm))).first;
  }
  return it->second;
}

int dense_split(const hata_dims_t& d) {
  const int slots = dense_slots();
  const long long units = (long long)d.batch * d.n_kv_heads;
  const long long per_unit = std::max(1LL, slots / units);
  const long long split = (d.max_seq + per_unit - 1) / per_unit;
  return (int)std::max<long long>(kDnTile, (split + kDnTile - 1) / kDnTile * kDnTile);
}

size_t dense_ws_bytes(const hata_dims_t& d) {
  const size_t units = (size_t)d.batch * d.n_kv_heads, G = d.n_q_heads / d.n_kv_heads;
  const int split = dense_split(d);
  const size_t nsplit = (d.max_seq + split - 1) / split;
  return align_up(kAlign + units * 4, kAlign) + units * nsplit * G * (kHeadDim + 2) * 4;
}

cudaError_t launch_dense_decode(const hata_dims_t& d, const void* q, const void* K, const void* V,
                                const int32_t* seq_lens, float scale, void* out, char* ws, cudaStream_t st) {
  DenseParams prm;
  prm.q = static_cast<const __nv_bfloat16*>(q);
  prm.K = static_cast<const __nv_bfloat16*>(K);
  prm.V = static_cast<const __nv_bfloat16*>(V);
  prm.seq_lens = seq_lens;
  prm.out = static_cast<__nv_bfloat16*>(out);
  const size_t units = (size_t)d.batch * d.n_kv_heads;
  // workspace: status word, arrival counters, then the partials
  prm.status = reinterpret_cast<uint32_t*>(ws);
  prm.count = reinterpret_cast<uint32_t*>(ws + kAlign);
  prm.part = reinterpret_cast<float*>(ws + align_up(kAlign + units * 4, kAlign));
  prm.Hq = d.n_q_heads;
  prm.Hkv = d.n_kv_heads;
  prm.max_seq = d.max_seq;
  prm.split = dense_split(d);
  prm.nsplit = (d.max_seq + prm.split - 1) / prm.split;
  prm.scale_log2 = scale * 1.4426950408889634f;
  const int G = d.n_q_heads / d.n_kv_heads;
  const size_t smem = 2 * kDnStageB + (size_t)G * kDnTile * 6;
  switch (G) {
    case 1: return launch_dense_g<1>(prm, (int)units, smem, st);
    case 2: return launch_dense_g<2>(prm, (int)units, smem, st);
    case 3: return launch_dense_g<3>(prm, (int)units, smem, st);
    case 4: return launch_dense_g<4>(prm, (int)units, smem, st);
    case 5: return launch_dense_g<5>(prm, (int)units, smem, st);
    case 6: return launch_dense_g<6>(prm, (int)units, smem, st);
    case 7: return launch_dense_g<7>(prm, (int)units, smem, st);
    case 8: return launch_dense_g<8>(prm, (int)units, smem, st);
  }
  return cudaErrorNotSupported;
}

}  // namespace hata
