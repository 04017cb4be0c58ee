// Gather-fused sparse flash-decode ("HATA" paper notes, Decode 阶段算法: gather
// the selected K/V pairs and run exact attention on them; 硬件高效优化: gather
// fused into the flash-attention kernel).
//
// Grid = (splits, Hkv, B).  Each CTA takes 32 consecutive entries of idx for one
// (batch, KV head), gathers those K and V rows straight into shared memory with
// 16-byte cp.async (no staging through registers, all rows in flight at once),
// and computes for every query head of the group the flash-decode partial
// (m = max logit, l = sum of exp, o = sum exp * V) over its rows, with logits
// in the exp2 domain.  Partials go to the workspace; the last CTA of each
// (batch, KV head) to arrive (atomic counter, no waiting) merges them with the
// log-sum-exp rule, rounds once to the output type and resets the counter.
#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kSdThreads = 128;
constexpr int kSdMaxG = 16;  // query heads per KV group supported here

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned s = (unsigned)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

template <typename T>
__global__ void __launch_bounds__(kSdThreads)
    sparse_decode_kernel(const T* __restrict__ q, const T* __restrict__ K, const T* __restrict__ V,
                         const int32_t* __restrict__ idx, int k, float scale_log2, T* __restrict__ out,
                         float* part, uint32_t* count, int max_seq, int hkv, int G, uint32_t* status) {
  constexpr int D = kHeadDim, R = kSparseRows;
  constexpr int CPR = D * (int)sizeof(T) / 16;  // 16-byte chunks per row
  __shared__ __align__(16) T Ks[R][D];
  __shared__ __align__(16) T Vs[R][D];
  __shared__ float qs[kSdMaxG][D];
  __shared__ float ps[kSdMaxG][R];
  __shared__ float ms[kSdMaxG], ls[kSdMaxG];
  __shared__ int tok[R];
  __shared__ int s_last;

  const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int nsplit = gridDim.x;
  const size_t bg = (size_t)b * hkv + g;
  const int j0 = sp * R;

  if (tid < R) {
    int t = -1;
    if (j0 + tid < k) {
      t = __ldg(idx + bg * k + j0 + tid);
      if (t >= max_seq) {
        set_status(status, HATA_ERR_INVALID_ARG);
        t = -1;
      }
    }
    tok[tid] = t;
  }
  __syncthreads();
  const T* Kb = K + bg * (size_t)max_seq * D;
  const T* Vb = V + bg * (size_t)max_seq * D;
  for (int e = tid; e < R * CPR; e += kSdThreads) {
    const int r = e / CPR, c = e % CPR;
    const int t = tok[r];
    if (t >= 0) {
      cp_async16(reinterpret_cast<char*>(&Ks[r][0]) + 16 * c, reinterpret_cast<const char*>(Kb + (size_t)t * D) + 16 * c);
      cp_async16(reinterpret_cast<char*>(&Vs[r][0]) + 16 * c, reinterpret_cast<const char*>(Vb + (size_t)t * D) + 16 * c);
    }
  }
  const T* qb = q + ((size_t)b * hkv * G + (size_t)g * G) * D;
  for (int e = tid; e < G * D; e += kSdThreads) qs[e / D][e % D] = to_f32(qb[e]);
  cp_async_wait_all();
  __syncthreads();

  // logits: one warp per (head, row) pair, lanes split d, warp reduction
  const int lane = tid & 31, warp = tid >> 5;
  for (int pr = warp; pr < G * R; pr += kSdThreads / 32) {
    const int h = pr / R, r = pr % R;
    float s = -INFINITY;
    if (tok[r] >= 0) {
      float a = 0.f;
#pragma unroll
      for (int u = 0; u < D / 32; ++u) a = fmaf(qs[h][lane + 32 * u], to_f32(Ks[r][lane + 32 * u]), a);
#pragma unroll
      for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      s = a * scale_log2;
    }
    if (lane == 0) ps[h][r] = s;
  }
  __syncthreads();
  // per-head max and exp (R == 32: one lane per row)
  for (int h = warp; h < G; h += kSdThreads / 32) {
    const float s = ps[h][lane];
    float m = s;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float p = (m == -INFINITY) ? 0.f : exp2f(s - m);
    float l = p;
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    ps[h][lane] = p;
    if (lane == 0) {
      ms[h] = m;
      ls[h] = l;
    }
  }
  __syncthreads();
  // o[h][i] = sum_r p[h][r] * V[r][i]; thread i = tid (D == kSdThreads)
  float* pb = part + bg * (size_t)nsplit * G * (D + 2);
  for (int h = 0; h < G; ++h) {
    float o = 0.f;
#pragma unroll 8
    for (int r = 0; r < R; ++r)
      if (tok[r] >= 0) o = fmaf(ps[h][r], to_f32(Vs[r][tid]), o);
    float* dst = pb + ((size_t)sp * G + h) * (D + 2);
    dst[2 + tid] = o;
    if (tid == 0) {
      dst[0] = ms[h];
      dst[1] = ls[h];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&count[bg], 1u) == (unsigned)(nsplit - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // merge the partials of every split (log-sum-exp), thread i = output column
  T* ob = out + ((size_t)b * hkv * G + (size_t)g * G) * D;
  for (int h = 0; h < G; ++h) {
    float M = -INFINITY;
    for (int s2 = 0; s2 < nsplit; ++s2) M = fmaxf(M, __ldcg(pb + ((size_t)s2 * G + h) * (D + 2)));
    float l = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < nsplit; ++s2) {
        const float* src = pb + ((size_t)s2 * G + h) * (D + 2);
        const float ms2 = __ldcg(src);
        if (ms2 == -INFINITY) continue;
        const float w = exp2f(ms2 - M);
        l = fmaf(__ldcg(src + 1), w, l);
        o = fmaf(__ldcg(src + 2 + tid), w, o);
      }
    }
    ob[(size_t)h * D + tid] = from_f32<T>(l > 0.f ? o / l : 0.f);
  }
  if (tid == 0) count[bg] = 0u;
}

template <typename T>
cudaError_t launch_t(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K, const void* V,
                     const int32_t* idx, int k, float scale, void* out, char* ws, cudaStream_t st) {
  const int G = d.n_q_heads / d.n_kv_heads;
  dim3 grid(L.nsplit, d.n_kv_heads, d.batch);
  const float scale_log2 = scale * 1.4426950408889634f;
  sparse_decode_kernel<T><<<grid, kSdThreads, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(K), static_cast<const T*>(V), idx, k, scale_log2,
      static_cast<T*>(out), reinterpret_cast<float*>(ws + L.sp_part), reinterpret_cast<uint32_t*>(ws + L.sp_count),
      d.max_seq, d.n_kv_heads, G, reinterpret_cast<uint32_t*>(ws + L.status));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_decode(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K,
                                 const void* V, const int32_t* idx, int k, float scale, void* out, char* ws,
                                 cudaStream_t stream) {
  if (d.dtype == HATA_BF16) return launch_t<__nv_bfloat16>(d, L, q, K, V, idx, k, scale, out, ws, stream);
  return launch_t<float>(d, L, q, K, V, idx, k, scale, out, ws, stream);
}

}  // namespace hata
