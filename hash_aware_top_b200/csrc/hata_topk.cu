// Top-k select over the small integer score range ("HATA" paper notes, Decode
// 阶段算法: select top-k; ties go to the lower token index, indices ascending).
//
// Scores of one (batch, KV head) lie in [0, G * r], so top-k is a counting
// problem: with hist[v] = #(score == v), the threshold T is the smallest v with
// #(score <= T) >= n = min(k, L); every token below T is selected, plus the
// first m = n - #(score < T) tokens (in index order) that equal T.
//
// Pass 1 (one CTA per 4096-token chunk): shared-memory histogram of the chunk,
// written to the workspace; the last CTA of each (batch, KV head) to arrive
// (atomic counter, no waiting) sums the chunk histograms, finds T and m, and
// turns per-chunk counts into two prefixes per chunk: selected-before and
// ties-before.  Pass 2 (same grid): each chunk ranks its own tokens with two
// block scans and writes their indices at their final ascending positions.
#include <climits>

#include "hata_kernels.cuh"

namespace hata {

namespace {

constexpr int kTkThreads = 512;
constexpr int kTkTPT = kTopkChunk / kTkThreads;  // 8 consecutive tokens per thread

__global__ void __launch_bounds__(kTkThreads)
    topk_hist_kernel(const int32_t* __restrict__ scores, const int32_t* __restrict__ seq_lens, int k, int max_seq,
                     int hkv, int nbins, int nchunk, int32_t* hist_ws, int32_t* chunk_ws, int32_t* thr_ws,
                     uint32_t* count_ws, uint32_t* status) {
  extern __shared__ int hist[];  // [max(nbins, 2 * nchunk)]
  __shared__ int warp_sums[kTkThreads / 32];
  __shared__ int s_last, s_T, s_m;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = clamp_len(seq_lens, b, max_seq, status);
  const int nact = (L + kTopkChunk - 1) / kTopkChunk;
  if (c >= nact) return;
  const size_t bg = (size_t)b * hkv + g;

  for (int v = tid; v < nbins; v += kTkThreads) hist[v] = 0;
  __syncthreads();
  const int32_t* sc = scores + bg * max_seq;
  const int t_end = min(L, (c + 1) * kTopkChunk);
  for (int t = c * kTopkChunk + tid; t < t_end; t += kTkThreads) {
    int v = __ldg(sc + t);
    if (v < 0 || v >= nbins) {
      set_status(status, HATA_ERR_INVALID_ARG);
      v = v < 0 ? 0 : nbins - 1;
    }
    atomicAdd(&hist[v], 1);
  }
  __syncthreads();
  int32_t* hb = hist_ws + bg * nchunk * nbins;
  for (int v = tid; v < nbins; v += kTkThreads) hb[(size_t)c * nbins + v] = hist[v];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&count_ws[bg], 1u) == (unsigned)(nact - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last CTA of this (b, g): total histogram, threshold, per-chunk prefixes.
  for (int v = tid; v < nbins; v += kTkThreads) {
    int s = 0;
    for (int cc = 0; cc < nact; ++cc) s += __ldcg(hb + (size_t)cc * nbins + v);
    hist[v] = s;
  }
  __syncthreads();
  const int n = min(k, L);
  if (tid == 0) {  // always overwritten below (the histogram holds L >= n tokens); set for safety
    s_T = nbins - 1;
    s_m = 0;
  }
  const int span = (nbins + kTkThreads - 1) / kTkThreads;
  const int v0 = tid * span, v1 = min(nbins, v0 + span);
  int local = 0;
  for (int v = v0; v < v1; ++v) local += hist[v];
  int tot;
  int before = block_exclusive_scan<kTkThreads>(local, warp_sums, &tot);
  for (int v = v0; v < v1; ++v) {
    if (before < n && before + hist[v] >= n) {
      s_T = v;
      s_m = n - before;
    }
    before += hist[v];
  }
  __syncthreads();
  const int T = s_T, m = s_m;
  // per-chunk counts below T and equal to T (one warp per chunk), then a serial prefix
  int* less = hist;           // reuse shared memory: [nact]
  int* eq = hist + nact;      // [nact]
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  for (int cc = warp; cc < nact; cc += kTkThreads / 32) {
    int s = 0;
    for (int v = lane; v < T; v += 32) s += __ldcg(hb + (size_t)cc * nbins + v);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      less[cc] = s;
      eq[cc] = __ldcg(hb + (size_t)cc * nbins + T);
    }
  }
  __syncthreads();
  if (tid == 0) {
    int sel = 0, ties = 0;
    int32_t* cw = chunk_ws + bg * nchunk * 2;
    for (int cc = 0; cc < nact; ++cc) {
      cw[2 * cc] = sel;
      cw[2 * cc + 1] = ties;
      const int take = min(max(m - ties, 0), eq[cc]);
      sel += less[cc] + take;
      ties += eq[cc];
    }
    thr_ws[bg * 2] = T;
    thr_ws[bg * 2 + 1] = m;
    count_ws[bg] = 0u;
  }
}

__global__ void __launch_bounds__(kTkThreads)
    topk_select_kernel(const int32_t* __restrict__ scores, const int32_t* __restrict__ seq_lens, int k, int max_seq,
                       int hkv, int nbins, int nchunk, const int32_t* chunk_ws, const int32_t* thr_ws,
                       int32_t* __restrict__ idx, int32_t* __restrict__ n_sel) {
  __shared__ int warp_sums[kTkThreads / 32];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = clamp_len(seq_lens, b, max_seq, nullptr);
  const int n = min(k, L);
  const size_t bg = (size_t)b * hkv + g;
  int32_t* ib = idx + bg * k;
  for (int j = n + c * kTkThreads + tid; j < k; j += nchunk * kTkThreads) ib[j] = -1;
  if (n_sel && c == 0 && g == 0 && tid == 0) n_sel[b] = n;
  const int nact = (L + kTopkChunk - 1) / kTopkChunk;
  if (c >= nact) return;

  const int T = __ldcg(thr_ws + bg * 2), m = __ldcg(thr_ws + bg * 2 + 1);
  const int sel_before = __ldcg(chunk_ws + (bg * nchunk + c) * 2);
  const int ties_before = __ldcg(chunk_ws + (bg * nchunk + c) * 2 + 1);
  const int32_t* sc = scores + bg * max_seq;
  const int t0 = c * kTopkChunk + tid * kTkTPT;
  int v[kTkTPT];
  int n_eq = 0;
#pragma unroll
  for (int u = 0; u < kTkTPT; ++u) {
    const int t = t0 + u;
    int s = t < L ? __ldg(sc + t) : INT_MAX;
    s = s < 0 ? 0 : (s >= nbins && t < L ? nbins - 1 : s);
    v[u] = s;
    n_eq += (s == T);
  }
  int tot;
  int tie_rank = ties_before + block_exclusive_scan<kTkThreads>(n_eq, warp_sums, &tot);
  unsigned selmask = 0;
#pragma unroll
  for (int u = 0; u < kTkTPT; ++u) {
    bool s = v[u] < T;
    if (v[u] == T) {
      s = tie_rank < m;
      ++tie_rank;
    }
    selmask |= (unsigned)s << u;
  }
  int pos = sel_before + block_exclusive_scan<kTkThreads>(__popc(selmask), warp_sums, &tot);
#pragma unroll
  for (int u = 0; u < kTkTPT; ++u)
    if (selmask >> u & 1u) {
      if (pos < n) ib[pos] = t0 + u;  // always true when scores are unchanged since pass 1
      ++pos;
    }
}

}  // namespace

cudaError_t launch_topk(const hata_dims_t& d, const WsLayout& L, const int32_t* scores, const int32_t* seq_lens,
                        int k, int32_t* idx, int32_t* n_sel, char* ws, cudaStream_t st) {
  dim3 grid(L.nchunk, d.n_kv_heads, d.batch);
  const size_t smem = (size_t)max(L.nbins, 2 * L.nchunk) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  topk_hist_kernel<<<grid, kTkThreads, smem, st>>>(
      scores, seq_lens, k, d.max_seq, d.n_kv_heads, L.nbins, L.nchunk, reinterpret_cast<int32_t*>(ws + L.topk_hist),
      reinterpret_cast<int32_t*>(ws + L.topk_chunk), reinterpret_cast<int32_t*>(ws + L.topk_thr),
      reinterpret_cast<uint32_t*>(ws + L.topk_count), status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<grid, kTkThreads, 0, st>>>(scores, seq_lens, k, d.max_seq, d.n_kv_heads, L.nbins, L.nchunk,
                                                  reinterpret_cast<const int32_t*>(ws + L.topk_chunk),
                                                  reinterpret_cast<const int32_t*>(ws + L.topk_thr), idx, n_sel);
  return cudaGetLastError();
}

}  // namespace hata
