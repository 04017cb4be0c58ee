// Fused HATA decode step: one kernel, one thread-block cluster per
// (batch, KV head) unit ("HATA" paper notes, Decode 阶段算法 end to end, with the
// fusions of 硬件高效优化).
//
// A unit's L cached tokens are split evenly over the CS CTAs of its cluster.
// Each CTA:
//   1. streams its slice of the code cache into a 4-8 stage shared-memory ring
//      with bulk (TMA) copies, evict-first in L2, issued as soon as L is known;
//   2. encodes the G queries and the new key for its slice of the W_H columns
//      (warp_dot128: the same arithmetic as hata_encode_append's decode form),
//      stores its code bits into a per-source slot of every CTA of the cluster;
//      after a cluster barrier each CTA ORs the slots locally, and the CTA
//      owning slot L - 1 appends the key code to the cache;
//   3. scores every token of its slice (xor + popc with the GQA sum folded into
//      per-word constants and a carry-save popc sum), keeping the u16 scores and
//      their histogram in shared memory; warps release ring stages on their own;
//   4. turns the histogram into a cumulative one and stores it (u16) into its
//      slot of every CTA; guesses its own share of the selection from it and
//      starts gathering those candidate K/V rows (cp.async) right away;
//   5. after a cluster barrier, every CTA sums the CS cumulative histograms
//      (one bin per thread) to find the unit's threshold T (the smallest score
//      with at least n = min(k, L) tokens at or below it), the tie quota m and
//      the counts of earlier CTAs, so ties go to the lower token index exactly
//      as in a global sort;
//   6. computes the flash-decode partial (max, sum, weighted V) of each of the G
//      query heads over its selected rows (falling back to a second gather when
//      the guess missed), and stores each partial's column slice into the CTA
//      that owns those output columns; after a last cluster barrier every CTA
//      merges its columns (log-sum-exp) and writes them.
// Cross-CTA traffic is only stores into other CTAs' shared memory before a
// hardware cluster barrier: no remote loads, no global-memory flags, no
// workspace.  The only waits are bounded mbarrier waits on this CTA's own
// bulk copies.
#include <algorithm>
#include <climits>
#include <map>
#include <mutex>
#include <tuple>

#include "hata_kernels.cuh"
#include "hata_ptx.cuh"

namespace hata {

namespace {

constexpr int kFThreads = 512;
constexpr int kNWarp = kFThreads / 32;
constexpr int kMaxStages = 6;        // ring stages (32 KB each), 2..6 depending on shared memory left
constexpr int kMinStages = 2;
constexpr int kStageBytes = 32768;
constexpr int kTokCap = 65520;       // max tokens per CTA: u16 scores and u16 cumulative counts
constexpr int kWCols = 32;           // W_H columns staged per encode batch
constexpr int kMaxCS = 16;           // largest cluster
constexpr int kMaxGB = 256;          // largest gather batch (rows)
constexpr int kOneCtaSmem = 116 * 1024;  // dynamic shared memory that keeps one CTA per SM
constexpr uint32_t kWaitTries = 1u << 22;

struct FusedParams {
  const void* q;
  const void* K;
  const void* V;
  const float* W;
  uint32_t* codes;
  const int32_t* seq_lens;
  void* out;
  uint32_t* qcode_out;
  int32_t* idx_out;
  uint32_t* status;
  int Hq, Hkv, max_seq, k, nbins, tok_cap, sel_cap, wcols, flags, stages;
  float scale_log2;
};

struct SmemLayout {
  uint32_t ring, D, hist, hslot, xs, wsl, enc, qslot, sel, lg, part, mslot, stat, mbar, total;
  int nbp, mcols, gb;
};

struct Bump {
  uint32_t o = 0;
  __host__ __device__ uint32_t take(uint32_t bytes, uint32_t align) {
    o = (o + align - 1) / align * align;
    const uint32_t r = o;
    o += bytes;
    return r;
  }
};

// W_H columns encoded by each CTA of a cluster of CS: ceil(r / CS) rounded up to
// a multiple of 4 (the last ranks may get fewer, or none).
__host__ __device__ inline int enc_cols_per_cta(int R, int CS) { return ((R + CS - 1) / CS + 3) / 4 * 4; }

// Output columns merged by each CTA of a cluster of CS (the last one may have fewer).
__host__ __device__ inline int merge_cols(int G, int CS) { return (G * kHeadDim + CS - 1) / CS; }

__host__ __device__ inline SmemLayout smem_layout(int G, int NW, int esize, int tok_cap, int sel_cap, int nbins,
                                                  int wcols, int CS, int stages) {
  SmemLayout s;
  Bump b;
  s.nbp = (nbins + 7) / 8 * 8;  // histogram bins padded to whole 16-byte groups of u16
  s.mcols = merge_cols(G, CS);
  s.gb = stages * kStageBytes / (2 * kHeadDim * esize);
  if (s.gb > kMaxGB) s.gb = kMaxGB;
  s.ring = b.take(stages * kStageBytes, 128);
  s.D = b.take(tok_cap * 2, 16);
  s.hist = b.take(s.nbp * 4, 16);                     // local counts, then cumulative, then unit totals
  s.hslot = b.take(CS * s.nbp * 2, 16);               // u16 cumulative histograms from every CTA
  s.xs = b.take((G + 1) * kHeadDim * 4, 16);          // G queries + new key, fp32
  s.wsl = b.take(wcols * kHeadDim * 4, 16);           // W_H column slice, transposed
  s.enc = b.take((G + 1) * NW * 4, 16);               // this CTA's code bits
  s.qslot = b.take(CS * (G + 1) * NW * 4, 16);        // code bits from every CTA
  s.sel = b.take(sel_cap * 4, 16);                    // selected rows (fallback path)
  s.lg = b.take(G * s.gb * 4, 16);                    // logits / probabilities
  s.part = b.take(G * 4 * 4, 16);                     // running (max, sum, alpha) per head
  s.mslot = b.take(CS * (s.mcols + 2 * G) * 4, 16);   // partials for this CTA's output columns
  s.stat = b.take(16 * 4, 16);
  s.mbar = b.take((kMaxStages + 1) * 8, 8);  // ring stages + the row-gather barrier
  s.total = b.take(0, 128);
  return s;
}

enum { ST_T = 0, ST_M, ST_LESS_BEFORE, ST_EQ_BEFORE, ST_SPEC, ST_ABORT, ST_MYLESS, ST_MYEQ, ST_NBELOW };

template <typename T>
struct Vec16;  // 16-byte vector of T as fp32
template <>
struct Vec16<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      o[2 * j] = f.x;
      o[2 * j + 1] = f.y;
    }
  }
  __device__ __forceinline__ static void convert(const uint4& v, float (&o)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      o[2 * j] = f.x;
      o[2 * j + 1] = f.y;
    }
  }
};
template <>
struct Vec16<float> {
  __device__ __forceinline__ static void load(const float* p, float (&o)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x;
    o[1] = v.y;
    o[2] = v.z;
    o[3] = v.w;
  }
  __device__ __forceinline__ static void convert(const uint4& v, float (&o)[4]) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};

template <typename T, int NW, int G>
__global__ void __launch_bounds__(kFThreads, 1) fused_step_kernel(const FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int D = kHeadDim;
  constexpr int ESZ = (int)sizeof(T);
  constexpr int ST = kStageBytes / (4 * NW);      // tokens per ring stage
  constexpr int NV = G + 1;                       // encoded vectors: G queries + new key
  constexpr int BULK_Q = NW >= 4 ? 1 : 4 / NW;    // tokens per 16 bytes
  constexpr int XV = NV * D * ESZ / 16;           // 16-byte vectors of q + new key
  constexpr int QV = G * D * ESZ / 16;            // ... of which the queries
  constexpr int EPV = 16 / ESZ;                   // elements per 16-byte vector
  constexpr int LT = 16;                          // threads per row in the logits
  constexpr int LE = D / LT;                      // elements per thread in the logits (8)
  constexpr int PVG = kFThreads / (D / 2);        // row groups in P.V (8): thread = (column pair, row group)
  static_assert(XV <= kFThreads, "one vector of q / new key per thread");

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CS = (int)ptx::cluster_nctarank();
  const int rank = (int)ptx::cluster_ctarank();
  const int kStages = p.stages;
  const SmemLayout S = smem_layout(G, NW, ESZ, p.tok_cap, p.sel_cap, p.nbins, p.wcols, CS, kStages);
  const int GB = S.gb, nbp = S.nbp;
  unsigned char* ring = smem + S.ring;
  uint16_t* Ds = reinterpret_cast<uint16_t*>(smem + S.D);
  int* hist = reinterpret_cast<int*>(smem + S.hist);
  uint16_t* hslot = reinterpret_cast<uint16_t*>(smem + S.hslot);
  float* xs = reinterpret_cast<float*>(smem + S.xs);
  float* wsl = reinterpret_cast<float*>(smem + S.wsl);
  uint32_t* enc = reinterpret_cast<uint32_t*>(smem + S.enc);
  uint32_t* qslot = reinterpret_cast<uint32_t*>(smem + S.qslot);
  int* sel = reinterpret_cast<int*>(smem + S.sel);
  float* lg = reinterpret_cast<float*>(smem + S.lg);
  float* part = reinterpret_cast<float*>(smem + S.part);
  float* mslot = reinterpret_cast<float*>(smem + S.mslot);
  int* stat = reinterpret_cast<int*>(smem + S.stat);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + S.mbar);
  __shared__ int warp_sums[kNWarp];
  __shared__ int done[kMaxStages];
  __shared__ int cand[kMaxGB];
  __shared__ uint8_t candf[kMaxGB];
  __shared__ uint32_t qc[NV * NW];

  const int u = blockIdx.x / CS;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const bool early = (p.flags & HATA_FLAG_EARLY_PREFETCH) != 0;

  ptx::cluster_arrive_relaxed();  // completed by the wait before the first remote store
  if (!early) ptx::pdl_wait();
  ptx::pdl_launch_dependents();

  // ---- 1. first wave of loads: W_H slice, seq_lens; then the codes stream -----
  const int R = NW * 32;
  const int cpr = enc_cols_per_cta(R, CS);  // a multiple of 4: 16-byte aligned W_H slices
  const int j0 = rank * cpr;
  const int ncols = max(0, min(cpr, R - j0));  // the last ranks may get fewer (or no) columns
  const uint64_t pol_keep = ptx::policy_evict_last();
  const float* Wg = p.W + (size_t)g * D * R + j0;
  const int nc0 = min(p.wcols, ncols);  // a multiple of 4
  float4 wv[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = tid + q * kFThreads;
    wv[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e < D * nc0 / 4) wv[q] = ptx::ld_f4_policy(Wg + (size_t)(e / (nc0 / 4)) * R + (e % (nc0 / 4)) * 4, pol_keep);
  }
  // query vectors do not depend on L: load them now unless they may still be being written
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * D;
  uint4 xv = make_uint4(0u, 0u, 0u, 0u);
  if (!early && tid < QV) xv = reinterpret_cast<const uint4*>(qg)[tid];
  const int L = clamp_len(p.seq_lens, b, p.max_seq, p.status);
  int C = (L + CS - 1) / CS;
  C = (C + 15) & ~15;
  const int t0 = min(L, rank * C), t1 = min(L, t0 + C);
  const int nmine = t1 - t0;
  const int nst = (nmine + ST - 1) / ST;
  uint32_t* cu = p.codes + (size_t)u * p.max_seq * NW;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) ptx::mbar_init(&mbar[s], 1);
    ptx::mbar_init(&mbar[kMaxStages], 1);
    ptx::fence_mbarrier_init();
  }
  if (tid < kStages) done[tid] = 0;
  if (tid == 0) stat[ST_ABORT] = 0;
  __syncthreads();
  const uint64_t pol_stream = ptx::policy_evict_first();
  auto issue = [&](int s) {
    const int ts = t0 + s * ST, nt = min(ST, t1 - ts);
    const int nb = nt / BULK_Q * BULK_Q;  // tokens moved by the bulk copy (16-byte multiple)
    const uint32_t bytes = (uint32_t)nb * NW * 4;
    uint64_t* bar = &mbar[s % kStages];
    ptx::mbar_arrive_expect_tx(bar, bytes);
    if (bytes) ptx::bulk_g2s(ring + (s % kStages) * kStageBytes, cu + (size_t)ts * NW, bytes, bar, pol_stream);
  };
  if (tid == 0)
    for (int s = 0; s < min(nst, kStages); ++s) issue(s);

  // ---- 2. encode the G queries and the new key, this CTA's column slice --------
  if (early) {
    ptx::pdl_wait();  // q and the new key row come from the preceding kernel
    if (tid < QV) xv = reinterpret_cast<const uint4*>(qg)[tid];
  }
  {
    const T* kn = static_cast<const T*>(p.K) + (((size_t)u * p.max_seq) + (L > 0 ? L - 1 : 0)) * D;
    if (tid >= QV && tid < XV && L > 0) xv = reinterpret_cast<const uint4*>(kn)[tid - QV];
  }
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int e = tid + q * kFThreads;
    if (e < D * nc0 / 4) {
      const int i = e / (nc0 / 4), c4 = (e % (nc0 / 4)) * 4;
      wsl[(c4 + 0) * D + i] = wv[q].x;
      wsl[(c4 + 1) * D + i] = wv[q].y;
      wsl[(c4 + 2) * D + i] = wv[q].z;
      wsl[(c4 + 3) * D + i] = wv[q].w;
    }
  }
  if (tid < XV) {
    float xe[EPV];
    Vec16<T>::convert(xv, xe);
#pragma unroll
    for (int j = 0; j < EPV; ++j) xs[tid * EPV + j] = xe[j];
  }
  if (tid < NV * NW) enc[tid] = 0u;
  for (int v = tid; v < nbp; v += kFThreads) hist[v] = 0;
  for (int cb = 0; cb < ncols; cb += p.wcols) {
    const int nc = min(p.wcols, ncols - cb);
    if (cb > 0) {  // further column batches (small clusters): scalar staging
      __syncthreads();
      for (int e = tid; e < D * nc; e += kFThreads) {
        const int i = e / nc, c = e % nc;
        wsl[c * D + i] = __ldg(Wg + cb + (size_t)i * R + c);
      }
    }
    __syncthreads();
    // each warp takes up to 4 (vector, column) pairs at a time, interleaved
    for (int d0 = warp * 4; d0 < NV * nc; d0 += kNWarp * 4) {
      const int nd = min(4, NV * nc - d0);
      const float* xp[4];
      const float* wp[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int dj = d0 + min(j, nd - 1);
        xp[j] = xs + (dj / nc) * D;
        wp[j] = wsl + (dj % nc) * D;
      }
      float y[4];
      warp_dot128_multi<4>(xp, wp, lane, y);
      float yl = y[0];
#pragma unroll
      for (int j = 1; j < 4; ++j) yl = lane == j ? y[j] : yl;
      if (lane < nd && yl > 0.f) {  // lane j (< nd) publishes pair j's bit
        const int dj = d0 + lane, col = j0 + cb + dj % nc;
        atomicOr(&enc[(dj / nc) * NW + (col >> 5)], 1u << (col & 31));
      }
    }
  }
  __syncthreads();
  ptx::cluster_wait();  // every CTA of the cluster has started
  for (int e = tid; e < NV * NW * CS; e += kFThreads) {  // this CTA's bits into slot `rank` of every CTA
    const int w = e % (NV * NW), c = e / (NV * NW);
    ptx::st_dsmem_u32(ptx::dsmem_addr(&qslot[rank * NV * NW + w], c), enc[w]);
  }
  ptx::cluster_sync();  // #1: every CTA holds every CTA's code bits
  if (tid < NV * NW) {
    uint32_t acc = 0;
    for (int c = 0; c < CS; ++c) acc |= qslot[c * NV * NW + tid];
    qc[tid] = acc;
  }
  __syncthreads();
  if (rank == 0 && p.qcode_out && tid < G * NW) p.qcode_out[((size_t)b * p.Hq + (size_t)g * G) * NW + tid] = qc[tid];
  const bool own_last = L > 0 && t0 <= L - 1 && L - 1 < t1;
  if (own_last && tid < NW) cu[(size_t)(L - 1) * NW + tid] = qc[G * NW + tid];
  // ---- 3. scan: scores + histogram; each warp releases ring stages on its own ---
  {
    GroupQuery<NW, G> gq;
    gq.init(qc);
    uint32_t keyc[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) keyc[w] = qc[G * NW + w];
    // Each thread scores TPS tokens of a stage (all loads first, then the
    // arithmetic, for ILP).  Warps release stages on their own: lane 0 adds to the
    // stage's counter and checks the returned count one stage later, so no lane
    // waits on the atomic; the warp that completed a stage refills it.
    constexpr int TPS = ST / kFThreads;
    int rel_old = -1, rel_s = -1;  // lane 0: ticket of the previous stage's release
    for (int s = 0; s < nst; ++s) {
      if (!ptx::mbar_wait_spin(&mbar[s % kStages], (uint32_t)(s / kStages) & 1u, kWaitTries)) {
        set_status(p.status, HATA_ERR_TIMEOUT);
        stat[ST_ABORT] = 1;
      }
      const int ts = t0 + s * ST, nt = min(ST, t1 - ts);
      const int nb = nt / BULK_Q * BULK_Q;
      const uint32_t* buf = reinterpret_cast<const uint32_t*>(ring + (s % kStages) * kStageBytes);
      uint32_t kw[TPS][NW];
#pragma unroll
      for (int j = 0; j < TPS; ++j) {
        const int i = tid + j * kFThreads;
        if (i < nb) {
          if constexpr (NW >= 4) {
#pragma unroll
            for (int w4 = 0; w4 < NW / 4; ++w4) {
              const uint4 v4 = reinterpret_cast<const uint4*>(buf + (size_t)i * NW)[w4];
              kw[j][4 * w4] = v4.x;
              kw[j][4 * w4 + 1] = v4.y;
              kw[j][4 * w4 + 2] = v4.z;
              kw[j][4 * w4 + 3] = v4.w;
            }
          } else if constexpr (NW == 2) {
            const uint2 v2 = reinterpret_cast<const uint2*>(buf + (size_t)i * NW)[0];
            kw[j][0] = v2.x;
            kw[j][1] = v2.y;
          } else {
            kw[j][0] = buf[i];
          }
        } else if (i < nt) {
#pragma unroll
          for (int w = 0; w < NW; ++w) kw[j][w] = cu[(size_t)(ts + i) * NW + w];
        }
      }
#pragma unroll
      for (int j = 0; j < TPS; ++j) {
        const int i = tid + j * kFThreads;
        if (i < nt) {
          const int dv = gq.score(kw[j], qc, G);  // <= G * r by construction
          Ds[ts + i - t0] = (uint16_t)dv;
          atomicAdd(&hist[dv], 1);
        }
      }
      __syncwarp();
      if (lane == 0) {
        // counters never reset: the k-th use of buffer s % kStages ends at count k * kNWarp
        if (rel_s >= 0 && rel_old == ((rel_s / kStages) + 1) * kNWarp - 1 && rel_s + kStages < nst) {
          ptx::fence_proxy_async_smem();
          issue(rel_s + kStages);
        }
        rel_old = atomicAdd(&done[s % kStages], 1);
        rel_s = s;
      }
    }
    __syncthreads();
    // the ring (or global memory) may have held the old code of slot L - 1: rescore it
    // with the appended key code and move its histogram count
    if (own_last && tid == 0) {
      const int d_new = gq.score(keyc, qc, G), d_old = Ds[L - 1 - t0];
      if (d_new != d_old) {
        Ds[L - 1 - t0] = (uint16_t)d_new;
        hist[d_old] -= 1;
        hist[d_new] += 1;
      }
    }
  }
  __syncthreads();

  // ---- 4. cumulative histogram -> every CTA; local guess; speculative gather ---
  const int n = min(p.k, L);
  {
    // inclusive cumulative counts in place (each thread a contiguous span of bins)
    const int span = (nbp + kFThreads - 1) / kFThreads;
    const int v0 = min(nbp, tid * span), v1 = min(nbp, v0 + span);
    int local = 0;
    for (int v = v0; v < v1; ++v) local += hist[v];
    int total;
    int run = block_exclusive_scan<kFThreads>(local, warp_sums, &total);
    // guess: enough local rows for about 1.5x this CTA's fair share of the budget
    const int want = min(nmine, min(GB, 5 * ((n + CS - 1) / CS) / 4 + 8));
    if (tid == 0) stat[ST_SPEC] = want > 0 ? INT_MAX : -1;
    __syncthreads();
    for (int v = v0; v < v1; ++v) {
      const int before = run;
      run += hist[v];
      hist[v] = run;
      if (want > 0 && before < want && run >= want) stat[ST_SPEC] = v;
    }
  }
  __syncthreads();
  // u16 cumulative histogram into slot `rank` of every CTA (8 bins per 16-byte store)
  for (int e = tid; e < (nbp / 8) * CS; e += kFThreads) {
    const int v8 = e % (nbp / 8), c = e / (nbp / 8);
    uint4 pk;
    const int* h = hist + v8 * 8;
    pk.x = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
    pk.y = (uint32_t)h[2] | ((uint32_t)h[3] << 16);
    pk.z = (uint32_t)h[4] | ((uint32_t)h[5] << 16);
    pk.w = (uint32_t)h[6] | ((uint32_t)h[7] << 16);
    ptx::st_dsmem_v4(ptx::dsmem_addr(&hslot[rank * nbp + v8 * 8], c), pk);
  }
  const int Tspec = stat[ST_SPEC];

  const T* Kb = static_cast<const T*>(p.K) + (size_t)u * p.max_seq * D;
  const T* Vb = static_cast<const T*>(p.V) + (size_t)u * p.max_seq * D;
  T* Kr = reinterpret_cast<T*>(ring);
  T* Vr = reinterpret_cast<T*>(ring) + (size_t)GB * D;
  // Row gathers: one bulk copy per K row and per V row, all completing on the
  // gather mbarrier (one phase per gather).  An index outside this CTA's slice
  // (never expected) is flagged and replaced by row t0, so the byte count holds.
  uint64_t* gbar = &mbar[kMaxStages];
  uint32_t gphase = 0;
  const uint64_t pol_rows = ptx::policy_evict_first();
  auto gather = [&](const int* list, int nr) {
    if (tid == 0) ptx::mbar_arrive_expect_tx(gbar, (uint32_t)(2 * nr * D * ESZ));
    for (int e = tid; e < 2 * nr; e += kFThreads) {
      const int r = e >> 1;
      int t = list[r];
      if (t < t0 || t >= t1) {
        set_status(p.status, HATA_ERR_INVALID_ARG);
        t = t0;
      }
      if (e & 1) ptx::bulk_g2s(Vr + (size_t)r * D, Vb + (size_t)t * D, D * ESZ, gbar, pol_rows);
      else ptx::bulk_g2s(Kr + (size_t)r * D, Kb + (size_t)t * D, D * ESZ, gbar, pol_rows);
    }
  };
  auto gather_wait = [&]() {
    if (!ptx::mbar_wait_spin(gbar, gphase & 1u, kWaitTries)) {
      set_status(p.status, HATA_ERR_TIMEOUT);
      stat[ST_ABORT] = 1;
    }
    ++gphase;
  };
  // Passes over this CTA's scores go 8192 at a time: each thread owns 16
  // consecutive scores of the pass (two 16-byte loads); scores past nmine read as 0xffff.
  constexpr int TPT = 16, CHUNK = kFThreads * TPT;
  auto load16 = [&](int base, uint16_t (&dv)[TPT]) {
    const int a = base + tid * TPT;  // a multiple of 16; a < nmine <= tok_cap keeps both loads in the array
    uint4 v0 = make_uint4(0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu), v1 = v0;
    if (a < nmine) {
      v0 = reinterpret_cast<const uint4*>(Ds + a)[0];
      v1 = reinterpret_cast<const uint4*>(Ds + a)[1];
    }
    const uint16_t* h0 = reinterpret_cast<const uint16_t*>(&v0);
    const uint16_t* h1 = reinterpret_cast<const uint16_t*>(&v1);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      dv[i] = a + i < nmine ? h0[i] : (uint16_t)0xffffu;
      dv[8 + i] = a + 8 + i < nmine ? h1[i] : (uint16_t)0xffffu;
    }
  };
  int ncand = 0;
  for (int base = 0; base < nmine && Tspec >= 0; base += CHUNK) {
    uint16_t dv[TPT];
    load16(base, dv);
    int mine = 0;
#pragma unroll
    for (int i = 0; i < TPT; ++i) mine += (int)dv[i] <= Tspec;
    int tot;
    int pos = ncand + block_exclusive_scan<kFThreads>(mine, warp_sums, &tot);
#pragma unroll
    for (int i = 0; i < TPT; ++i)
      if ((int)dv[i] <= Tspec) {
        if (pos < GB) cand[pos] = t0 + base + tid * TPT + i;
        ++pos;
      }
    ncand += tot;
  }
  const bool truncated = ncand > GB;
  ncand = min(ncand, GB);
  if (stat[ST_ABORT]) ncand = 0;  // a bulk copy never completed: the ring may still be written
  __syncthreads();
  gather(cand, ncand);  // speculative: waited for in section 8

  // ---- 5. unit threshold from the CS cumulative histograms -------------------
  ptx::cluster_sync();  // #2: every CTA holds every CTA's cumulative histogram
  {
    // unit totals, one bin per thread; T = number of bins whose cumulative total is below n
    int below = 0;
    for (int v = tid; v < nbp; v += kFThreads) {
      int cv[kMaxCS];
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) cv[c] = c < CS ? (int)hslot[c * nbp + v] : 0;
      int tv = 0;
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) tv += cv[c];
      hist[v] = tv;  // the local counts are no longer needed (this CTA's are in hslot[rank])
      below += (v < p.nbins && tv < n);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
    if (lane == 0) warp_sums[warp] = below;
    __syncthreads();
    if (warp == 0) {
      int Tth = lane < kNWarp ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 16; o; o >>= 1) Tth += __shfl_xor_sync(0xffffffffu, Tth, o);
      const int Tc = min(Tth, p.nbins - 1);
      // per source CTA (lane c): cumulative count below T and at T
      int cb = 0, ce = 0;
      if (lane < CS) {
        cb = Tc > 0 ? (int)hslot[lane * nbp + Tc - 1] : 0;
        ce = (int)hslot[lane * nbp + Tc] - cb;
      }
      const int lb = __reduce_add_sync(0xffffffffu, lane < rank ? cb : 0);
      const int eb = __reduce_add_sync(0xffffffffu, lane < rank ? ce : 0);
      const int myl = __shfl_sync(0xffffffffu, cb, rank);
      const int mye = __shfl_sync(0xffffffffu, ce, rank);
      if (lane == 0) {
        stat[ST_T] = n == 0 ? 0 : Tth;
        stat[ST_M] = n == 0 ? 0 : n - (Tc > 0 ? hist[Tc - 1] : 0);
        stat[ST_LESS_BEFORE] = lb;
        stat[ST_EQ_BEFORE] = eb;
        stat[ST_MYLESS] = myl;
        stat[ST_MYEQ] = mye;
      }
    }
    __syncthreads();
  }
  const int Tt = stat[ST_T], m = stat[ST_M];
  const int less_before = stat[ST_LESS_BEFORE], eq_before = stat[ST_EQ_BEFORE];
  const int sel_before = less_before + min(eq_before, m);
  const int ties_here = max(0, min(m - eq_before, stat[ST_MYEQ]));
  const int nsel_here = stat[ST_MYLESS] + ties_here;  // this CTA's share of the selection
  // the candidates cover the selection when every selected score is <= Tspec and none was cut off
  const bool covered = nsel_here == 0 || (!truncated && Tt <= Tspec);

  // ---- 7. ascending indices (only when asked for) and the row list --------------
  int32_t* ix = p.idx_out ? p.idx_out + (size_t)u * p.k : nullptr;
  if (ix || !covered) {
    // one packed scan per pass: low half counts scores < T, high half scores == T
    int lp_carry = 0, ep_carry = 0;
    const int took_before = min(m, eq_before);
    for (int base = 0; base < nmine; base += CHUNK) {
      uint16_t dv16[TPT];
      load16(base, dv16);
      int lt = 0, eq = 0;
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        lt += (int)dv16[i] < Tt;
        eq += (int)dv16[i] == Tt;
      }
      int tot;
      const int pre = block_exclusive_scan<kFThreads>(lt | (eq << 16), warp_sums, &tot);
      int lp = lp_carry + (pre & 0xffff), ep = ep_carry + (pre >> 16);
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        const int dv = dv16[i];
        const bool s_ = dv < Tt || (dv == Tt && eq_before + ep < m);
        if (s_) {
          const int pos = lp + min(m, eq_before + ep) - took_before;  // rank among this CTA's selected
          const int t = t0 + base + tid * TPT + i;
          if (ix && sel_before + pos < n) ix[sel_before + pos] = t;
          if (!covered && pos < p.sel_cap) sel[pos] = t;
        }
        lp += dv < Tt;
        ep += dv == Tt;
      }
      lp_carry += tot & 0xffff;
      ep_carry += tot >> 16;
    }
    if (ix && rank == 0)
      for (int j = n + tid; j < p.k; j += kFThreads) ix[j] = -1;
  }
  // selection flags of the candidates (covered case): every tie of this CTA is a
  // candidate, in index order, so a tie's rank is eq_before + ties among earlier candidates
  if (covered && warp == 0) {
    int run = eq_before;
    for (int r0 = 0; r0 < ncand; r0 += 32) {
      const int r = r0 + lane;
      const int dv = r < ncand ? (int)Ds[cand[r] - t0] : INT_MAX;
      const bool is_eq = dv == Tt;
      const unsigned eqm = __ballot_sync(0xffffffffu, is_eq);
      const int rk = run + __popc(eqm & ((1u << lane) - 1u));
      if (r < ncand) candf[r] = (uint8_t)(dv < Tt || (is_eq && rk < m));
      run += __popc(eqm);
    }
  }

  // ---- 8. attention partials over this CTA's selected rows -----------------------
  constexpr int OPT = (G * D + kFThreads - 1) / kFThreads;  // output elements per thread
  float oacc[OPT];
#pragma unroll
  for (int q = 0; q < OPT; ++q) oacc[q] = 0.f;
  if (tid < G) {
    part[tid * 4] = -INFINITY;
    part[tid * 4 + 1] = 0.f;
  }
  const int nrows_total = covered ? ncand : (stat[ST_ABORT] ? 0 : min(nsel_here, p.sel_cap));
  gather_wait();  // the speculative rows (they were issued before the threshold was known)
  for (int r0 = 0; r0 < nrows_total; r0 += GB) {
    const int nr = min(GB, nrows_total - r0);
    if (!covered) {  // the guess missed: gather the selected rows batch by batch
      __syncthreads();  // previous batch's readers are done with the buffers
      gather(sel + r0, nr);
      gather_wait();
    }
    __syncthreads();
    // logits (exp2 domain): 16 threads per row, 8 elements each, every head at once;
    // each thread keeps its 8-element slice of the G query vectors in registers
    {
      const int sgi = lane % LT;
      float xq[G][LE];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 a = reinterpret_cast<const float4*>(xs + h * D + sgi * LE)[0];
        const float4 c = reinterpret_cast<const float4*>(xs + h * D + sgi * LE)[1];
        xq[h][0] = a.x; xq[h][1] = a.y; xq[h][2] = a.z; xq[h][3] = a.w;
        xq[h][4] = c.x; xq[h][5] = c.y; xq[h][6] = c.z; xq[h][7] = c.w;
      }
      for (int rb = warp * (32 / LT); rb < nr; rb += kFThreads / LT) {  // warp-uniform trip count
        const int r = rb + lane / LT;
        const bool valid = r < nr;
        float kv[LE];
#pragma unroll
        for (int j = 0; j < LE; ++j) kv[j] = 0.f;
        if (valid) {
#pragma unroll
          for (int v = 0; v < LE / EPV; ++v) {
            float t8[EPV];
            Vec16<T>::load(Kr + (size_t)r * D + sgi * LE + v * EPV, t8);
#pragma unroll
            for (int j = 0; j < EPV; ++j) kv[v * EPV + j] = t8[j];
          }
        }
        float acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = xq[h][0] * kv[0];
#pragma unroll
          for (int j = 1; j < LE; ++j) a = fmaf(xq[h][j], kv[j], a);
          acc[h] = a;
        }
#pragma unroll
        for (int o = 1; o < LT; o <<= 1)
#pragma unroll
          for (int h = 0; h < G; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
        if (valid && sgi == 0) {
          const bool use = !covered || candf[r];
#pragma unroll
          for (int h = 0; h < G; ++h) lg[h * GB + r] = use ? acc[h] * p.scale_log2 : -INFINITY;
        }
      }
    }
    __syncthreads();
    for (int h = warp; h < G; h += kNWarp) {
      float mx = -INFINITY;
      for (int r = lane; r < nr; r += 32) mx = fmaxf(mx, lg[h * GB + r]);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = part[h * 4];
      const float m_new = fmaxf(m_old, mx);
      float ssum = 0.f;
      for (int r = lane; r < nr; r += 32) {
        const float lv = lg[h * GB + r];
        const float pr_ = lv == -INFINITY ? 0.f : exp2f(lv - m_new);
        lg[h * GB + r] = pr_;
        ssum += pr_;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
      __syncwarp();
      if (lane == 0) {
        const float alpha = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
        part[h * 4] = m_new;
        part[h * 4 + 1] = part[h * 4 + 1] * alpha + ssum;
        part[h * 4 + 2] = alpha;
      }
    }
    __syncthreads();
    // P.V: thread (column pair cp, row group rg) sums rows rg, rg + PVG, ... for every head,
    // then the PVG partial sums of each output go through shared memory (the K rows'
    // buffer, free once the logits are done)
    {
      const int cp = tid % (D / 2), rg = tid / (D / 2);
      float pacc[G][2];
#pragma unroll
      for (int h = 0; h < G; ++h) pacc[h][0] = pacc[h][1] = 0.f;
      for (int r = rg; r < nr; r += PVG) {
        float v0, v1;
        if constexpr (ESZ == 2) {
          const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Vr + (size_t)r * D)[cp]);
          v0 = f.x;
          v1 = f.y;
        } else {
          const float2 f = reinterpret_cast<const float2*>(Vr + (size_t)r * D)[cp];
          v0 = f.x;
          v1 = f.y;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pr_ = lg[h * GB + r];
          pacc[h][0] = fmaf(pr_, v0, pacc[h][0]);
          pacc[h][1] = fmaf(pr_, v1, pacc[h][1]);
        }
      }
      float* red = reinterpret_cast<float*>(Kr);  // [PVG][G][D]
#pragma unroll
      for (int h = 0; h < G; ++h)
        reinterpret_cast<float2*>(red + ((size_t)rg * G + h) * D)[cp] = make_float2(pacc[h][0], pacc[h][1]);
      __syncthreads();
#pragma unroll
      for (int q = 0; q < OPT; ++q) {
        const int e = tid + q * kFThreads;
        if (e < G * D) {
          const int h = e / D, i = e % D;
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < PVG; ++j) sum += red[((size_t)j * G + h) * D + i];
          oacc[q] = fmaf(oacc[q], part[h * 4 + 2], sum);
        }
      }
    }
  }
  __syncthreads();

  // ---- 9. partials to the CTAs owning each output column, then merge ----------
  // mslot layout in the owner: [source rank][ (max, sum) x G, then its mcols columns ]
  const int mc = S.mcols, stride = mc + 2 * G;
#pragma unroll
  for (int q = 0; q < OPT; ++q) {
    const int e = tid + q * kFThreads;
    if (e < G * D) {
      const int owner = e / mc, col = e % mc;
      ptx::st_dsmem_f32(ptx::dsmem_addr(&mslot[rank * stride + 2 * G + col], owner), oacc[q]);
    }
  }
  for (int e = tid; e < 2 * G * CS; e += kFThreads) {
    const int owner = e / (2 * G), w = e % (2 * G);
    ptx::st_dsmem_f32(ptx::dsmem_addr(&mslot[rank * stride + w], owner), part[(w >> 1) * 4 + (w & 1)]);
  }
  ptx::cluster_sync();  // #4: every CTA holds the partials of its columns
  for (int col = tid; col < mc; col += kFThreads) {
    const int e = rank * mc + col;
    if (e < G * D) {
      const int h = e / D, i = e % D;
      float M = -INFINITY;
      for (int c = 0; c < CS; ++c) M = fmaxf(M, mslot[c * stride + 2 * h]);
      float l = 0.f, o = 0.f;
      if (M != -INFINITY)
        for (int c = 0; c < CS; ++c) {
          const float mcv = mslot[c * stride + 2 * h];
          if (mcv == -INFINITY) continue;
          const float w = exp2f(mcv - M);
          l = fmaf(mslot[c * stride + 2 * h + 1], w, l);
          o = fmaf(mslot[c * stride + 2 * G + col], w, o);
        }
      static_cast<T*>(p.out)[((size_t)b * p.Hq + (size_t)g * G + h) * D + i] = from_f32<T>(l > 0.f ? o / l : 0.f);
    }
  }
  if (stat[ST_ABORT] && tid == 0) {
    // give outstanding bulk copies one more bounded chance to land before exit
    for (int s = 0; s < min(nst, kStages); ++s) {
      const int last = nst - 1 - ((nst - 1 - s) % kStages);
      ptx::mbar_wait_bounded(&mbar[s], (uint32_t)(last / kStages) & 1u, kWaitTries);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct Plan {
  bool ok;
  int CS, tok_cap, sel_cap, nbins, wcols, stages;
  size_t smem;
};

// Clusters of CS CTAs that can be resident at once (one CTA per SM), cached per
// (kernel, device, CS, shared memory).
int max_active_clusters(const void* kern, int CS, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, int, size_t>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(kern, dev, CS, smem);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)CS, 1, 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = n;
  return n;
}

// Allow the largest dynamic shared memory and 16-CTA clusters, once per kernel
// and device (attributes only ever grow, so any planned launch fits).
cudaError_t configure_kernel(const void* kern) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, cudaError_t> done_;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = done_.find({kern, dev});
  if (it != done_.end()) return it->second;
  int optin = 0;
  cudaFuncAttributes fa;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) (void)cudaGetLastError();
  done_[{kern, dev}] = e;
  return e;
}

// Cluster size: a single wave of clusters when possible (largest CS that fits
// every unit at once), otherwise the size with the smallest estimated time
// (waves x (fixed latency + scan + gather of one CTA's share)).
template <typename T, int NW, int G>
Plan make_plan_t(const hata_dims_t& d, int k) {
  Plan best{};
  const void* kern = (const void*)fused_step_kernel<T, NW, G>;
  const int R = NW * 32, esize = (int)sizeof(T);
  const long long units = (long long)d.batch * d.n_kv_heads;
  static const int cands[] = {16, 15, 14, 12, 10, 8, 6, 4, 3, 2, 1};
  double best_t = 1e30;
  for (int CS : cands) {
    const int tok_cap = ((d.max_seq + CS - 1) / CS + 15) / 16 * 16;
    if (tok_cap > kTokCap) continue;
    Plan pl{};
    pl.CS = CS;
    pl.tok_cap = tok_cap;
    pl.sel_cap = std::min(k, tok_cap);
    pl.nbins = G * d.hash_bits + 1;
    pl.wcols = std::min(kWCols, enc_cols_per_cta(R, CS));
    pl.stages = 0;
    for (int st = kMaxStages; st >= kMinStages; --st) {
      const size_t sm = smem_layout(G, NW, esize, tok_cap, pl.sel_cap, pl.nbins, pl.wcols, CS, st).total;
      if (sm + 2048 <= 227 * 1024) {  // + static shared memory
        pl.stages = st;
        pl.smem = std::max<size_t>(sm, kOneCtaSmem);
        break;
      }
    }
    if (!pl.stages) continue;
    if (configure_kernel(kern) != cudaSuccess) return best;
    const int active = max_active_clusters(kern, CS, pl.smem);
    if (active < 1) continue;
    const long long waves = (units + active - 1) / active;
    const double rows = std::min<double>(k, tok_cap) * (CS > 1 ? 1.0 / CS * 1.5 : 1.0);
    const double t = (double)waves * (4.0 + tok_cap * (R / 8.0) / 45e3 + rows * 2.0 * kHeadDim * esize / 30e3);
    if (waves == 1) {  // largest single-wave cluster wins outright
      pl.ok = true;
      return pl;
    }
    if (t < best_t) {
      best_t = t;
      best = pl;
      best.ok = true;
    }
  }
  return best;
}

template <typename T, int NW, int G>
cudaError_t launch_fused_t(const Plan& pl, const hata_dims_t& d, const FusedParams& prm, cudaStream_t st) {
  auto kern = fused_step_kernel<T, NW, G>;
  const cudaError_t ce = configure_kernel((const void*)kern);
  if (ce != cudaSuccess) return ce;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(d.batch * d.n_kv_heads * pl.CS), 1, 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = pl.CS;
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

// Typed dispatch: fn<T, NW, G>(args...) for the runtime type, code words and group size.
template <template <typename, int, int> class F, typename... A>
auto dispatch(const hata_dims_t& d, A&&... a) -> decltype(F<float, 1, 1>::run(a...)) {
  const int G = d.n_q_heads / d.n_kv_heads, NW = d.hash_bits / 32;
#define HATA_G(T, NW_)                                            \
  switch (G) {                                                    \
    case 1: return F<T, NW_, 1>::run(a...);                       \
    case 2: return F<T, NW_, 2>::run(a...);                       \
    case 4: return F<T, NW_, 4>::run(a...);                       \
    case 8: return F<T, NW_, 8>::run(a...);                       \
  }                                                               \
  break;
#define HATA_NW(T)                     \
  switch (NW) {                        \
    case 1: HATA_G(T, 1)               \
    case 2: HATA_G(T, 2)               \
    case 4: HATA_G(T, 4)               \
    case 8: HATA_G(T, 8)               \
  }
  if (d.dtype == HATA_BF16) {
    HATA_NW(__nv_bfloat16)
  } else {
    HATA_NW(float)
  }
#undef HATA_NW
#undef HATA_G
  return F<float, 1, 1>::fail();
}

template <typename T, int NW, int G>
struct PlanFn {
  static Plan run(const hata_dims_t& d, int k) { return make_plan_t<T, NW, G>(d, k); }
  static Plan fail() { return Plan{}; }
};

template <typename T, int NW, int G>
struct LaunchFn {
  static cudaError_t run(const Plan& pl, const hata_dims_t& d, const FusedParams& prm, cudaStream_t st) {
    return launch_fused_t<T, NW, G>(pl, d, prm, st);
  }
  static cudaError_t fail() { return cudaErrorNotSupported; }
};

Plan make_plan_uncached(const hata_dims_t& d, int k) {
  const int G = d.n_q_heads / d.n_kv_heads, NW = d.hash_bits / 32;
  if (G != 1 && G != 2 && G != 4 && G != 8) return Plan{};
  if ((long long)d.max_seq * NW % 4 != 0) return Plan{};  // 16-byte aligned per-unit code slabs
  if ((long long)d.batch * d.n_kv_heads * 16 > 0x7fffffffLL) return Plan{};
  return dispatch<PlanFn>(d, d, k);
}

// Plans are cached per (device, shape, budget): the first call for a shape sets
// kernel attributes and queries cluster occupancy; later calls (including ones
// made while a stream is being captured into a CUDA graph) only look it up.
Plan make_plan(const hata_dims_t& d, int k) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int, int, int, int>, Plan> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(dev, d.batch, d.n_q_heads, d.n_kv_heads, d.head_dim, d.hash_bits, d.max_seq,
                                   d.dtype, k);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const Plan pl = make_plan_uncached(d, k);
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = pl;
  return pl;
}

}  // namespace

bool fused_step_applies(const hata_dims_t& d, int k) { return make_plan(d, k).ok; }

size_t fused_step_ws_bytes(const hata_dims_t&, int) { return 0; }

cudaError_t launch_fused_step(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K, const void* V,
                              const float* W, uint32_t* codes, const int32_t* seq_lens, int k, float scale,
                              void* out, uint32_t* qcode_out, int32_t* idx_out, char* ws, cudaStream_t st) {
  const Plan pl = make_plan(d, k);
  if (!pl.ok) return cudaErrorNotSupported;
  FusedParams prm;
  prm.q = q;
  prm.K = K;
  prm.V = V;
  prm.W = W;
  prm.codes = codes;
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.qcode_out = qcode_out;
  prm.idx_out = idx_out;
  prm.status = reinterpret_cast<uint32_t*>(ws + L.status);
  prm.Hq = d.n_q_heads;
  prm.Hkv = d.n_kv_heads;
  prm.max_seq = d.max_seq;
  prm.k = k;
  prm.nbins = pl.nbins;
  prm.tok_cap = pl.tok_cap;
  prm.sel_cap = pl.sel_cap;
  prm.wcols = pl.wcols;
  prm.flags = d.flags;
  prm.stages = pl.stages;
  prm.scale_log2 = scale * 1.4426950408889634f;
  return dispatch<LaunchFn>(d, pl, d, prm, st);
}

}  // namespace hata
