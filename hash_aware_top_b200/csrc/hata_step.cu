// Fused HATA decode step: one kernel, one thread-block cluster per
// (batch, KV head) unit ("HATA" paper notes, Decode 阶段算法 end to end, with the
// fusions of 硬件高效优化).
//
// A unit's L cached tokens are split evenly over the CS CTAs of its cluster.
// Each CTA:
//   1. streams its slice of the code cache into a shared-memory ring with bulk
//      (TMA) copies, evict-first in L2, issued as soon as L is known, and copies
//      the KV head's W_H (bulk, kept in L2) into shared memory;
//   2. encodes the G queries and the new key over all r columns itself (the
//      arithmetic of warp_dot128, so the codes equal hata_encode_append's decode
//      form bit for bit; no exchange between CTAs); the CTA owning slot L - 1
//      appends the key code to the cache;
//   3. scores every token of its slice (xor + popc with the GQA sum folded into
//      per-word constants and a carry-save popc sum), keeping the u16 scores and
//      their histogram in shared memory; warps release ring stages on their own;
//   4. turns the histogram into a cumulative one and stores the bins the others
//      can need (u16) into its slot of every CTA; takes as candidates, in token
//      order, every token scoring at most Tc (the largest score whose count fits
//      about 1.5x its fair share of the selection), gathers their K/V rows with
//      cp.async and computes their logits while the cluster barrier completes;
//   5. one warp sums the CS cumulative histograms to find the unit's threshold T
//      (the smallest score with at least n = min(k, L) tokens at or below it), the
//      tie quota m and the counts of earlier CTAs, so ties go to the lower token
//      index exactly as in a global sort, and marks the selected candidates;
//   6. computes the flash-decode partial (max, sum, weighted V) of each of the G
//      query heads over its selected rows (falling back to gathering them when
//      T > Tc), and stores each partial's column slice into the CTA that owns
//      those output columns; after a last cluster barrier every CTA merges its
//      columns (log-sum-exp) and writes them.
// Cross-CTA traffic is only stores into other CTAs' shared memory before a
// hardware cluster barrier: no remote loads, no global-memory flags, no
// workspace.  The only waits are bounded mbarrier waits on this CTA's own
// copies.
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
static_assert(256 < kFThreads, "candidate passes give each candidate its own thread");
constexpr int kMaxStages = 6;        // ring stages (32 KB each), 2..6 depending on shared memory left
constexpr int kMinStages = 2;
constexpr int kStageBytes = 32768;
constexpr int kTokCap = 65520;       // max tokens per CTA: u16 scores and u16 cumulative counts
constexpr int kXS = 36;              // floats per residue row of an encoded vector (32 used, padded)
constexpr int kMaxCS = 16;           // largest cluster
constexpr int kPagedBt = 256;        // block-table entries of a CTA's slice kept in shared memory (paged cache)
constexpr int kMaxGB = 256;          // largest gather batch (rows); below kFThreads: one candidate per thread
constexpr int kOneCtaSmem = 116 * 1024;  // dynamic shared memory that keeps one CTA per SM
constexpr uint32_t kWaitTries = 1u << 22;

struct SmemLayout {
  uint32_t ring, W, D, hist, hslot, xr, xp, sel, lg, part, mslot, stat, mbar, total;
  int nbp, mcols, gb;
};

struct FusedParams {
  const void* q;
  const void* K;
  const void* V;
  const float* W;
  const float* Wk;  // separate key encoder [Hkv][d][r] (HashAttention form), or null: W encodes keys too
  uint32_t* codes;
  const int32_t* seq_lens;
  void* out;
  uint32_t* qcode_out;
  int32_t* idx_out;
  uint32_t* status;
  int Hq, Hkv, max_seq, k, nbins, tok_cap, sel_cap, flags, stages;
  float scale_log2;
  SmemLayout lay;  // shared-memory layout of the launch (computed on the host)
  // paged cache (K, V and codes are pools of blocks [n_blocks][Hkv][1 << block_shift][...])
  const int32_t* block_table;  // [B][max_blocks] physical block of each logical block
  int block_shift, n_blocks, max_blocks;
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

// Output columns merged by each CTA of a cluster of CS (the last one may have fewer).
__host__ __device__ inline int merge_cols(int G, int CS) { return (G * kHeadDim + CS - 1) / CS; }

__host__ __device__ inline SmemLayout smem_layout(int G, int NW, int esize, int tok_cap, int sel_cap, int nbins,
                                                  int CS, int stages) {
  SmemLayout s;
  Bump b;
  s.nbp = (nbins + 7) / 8 * 8;  // histogram bins padded to whole 16-byte groups of u16
  s.mcols = merge_cols(G, CS);
  s.gb = stages * kStageBytes / (2 * kHeadDim * esize);
  if (s.gb > kMaxGB) s.gb = kMaxGB;
  s.ring = b.take(stages * kStageBytes, 128);
  s.W = b.take(kHeadDim * NW * 32 * 4, 128);        // W_H of the unit's KV head, fp32
  s.D = b.take(max(tok_cap * 2, (G + 1) * 4 * NW * 32 * 4), 16);  // scores; first the encode's residue sums
  s.hist = b.take((s.nbp + kFThreads - 1) / kFThreads * kFThreads * 4, 16);  // counts, then cumulative (padded)
  s.hslot = b.take(CS * s.nbp * 2, 16);               // u16 cumulative histograms from every CTA
  s.xr = b.take((G + 1) * 4 * kXS * 4, 16);           // G queries + new key, fp32, residue-major
  s.xp = b.take(G * kHeadDim * 4, 16);                // G queries, fp32
  s.sel = b.take(sel_cap * 4, 16);                    // selected rows (fallback path)
  s.lg = b.take(G * s.gb * 4, 16);                    // logits / probabilities
  s.part = b.take(G * 4 * 4, 16);                     // running (max, sum, alpha) per head
  s.mslot = b.take(CS * (s.mcols + 2 * G) * 4, 16);   // partials for this CTA's output columns
  s.stat = b.take(16 * 4, 16);
  s.mbar = b.take((kMaxStages + 2) * 8, 8);  // ring stages, the row gathers, W_H
  s.total = b.take(0, 128);
  return s;
}

// Order-preserving map of a float (not NaN) to an int, for integer atomicMax.
__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float float_of_ord(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

enum { ST_T = 0, ST_M, ST_LESS_BEFORE, ST_EQ_BEFORE, ST_SPEC, ST_ABORT, ST_MYLESS, ST_MYEQ, ST_LO, ST_HI };

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

template <typename T, int NW, int G, bool PAGED>
__global__ void __launch_bounds__(kFThreads, 1) fused_step_kernel(const FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int D = kHeadDim;
  constexpr int ESZ = (int)sizeof(T);
  constexpr int R = NW * 32;                      // hash bits
  constexpr int ST = kStageBytes / (4 * NW);      // tokens per ring stage
  constexpr int NV = G + 1;                       // encoded vectors: G queries + new key
  constexpr int BULK_Q = NW >= 4 ? 1 : 4 / NW;    // tokens per 16 bytes
  constexpr int XV = NV * D * ESZ / 16;           // 16-byte vectors of q + new key
  constexpr int QV = G * D * ESZ / 16;            // ... of which the queries
  constexpr int EPV = 16 / ESZ;                   // elements per 16-byte vector
  constexpr int RPR = D * ESZ / 16;               // 16-byte pieces per K or V row
  static_assert((2 * RPR) % 32 == 0, "a candidate's K and V pieces fill whole warps");
  constexpr int LT = 16;                          // threads per row in the logits
  constexpr int LE = D / LT;                      // elements per thread in the logits (8)
  constexpr int PVG = kFThreads / (D / 2);        // row groups in P.V (8): thread = (column pair, row group)
  constexpr int NBP = (G * R + 1 + 7) / 8 * 8;    // histogram bins padded to whole 8-bin groups
  constexpr int BPT = (NBP + kFThreads - 1) / kFThreads;  // bins per thread in the cumulative sum
  static_assert(XV <= kFThreads, "one vector of q / new key per thread");

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CS = (int)ptx::cluster_nctarank();
  const int rank = (int)ptx::cluster_ctarank();
  const int kStages = p.stages;
  const SmemLayout& S = p.lay;
  const int GB = S.gb;
  unsigned char* ring = smem + S.ring;
  uint16_t* Ds = reinterpret_cast<uint16_t*>(smem + S.D);
  int* hist = reinterpret_cast<int*>(smem + S.hist);
  uint16_t* hslot = reinterpret_cast<uint16_t*>(smem + S.hslot);
  float* xr = reinterpret_cast<float*>(smem + S.xr);
  float* xp = reinterpret_cast<float*>(smem + S.xp);
  int* sel = reinterpret_cast<int*>(smem + S.sel);
  float* lg = reinterpret_cast<float*>(smem + S.lg);
  float* part = reinterpret_cast<float*>(smem + S.part);
  float* mslot = reinterpret_cast<float*>(smem + S.mslot);
  int* stat = reinterpret_cast<int*>(smem + S.stat);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + S.mbar);
  uint64_t* gbar = &mbar[kMaxStages];  // completion of the row gathers (cp.async)
  __shared__ int warp_sums[kNWarp];
  __shared__ int done[kMaxStages];
  __shared__ int lastv[kMaxStages];       // last stage issued into each ring buffer
  __shared__ __align__(16) int cand[kMaxGB];  // candidate token indices, ascending
  __shared__ uint16_t rowl[kMaxGB];       // slots of the selected candidates, ascending token index
  __shared__ __align__(16) uint32_t qc[NV * NW];
  __shared__ int bmaxi[G];                // per-head logit maximum of a row batch (order-preserving int)
  __shared__ float redl[PVG * G];         // per-row-group probability sums
  __shared__ int s_nrow;
  __shared__ __align__(16) int hdr[kMaxCS * 4];  // per source CTA: range [lo, hi) of the histogram bins it sent
  __shared__ int bt_s[PAGED ? kPagedBt : 1];     // (paged) block numbers of this CTA's slice, from block bt0

  const int u = blockIdx.x / CS;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const bool early = (p.flags & HATA_FLAG_EARLY_PREFETCH) != 0;

  ptx::cluster_arrive_relaxed();  // completed by the wait before the first remote store
  if (!early) ptx::pdl_wait();
  ptx::pdl_launch_dependents();

  // ---- 1. loads: seq_lens, q, W_H (bulk copy); then the codes stream ----------
  const int Lraw = p.seq_lens ? p.seq_lens[b] : p.max_seq;
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * D;
  uint4 xv = make_uint4(0u, 0u, 0u, 0u);
  // query vectors do not depend on L: load them now unless they may still be being written
  if (!early && tid < QV) xv = reinterpret_cast<const uint4*>(qg)[tid];
  float* Wsm = reinterpret_cast<float*>(smem + S.W);  // W_H of this KV head, [D][R] fp32
  uint64_t* wbar = &mbar[kMaxStages + 1];
  if (tid == 0) {
    for (int s = 0; s < kMaxStages + 2; ++s) ptx::mbar_init(&mbar[s], s == kMaxStages ? (uint32_t)kFThreads : 1u);
    ptx::fence_mbarrier_init();
    // W_H: every CTA of the cluster reads the same matrix, so keep it in L2
    constexpr uint32_t WB = D * R * 4, WCH = 32768;
    const char* Wsrc = reinterpret_cast<const char*>(p.W + (size_t)g * D * R);
    const uint64_t pol_keep = ptx::policy_evict_last();
    ptx::mbar_arrive_expect_tx(wbar, WB);
    for (uint32_t o = 0; o < WB; o += WCH)
      ptx::bulk_g2s(reinterpret_cast<char*>(Wsm) + o, Wsrc + o, min(WCH, WB - o), wbar, pol_keep);
  }
  if (tid < kMaxStages) {
    done[tid] = 0;
    lastv[tid] = -1;
  }
  if (tid == 0) {
    stat[ST_ABORT] = 0;
    s_nrow = 0;
  }
  for (int v = tid; v < kFThreads * BPT; v += kFThreads) hist[v] = 0;
  __syncthreads();
  int L = Lraw;
  if (L > p.max_seq) {
    set_status(p.status, HATA_ERR_INVALID_ARG);
    L = p.max_seq;
  }
  L = max(L, 0);
  int C = (L + CS - 1) / CS;
  C = (C + 15) & ~15;
  const int t0 = min(L, rank * C), t1 = min(L, t0 + C);
  const int nmine = t1 - t0;
  const int nst = (nmine + ST - 1) / ST;
  // Slot of token t of this unit in the K, V and code arrays: slot t of the unit's
  // slab, or (paged) slot t mod bs of physical block block_table[b][t / bs], whose
  // KV head g part holds bs consecutive slots.  A block number outside the pool
  // is flagged and replaced by block 0.
  const int32_t* btab = PAGED ? p.block_table + (size_t)b * p.max_blocks : nullptr;
  auto phys_slot = [&](int pb, int t) -> size_t {  // (paged) slot of token t in pool block pb
    if ((unsigned)pb >= (unsigned)p.n_blocks) {
      set_status(p.status, HATA_ERR_INVALID_ARG);
      pb = 0;
    }
    return (((size_t)pb * p.Hkv + g) << p.block_shift) | (size_t)(t & ((1 << p.block_shift) - 1));
  };
  // (paged) the block numbers of this CTA's slice come from shared memory when the
  // slice spans at most kPagedBt blocks, else from the table in global memory
  const int bt0 = PAGED ? (t0 >> p.block_shift) : 0;
  const int nbt = PAGED && t1 > t0 ? ((t1 - 1) >> p.block_shift) - bt0 + 1 : 0;
  const bool bt_local = PAGED && nbt <= kPagedBt;
  if constexpr (PAGED) {
    if (bt_local) {
      for (int i = tid; i < nbt; i += kFThreads) bt_s[i] = btab[bt0 + i];
      __syncthreads();
    }
  }
  auto block_of = [&](int t) -> int {  // (paged) pool block of token t; t in [t0, t1) when bt_local
    const int i = t >> p.block_shift;
    return bt_local && i - bt0 >= 0 && i - bt0 < nbt ? bt_s[i - bt0] : btab[i];
  };
  auto slot_of = [&](int t) -> size_t {
    if constexpr (PAGED) {
      return phys_slot(block_of(t), t);
    } else {
      return (size_t)u * p.max_seq + t;
    }
  };
  uint32_t* cu = p.codes + (size_t)u * p.max_seq * NW;  // the unit's slab (unpaged cache)
  const bool own_last = L > 0 && t0 <= L - 1 && L - 1 < t1;  // this CTA appends the new key's code
  const uint64_t pol_stream = ptx::policy_evict_first();
  auto issue = [&](int s) {
    const int ts = t0 + s * ST, nt = min(ST, t1 - ts);
    const int nb = nt / BULK_Q * BULK_Q;  // tokens moved by the bulk copy (16-byte multiple)
    const uint32_t bytes = (uint32_t)nb * NW * 4;
    uint64_t* bar = &mbar[s % kStages];
    lastv[s % kStages] = s;
    ptx::mbar_arrive_expect_tx(bar, bytes);
    if constexpr (PAGED) {
      // one copy per block segment (segments start on 16-token boundaries: bs >= 16);
      // up to 8 segments' block numbers are loaded together before their copies
      const int bsz = 1 << p.block_shift;
      for (int x0 = 0; x0 < nb;) {
        int pbk[8], xs[8], sg[8], nseg = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (x0 < nb) {
            const int t = ts + x0, seg = min(nb - x0, bsz - (t & (bsz - 1)));
            pbk[k] = block_of(t);
            xs[k] = x0;
            sg[k] = seg;
            x0 += seg;
            nseg = k + 1;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < nseg)
            ptx::bulk_g2s(ring + (s % kStages) * kStageBytes + (size_t)xs[k] * NW * 4,
                          p.codes + phys_slot(pbk[k], ts + xs[k]) * NW, (uint32_t)sg[k] * NW * 4, bar, pol_stream);
      }
    } else {
      if (bytes) ptx::bulk_g2s(ring + (s % kStages) * kStageBytes, cu + (size_t)ts * NW, bytes, bar, pol_stream);
    }
  };
  if (tid == 0)
    for (int s = 0; s < min(nst, kStages); ++s) issue(s);

  // ---- 2. every CTA encodes the G queries and the new key itself (all r columns) --
  if (early) {
    ptx::pdl_wait();  // q and the new key row come from the preceding kernel
    if (tid < QV) xv = reinterpret_cast<const uint4*>(qg)[tid];
  }
  {
    const T* kn = static_cast<const T*>(p.K) + slot_of(L > 0 ? L - 1 : 0) * D;
    if (tid >= QV && tid < XV && L > 0) xv = reinterpret_cast<const uint4*>(kn)[tid - QV];
  }
  // fp32 copies: residue-major for the encode (element i of vector v at
  // xr[(v * 4 + i % 4) * kXS + (i / 32) * 8 + (i / 4) % 8]) and plain for the logits
  if (tid < XV) {
    float xe[EPV];
    Vec16<T>::convert(xv, xe);
    const int v = tid * EPV / D;
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      const int i = (tid * EPV + e) % D;
      xr[(v * 4 + (i & 3)) * kXS + (i >> 5) * 8 + ((i >> 2) & 7)] = xe[e];
      if (v < G) xp[v * D + i] = xe[e];
    }
  }
  if (!ptx::mbar_wait_spin(wbar, 0u, kWaitTries)) {
    set_status(p.status, HATA_ERR_TIMEOUT);
    stat[ST_ABORT] = 1;
  }
  __syncthreads();
  // y = x . W_H[:, j] in the order of warp_dot128: lane l of that function is
  // (residue s = l % 4, a = l / 4); its partial (u = 0 product, then FMAs for +32,
  // +64, +96) and the butterfly levels 16, 8, 4 stay inside one residue, so thread
  // (s, j) computes the residue sums S_s of column j for every vector, and the
  // levels 2 and 1 give y = (S_0 + S_2) + (S_1 + S_3).  A warp takes one residue and
  // 32 consecutive columns; the thread keeps its 32 W_H values in registers.
  {
    float* sb = reinterpret_cast<float*>(smem + S.D);  // [NV][4][R] residue sums (the scores' space, unused yet)
    // with a separate key encoder only the G queries use the shared-memory W_H; the
    // CTA that appends the key encodes it below from W_k in global memory
    const int nv_w = p.Wk ? G : NV;
    auto residue_sums = [&](const float (&wr)[32], int v, int s, int j) {
      const float* xs_ = xr + (v * 4 + s) * kXS;
      float P[8];
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4) {
        const float4 x0 = reinterpret_cast<const float4*>(xs_ + u4 * 8)[0];
        const float4 x1 = reinterpret_cast<const float4*>(xs_ + u4 * 8)[1];
        const float xx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a) P[a] = u4 == 0 ? xx[a] * wr[u4 * 8 + a] : fmaf(xx[a], wr[u4 * 8 + a], P[a]);
      }
      const float q0 = P[0] + P[4], q1 = P[1] + P[5], q2 = P[2] + P[6], q3 = P[3] + P[7];
      sb[(v * 4 + s) * R + j] = (q0 + q2) + (q1 + q3);
    };
    for (int it = tid; it < 4 * R; it += kFThreads) {
      const int s = (it >> 5) & 3, j = (it >> 7) * 32 + (it & 31);
      float wr[32];
#pragma unroll
      for (int u4 = 0; u4 < 4; ++u4)
#pragma unroll
        for (int a = 0; a < 8; ++a) wr[u4 * 8 + a] = Wsm[(s + 4 * a + 32 * u4) * R + j];
#pragma unroll
      for (int v = 0; v < NV; ++v)
        if (v < nv_w) residue_sums(wr, v, s, j);
    }
    if (p.Wk && own_last) {  // block-uniform
      const float* Wkg = p.Wk + (size_t)g * D * R;
      for (int it = tid; it < 4 * R; it += kFThreads) {
        const int s = (it >> 5) & 3, j = (it >> 7) * 32 + (it & 31);
        float wr[32];
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4)
#pragma unroll
          for (int a = 0; a < 8; ++a) wr[u4 * 8 + a] = __ldg(Wkg + (size_t)(s + 4 * a + 32 * u4) * R + j);
        residue_sums(wr, G, s, j);
      }
    }
    __syncthreads();
    for (int pi = warp; pi < NV * NW; pi += kNWarp) {  // one code word per warp item
      const int v = pi / NW, jw = pi % NW, j = jw * 32 + lane;
      const float* sv = sb + v * 4 * R;
      const float y = (sv[j] + sv[2 * R + j]) + (sv[R + j] + sv[3 * R + j]);
      const unsigned bits = __ballot_sync(0xffffffffu, y > 0.f);
      if (lane == 0) qc[v * NW + jw] = bits;
    }
  }
  __syncthreads();  // codes ready; the residue sums are consumed
  if (rank == 0 && p.qcode_out && tid < G * NW) p.qcode_out[((size_t)b * p.Hq + (size_t)g * G) * NW + tid] = qc[tid];
  if (own_last && tid < NW) p.codes[slot_of(L - 1) * NW + tid] = qc[G * NW + tid];
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
      if (!stat[ST_ABORT] && !ptx::mbar_wait_spin(&mbar[s % kStages], (uint32_t)(s / kStages) & 1u, kWaitTries)) {
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
          for (int w = 0; w < NW; ++w) kw[j][w] = p.codes[slot_of(ts + i) * NW + w];
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
        // no refill once a wait has expired: the copies left in flight are then exactly
        // the ones lastv records, which the drain before exit waits for
        if (rel_s >= 0 && rel_old == ((rel_s / kStages) + 1) * kNWarp - 1 && rel_s + kStages < nst &&
            !stat[ST_ABORT]) {
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
    if (tid < 8 && nmine + tid < ((nmine + 7) & ~7)) Ds[nmine + tid] = (uint16_t)0x7fff;  // whole 8-score vectors
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

  // ---- 4. cumulative histogram -> every CTA; candidates; speculative gather ----
  const int n = min(p.k, L);
  // Candidates: every token of this slice scoring at most Tc, the largest score
  // whose cumulative count stays within `want` (about 1.5x this CTA's fair share
  // of the selection), so the candidate rows always fit the gather buffers.
  const int want = min(nmine, min(GB, 3 * ((n + CS - 1) / CS) / 2 + 16));
  {
    // inclusive cumulative counts in place, BPT consecutive bins per thread; also the
    // range of bins the other CTAs can need: from the first non-empty bin (below it
    // every count is 0) to the first bin whose count reaches n (the unit threshold is
    // never above it, so higher bins are sent as "at least n")
    if (tid == 0) {
      stat[ST_SPEC] = p.nbins - 1;  // no crossing: every bin fits
      stat[ST_LO] = NBP;
      stat[ST_HI] = NBP;
    }
    const int v0 = tid * BPT;
    int hv[BPT], local = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      hv[i] = hist[v0 + i];
      local += hv[i];
    }
    int total;
    int run = block_exclusive_scan<kFThreads>(local, warp_sums, &total);
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int v = v0 + i, before = run;
      run += hv[i];
      hist[v] = run;
      if (before <= want && run > want) stat[ST_SPEC] = v - 1;  // each crossing is unique: counts never decrease
      if (before < n && run >= n) stat[ST_HI] = min(NBP, (v + 8) & ~7);
      if (before == 0 && run > 0) stat[ST_LO] = v & ~7;
    }
  }
  __syncthreads();
  // bins [lo, hi) of the u16 cumulative histogram into slot `rank` of every CTA (8
  // bins per 16-byte store), with (lo, hi) in the header
  ptx::cluster_wait();  // every CTA of the cluster has started (arrive at kernel start)
  {
    const int plo = stat[ST_LO], phi = stat[ST_HI];
    const int ng = (phi - plo) / 8;
    for (int e = tid; e < (ng + 1) * CS; e += kFThreads) {
      const int c = e / (ng + 1), k = e % (ng + 1);
      if (k == ng) {
        ptx::st_dsmem_v4(ptx::dsmem_addr(&hdr[rank * 4], c), make_uint4((uint32_t)plo, (uint32_t)phi, 0u, 0u));
      } else {
        const int v = plo + k * 8;
        const int* h = hist + v;
        uint4 pk;
        pk.x = (uint32_t)h[0] | ((uint32_t)h[1] << 16);
        pk.y = (uint32_t)h[2] | ((uint32_t)h[3] << 16);
        pk.z = (uint32_t)h[4] | ((uint32_t)h[5] << 16);
        pk.w = (uint32_t)h[6] | ((uint32_t)h[7] << 16);
        ptx::st_dsmem_v4(ptx::dsmem_addr(&hslot[rank * NBP + v], c), pk);
      }
    }
  }
  ptx::cluster_arrive_release();  // #1, completed by the threshold warp and after the logits (below)
  const int Tc = stat[ST_SPEC];
  const bool scan_cands = Tc >= 0 && !stat[ST_ABORT];

  const T* Kg = static_cast<const T*>(p.K);
  const T* Vg = static_cast<const T*>(p.V);
  T* Kr = reinterpret_cast<T*>(ring);
  T* Vr = reinterpret_cast<T*>(ring) + (size_t)GB * D;
  // Row gathers complete on the gather mbarrier: every thread arrives once per
  // gather (cp.async.mbarrier.arrive.noinc), so the phase ends when all its copies
  // have landed, and any thread may wait for it.
  uint32_t gphase = 0;
  auto gather_commit = [&]() { ptx::cp_async_mbar_arrive_noinc(gbar); };
  auto gather_wait = [&]() {
    if (!ptx::mbar_wait_spin(gbar, gphase & 1u, kWaitTries)) {
      set_status(p.status, HATA_ERR_TIMEOUT);
      stat[ST_ABORT] = 1;
    }
    ++gphase;
  };
  // Fallback gathers (selected rows listed in `list`): every thread takes pieces.
  // An index outside this CTA's slice (never expected) is flagged and replaced by row t0.
  auto gather_issue = [&](const int* list, int nr) {
    for (int e = tid; e < nr * 2 * RPR; e += kFThreads) {
      const int r = e / (2 * RPR), w = e % (2 * RPR);
      int t = list[r];
      if (t < t0 || t >= t1) {
        set_status(p.status, HATA_ERR_INVALID_ARG);
        t = t0;
      }
      const size_t row = slot_of(t) * D;
      if (w < RPR) ptx::cp_async16(Kr + (size_t)r * D + w * EPV, Kg + row + w * EPV);
      else ptx::cp_async16(Vr + (size_t)r * D + (w - RPR) * EPV, Vg + row + (w - RPR) * EPV);
    }
    gather_commit();
  };
  // logits (exp2 domain) of gather slots 0..nr-1 into lg[h * GB + slot], by warps
  // w_first.. (nw of them): 16 threads per row, 8 elements each, every head at once;
  // each thread keeps its 8-element slice of the G query vectors in registers.  With
  // track_max, the per-head maximum goes into bmaxi.
  auto compute_logits = [&](int nr, bool track_max, int w_first, int nw) {
    const int sgi = lane % LT;
    float xq[G][LE];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float4 a = reinterpret_cast<const float4*>(xp + h * D + sgi * LE)[0];
      const float4 c = reinterpret_cast<const float4*>(xp + h * D + sgi * LE)[1];
      xq[h][0] = a.x; xq[h][1] = a.y; xq[h][2] = a.z; xq[h][3] = a.w;
      xq[h][4] = c.x; xq[h][5] = c.y; xq[h][6] = c.z; xq[h][7] = c.w;
    }
    float mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
#pragma unroll 2
    for (int rb = (warp - w_first) * (32 / LT); rb < nr; rb += nw * (32 / LT)) {  // warp-uniform trip count
      const int r = rb + lane / LT;
      const bool valid = r < nr;
      const int rr = valid ? r : 0;
      float kv[LE];
#pragma unroll
      for (int v = 0; v < LE / EPV; ++v) {
        float t8[EPV];
        Vec16<T>::load(Kr + (size_t)rr * D + sgi * LE + v * EPV, t8);
#pragma unroll
        for (int j = 0; j < EPV; ++j) kv[v * EPV + j] = t8[j];
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
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float lv = acc[h] * p.scale_log2;
          lg[h * GB + r] = lv;
          mx[h] = fmaxf(mx[h], lv);
        }
      }
    }
    if (track_max) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], LT));
        if (lane == 0 && mx[h] != -INFINITY) atomicMax(&bmaxi[h], ord_of(mx[h]));
      }
    }
  };
  // Candidates in token order, without atomics: warp w owns a contiguous run of
  // 8-score vectors, lane l the vectors wv0 + 128 tr + 32 i + l (trip tr < 4, group
  // i < 4).  trip_flags packs the lane's hit flags of a trip into one word, byte i
  // for group i with bit k for token k of the vector.  Pass 1 counts them; after the
  // warps' totals are known, pass 2 recomputes the flags, places the hits at the
  // warp's offset (a shuffle scan per group) and the warp gathers their K and V
  // rows.  Scores are below 2^15, so in each 16-bit half of
  // (x + (0x7fff - Tc) * 0x10001) bit 15 is set exactly when that score exceeds Tc;
  // the scores past nmine read 0x7fff (set after the scan).
  const int nvec = (nmine + 7) / 8;  // whole vectors inside tok_cap (a multiple of 16)
  const int nvw = (nvec + kNWarp - 1) / kNWarp;
  const int wv0 = min(nvec, warp * nvw), wv1 = min(nvec, wv0 + nvw);
  const int ntrip = scan_cands ? (wv1 - wv0 + 127) / 128 : 0;  // warp-uniform; <= 4 since tok_cap <= kTokCap
  const uint32_t addc = (uint32_t)(0x7fff - max(Tc, 0)) * 0x10001u;
  auto trip_flags = [&](int tr) -> uint32_t {
    uint32_t M = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = wv0 + tr * 128 + 32 * i + lane;
      if (e < wv1) {
        const uint4 w4 = reinterpret_cast<const uint4*>(Ds)[e];
        // token 2j's flag to bit 2j, token 2j + 1's to bit 16 + 2j, then folded to 2j + 1
        const uint32_t y = ((~(w4.x + addc) & 0x80008000u) >> 15) | ((~(w4.y + addc) & 0x80008000u) >> 13) |
                           ((~(w4.z + addc) & 0x80008000u) >> 11) | ((~(w4.w + addc) & 0x80008000u) >> 9);
        M |= ((y | (y >> 15)) & 0xffu) << (8 * i);
      }
    }
    return M;
  };
  {
    int c = 0;
#pragma unroll 1
    for (int tr = 0; tr < ntrip; ++tr) c += __popc(trip_flags(tr));
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) warp_sums[warp] = c;
  }
  __syncthreads();
  int wbase = 0, ncand_all = 0;
#pragma unroll
  for (int w = 0; w < kNWarp; ++w) {
    const int x = warp_sums[w];
    wbase += w < warp ? x : 0;
    ncand_all += x;
  }
  const int ncand = min(ncand_all, GB);  // <= want <= GB by construction
  if (ntrip > 0) {
    const int wstart = wbase;
#pragma unroll 1
    for (int tr = 0; tr < ntrip; ++tr) {
      const uint32_t M = trip_flags(tr);
      if (__any_sync(0xffffffffu, M != 0u)) {
        // inclusive scans over the lanes of the four groups' counts, two per word
        int s01 = __popc(M & 0xffu) | (__popc(M & 0xff00u) << 16);
        int s23 = __popc(M & 0xff0000u) | (__popc(M & 0xff000000u) << 16);
        const int c01 = s01, c23 = s23;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y01 = __shfl_up_sync(0xffffffffu, s01, o), y23 = __shfl_up_sync(0xffffffffu, s23, o);
          if (lane >= o) {
            s01 += y01;
            s23 += y23;
          }
        }
        const int t01 = __shfl_sync(0xffffffffu, s01, 31), t23 = __shfl_sync(0xffffffffu, s23, 31);
        // exclusive start of each group's hits of this lane, in token order
        const int g0 = wbase + (s01 & 0xffff) - (c01 & 0xffff);
        const int g1 = wbase + (t01 & 0xffff) + (s01 >> 16) - (c01 >> 16);
        const int g2 = wbase + (t01 & 0xffff) + (t01 >> 16) + (s23 & 0xffff) - (c23 & 0xffff);
        const int g3 = wbase + (t01 & 0xffff) + (t01 >> 16) + (t23 & 0xffff) + (s23 >> 16) - (c23 >> 16);
        const int tb = t0 + (wv0 + tr * 128 + lane) * 8;
        // hits of the lane, group by group, ascending token within a group
        uint32_t mm = M;
        int gi = 0, pos = g0;
        while (mm) {
          const int bit = __ffs(mm) - 1;
          mm &= mm - 1u;
          const int i = bit >> 3;
          if (i != gi) {
            gi = i;
            pos = i == 1 ? g1 : (i == 2 ? g2 : g3);
          }
          if (pos < GB) cand[pos] = tb + 256 * i + (bit & 7);
          ++pos;
        }
        wbase += (t01 & 0xffff) + (t01 >> 16) + (t23 & 0xffff) + (t23 >> 16);
      }
    }
    __syncwarp();
    // this warp's candidate rows: (candidate, 16-byte piece) pairs over the lanes
    const int q0 = min(wstart, GB), nq = min(wbase, GB) - q0;
    if constexpr (PAGED) {
      // 32 candidates at a time: lane l looks up candidate l's row, the pieces take it by shuffle
      for (int c0 = 0; c0 < nq; c0 += 32) {  // warp-uniform
        const int qc = min(32, nq - c0);
        const unsigned long long myrow = lane < qc ? (unsigned long long)slot_of(cand[q0 + c0 + lane]) * D : 0ull;
        for (int e = lane; e < qc * 2 * RPR; e += 32) {  // 2 * RPR is a multiple of 32: uniform trip count
          const int qi = e / (2 * RPR), pc = e % (2 * RPR), q = q0 + c0 + qi;
          const size_t row = (size_t)__shfl_sync(0xffffffffu, myrow, qi);
          if (pc < RPR) ptx::cp_async16(Kr + (size_t)q * D + pc * EPV, Kg + row + pc * EPV);
          else ptx::cp_async16(Vr + (size_t)q * D + (pc - RPR) * EPV, Vg + row + (pc - RPR) * EPV);
        }
      }
    } else {
#pragma unroll 2
      for (int e = lane; e < nq * 2 * RPR; e += 32) {
        const int q = q0 + e / (2 * RPR), pc = e % (2 * RPR);
        const size_t row = slot_of(cand[q]) * D;
        if (pc < RPR) ptx::cp_async16(Kr + (size_t)q * D + pc * EPV, Kg + row + pc * EPV);
        else ptx::cp_async16(Vr + (size_t)q * D + (pc - RPR) * EPV, Vg + row + (pc - RPR) * EPV);
      }
    }
  }
  gather_commit();  // gather phase 0: the candidates' rows
  if (tid < G) {
    part[tid * 4] = -INFINITY;
    part[tid * 4 + 1] = 0.f;
    bmaxi[tid] = ord_of(-INFINITY);
  }

  // ---- 5. warp 0: unit threshold and the selected candidates; the other warps:
  //         the candidates' logits (as soon as their rows have landed) -----------
  if (warp == 0) {
    ptx::cluster_wait();  // #1: every CTA holds every CTA's cumulative histogram range
    // T = the smallest score v whose unit total (sum of the CS cumulative counts)
    // is at least n; the total at the top bin is L >= n.  Rounds of a 32-way split
    // of [lo, hi], one probe per lane.  Source c sent bins [lo_c, hi_c): below
    // lo_c its count is 0, from hi_c on it is at least n (counted as n).
    int loc[kMaxCS], hic[kMaxCS];
#pragma unroll
    for (int c = 0; c < kMaxCS; ++c) {  // sources past CS: an empty range below every bin
      const int cc = min(c, CS - 1);
      const int l_ = hdr[cc * 4], h_ = hdr[cc * 4 + 1];
      loc[c] = c < CS ? l_ : NBP;
      hic[c] = c < CS ? h_ : NBP + 1;
    }
    auto total_at = [&](int v) {
      int hv[kMaxCS];
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) hv[c] = hslot[min(c, CS - 1) * NBP + v];
      int t = 0;
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) t += v < loc[c] ? 0 : (v >= hic[c] ? n : hv[c]);
      return t;
    };
    int lo = 0, hi = p.nbins - 1;
    while (lo < hi) {  // warp-uniform
      const int step = (hi - lo + 32) / 32;
      const int v = min(hi, lo + (lane + 1) * step - 1);
      const unsigned ok = __ballot_sync(0xffffffffu, total_at(v) >= n);
      const int f = __ffs(ok) - 1;  // lane 31 probes hi, which always qualifies
      hi = min(hi, lo + (f + 1) * step - 1);
      lo = lo + f * step;
    }
    const int Tth = n == 0 ? 0 : lo;
    // per source CTA (lane c): cumulative count below T and at T (exact: T <= hi_c - 1)
    int cb = 0, ce = 0;
    if (lane < CS) {
      const int lo_c = hdr[lane * 4];
      const int h1 = Tth - 1 < lo_c ? 0 : (int)hslot[lane * NBP + max(Tth - 1, 0)];
      const int h0 = Tth < lo_c ? 0 : (int)hslot[lane * NBP + Tth];
      cb = Tth > 0 ? h1 : 0;
      ce = h0 - cb;
    }
    const int lb = __reduce_add_sync(0xffffffffu, lane < rank ? cb : 0);
    const int eb = __reduce_add_sync(0xffffffffu, lane < rank ? ce : 0);
    const int below_all = __reduce_add_sync(0xffffffffu, cb);
    const int myl = __shfl_sync(0xffffffffu, cb, rank);
    const int mye = __shfl_sync(0xffffffffu, ce, rank);
    const int mq = n == 0 ? 0 : n - below_all;
    if (lane == 0) {
      stat[ST_T] = Tth;
      stat[ST_M] = mq;
      stat[ST_LESS_BEFORE] = lb;
      stat[ST_EQ_BEFORE] = eb;
      stat[ST_MYLESS] = myl;
      stat[ST_MYEQ] = mye;
    }
    // the selected candidates (when they hold the whole selection of this slice),
    // in ascending token order: scores below T, and the first quota = m - (ties of
    // earlier CTAs) ties at T
    const int nsel_w = myl + max(0, min(mq - eb, mye));
    if ((nsel_w == 0 || Tth <= Tc) && nsel_w > 0) {
      const int quota = max(0, mq - eb);
      const unsigned lm = (1u << lane) - 1u;
      int lt_run = 0, eq_run = 0;
      for (int r0 = 0; r0 < ncand; r0 += 32) {
        const int r = r0 + lane;
        const int dv = r < ncand ? (int)Ds[cand[r] - t0] : INT_MAX;
        const bool lt = dv < Tth, eq = dv == Tth;
        const unsigned blt = __ballot_sync(0xffffffffu, lt), beq = __ballot_sync(0xffffffffu, eq);
        const int ltpre = lt_run + __popc(blt & lm), eqpre = eq_run + __popc(beq & lm);
        if (lt || (eq && eqpre < quota)) rowl[ltpre + min(eqpre, quota)] = (uint16_t)r;
        lt_run += __popc(blt);
        eq_run += __popc(beq);
      }
      if (lane == 0) s_nrow = lt_run + min(eq_run, quota);
    }
  } else {
    gather_wait();  // phase 0
    compute_logits(ncand, false, 1, kNWarp - 1);
    ptx::cluster_wait();  // #1 (these warps' side)
  }
  if (warp == 0) gphase = 1;  // warp 0 did not wait on phase 0; the barrier below orders it after
  __syncthreads();
  const int Tt = stat[ST_T], m = stat[ST_M];
  const int less_before = stat[ST_LESS_BEFORE], eq_before = stat[ST_EQ_BEFORE];
  const int sel_before = less_before + min(eq_before, m);
  const int ties_here = max(0, min(m - eq_before, stat[ST_MYEQ]));
  const int nsel_here = stat[ST_MYLESS] + ties_here;  // this CTA's share of the selection
  // the candidates hold every selected token of this slice when T <= Tc
  const bool covered = nsel_here == 0 || Tt <= Tc;

  // ---- 7. ascending indices (only when asked for) and the fallback row list -----
  int32_t* ix = p.idx_out ? p.idx_out + (size_t)u * p.k : nullptr;
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

  // ---- 8. attention partials over this CTA's selected rows -----------------------
  constexpr int OPT = (G * D + kFThreads - 1) / kFThreads;  // output elements per thread
  float oacc[OPT];
#pragma unroll
  for (int q = 0; q < OPT; ++q) oacc[q] = 0.f;
  // Softmax and P.V over nr rows whose logits are in lg (slot rmap[i], or i without
  // a map) against the running maximum max(part.m, bmaxi), folded into oacc and
  // the running (max, sum) in part.
  auto softmax_pv = [&](int nr, const uint16_t* rmap) {
    for (int e = tid; e < G * nr; e += kFThreads) {
      const int h = e / nr, i = e - h * nr;
      const int sl = rmap ? (int)rmap[i] : i;
      const float mn = fmaxf(part[h * 4], float_of_ord(bmaxi[h]));
      lg[h * GB + sl] = exp2f(lg[h * GB + sl] - mn);
    }
    __syncthreads();
    // P.V: thread (column pair cp, row group rg) sums rows rg, rg + PVG, ... for every
    // head (and the probabilities), then the PVG partial sums of each output go
    // through shared memory (the K rows' buffer, free once the logits are done)
    const int cp = tid % (D / 2), rg = tid / (D / 2);
    float pacc[G][2], lsum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) pacc[h][0] = pacc[h][1] = lsum[h] = 0.f;
#pragma unroll 4
    for (int r = rg; r < nr; r += PVG) {
      const int sl = rmap ? (int)rmap[r] : r;
      float v0, v1;
      if constexpr (ESZ == 2) {
        const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Vr + (size_t)sl * D)[cp]);
        v0 = f.x;
        v1 = f.y;
      } else {
        const float2 f = reinterpret_cast<const float2*>(Vr + (size_t)sl * D)[cp];
        v0 = f.x;
        v1 = f.y;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pr_ = lg[h * GB + sl];
        pacc[h][0] = fmaf(pr_, v0, pacc[h][0]);
        pacc[h][1] = fmaf(pr_, v1, pacc[h][1]);
        lsum[h] += pr_;
      }
    }
    float* red = reinterpret_cast<float*>(Kr);  // [PVG][G][D]
#pragma unroll
    for (int h = 0; h < G; ++h)
      reinterpret_cast<float2*>(red + ((size_t)rg * G + h) * D)[cp] = make_float2(pacc[h][0], pacc[h][1]);
    if (cp == 0)
#pragma unroll
      for (int h = 0; h < G; ++h) redl[rg * G + h] = lsum[h];
    __syncthreads();
#pragma unroll
    for (int q = 0; q < OPT; ++q) {
      const int e = tid + q * kFThreads;
      if (e < G * D) {
        const int h = e / D, i = e % D;
        const float m_old = part[h * 4];
        const float mn = fmaxf(m_old, float_of_ord(bmaxi[h]));
        const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - mn);
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < PVG; ++j) sum += red[((size_t)j * G + h) * D + i];
        oacc[q] = fmaf(oacc[q], alpha, sum);
      }
    }
    __syncthreads();  // every thread has read the running maxima of this batch
    if (tid < G) {
      const int h = tid;
      const float m_old = part[h * 4];
      const float mn = fmaxf(m_old, float_of_ord(bmaxi[h]));
      const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - mn);
      float ls = 0.f;
#pragma unroll
      for (int j = 0; j < PVG; ++j) ls += redl[j * G + h];
      part[h * 4 + 1] = part[h * 4 + 1] * alpha + ls;
      part[h * 4] = mn;
      bmaxi[h] = ord_of(-INFINITY);
    }
  };
  if (covered) {
    // the candidates' rows and logits are in place: one batch over the selected ones
    const int nsel = stat[ST_ABORT] ? 0 : s_nrow;
    for (int i = tid; i < nsel; i += kFThreads) {  // per-head maximum over the selected rows
      const int sl = rowl[i];
#pragma unroll
      for (int h = 0; h < G; ++h) atomicMax(&bmaxi[h], ord_of(lg[h * GB + sl]));
    }
    __syncthreads();
    if (nsel > 0) softmax_pv(nsel, rowl);
  } else if (!stat[ST_ABORT]) {
    // the guess missed: gather the selected rows batch by batch
    const int nrows_total = min(nsel_here, p.sel_cap);
    for (int r0 = 0; r0 < nrows_total; r0 += GB) {
      const int nr = min(GB, nrows_total - r0);
      __syncthreads();  // previous batch's readers are done with the buffers
      gather_issue(sel + r0, nr);
      gather_wait();
      compute_logits(nr, true, 0, kNWarp);
      __syncthreads();
      softmax_pv(nr, nullptr);
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
  ptx::cluster_sync();  // #2: every CTA holds the partials of its columns
  for (int col = tid; col < mc; col += kFThreads) {
    const int e = rank * mc + col;
    if (e < G * D) {
      const int h = e / D;
      // all sources' (max, sum, column) first, then the log-sum-exp merge
      float mv[kMaxCS], lv[kMaxCS], ov[kMaxCS];
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) {
        const int cc = min(c, CS - 1);
        mv[c] = c < CS ? mslot[cc * stride + 2 * h] : -INFINITY;
        lv[c] = mslot[cc * stride + 2 * h + 1];
        ov[c] = mslot[cc * stride + 2 * G + col];
      }
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) M = fmaxf(M, mv[c]);
      float l = 0.f, o = 0.f;
      if (M != -INFINITY)
#pragma unroll
        for (int c = 0; c < kMaxCS; ++c) {
          if (mv[c] == -INFINITY) continue;
          const float w = exp2f(mv[c] - M);
          l = fmaf(lv[c], w, l);
          o = fmaf(ov[c], w, o);
        }
      static_cast<T*>(p.out)[((size_t)b * p.Hq + (size_t)g * G + h) * D + (e % D)] = from_f32<T>(l > 0.f ? o / l : 0.f);
    }
  }
  if (stat[ST_ABORT]) {
    // nothing may land in shared memory after the CTA exits: every thread waits for its
    // own row gathers, and thread 0 gives the bulk copies one more bounded chance
    ptx::cp_async_wait_all();
    if (tid == 0) {
      for (int bi = 0; bi < kStages; ++bi)
        if (lastv[bi] >= 0) ptx::mbar_wait_bounded(&mbar[bi], (uint32_t)(lastv[bi] / kStages) & 1u, kWaitTries);
      ptx::mbar_wait_bounded(&mbar[kMaxStages + 1], 0u, kWaitTries);  // the W_H copy
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct Plan {
  bool ok;
  int CS, tok_cap, sel_cap, nbins, stages;
  size_t smem;
  SmemLayout lay;
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
  const void* kern = (const void*)fused_step_kernel<T, NW, G, false>;
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
    pl.stages = 0;
    cudaFuncAttributes fa, fa_paged;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
        cudaFuncGetAttributes(&fa_paged, (const void*)fused_step_kernel<T, NW, G, true>) != cudaSuccess) {
      (void)cudaGetLastError();
      return best;
    }
    fa.sharedSizeBytes = std::max(fa.sharedSizeBytes, fa_paged.sharedSizeBytes);  // one plan serves both
    for (int st = kMaxStages; st >= kMinStages; --st) {
      const size_t sm = smem_layout(G, NW, esize, tok_cap, pl.sel_cap, pl.nbins, CS, st).total;
      if (sm + fa.sharedSizeBytes <= 227 * 1024) {  // + static shared memory
        pl.stages = st;
        pl.lay = smem_layout(G, NW, esize, tok_cap, pl.sel_cap, pl.nbins, CS, st);
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

template <typename T, int NW, int G, bool PAGED>
cudaError_t launch_fused_t(const Plan& pl, const hata_dims_t& d, const FusedParams& prm, cudaStream_t st) {
  auto kern = fused_step_kernel<T, NW, G, PAGED>;
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
    return prm.block_table ? launch_fused_t<T, NW, G, true>(pl, d, prm, st)
                           : launch_fused_t<T, NW, G, false>(pl, d, prm, st);
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
                              const float* W, const float* Wk, uint32_t* codes, const int32_t* seq_lens, int k,
                              float scale, void* out, uint32_t* qcode_out, int32_t* idx_out,
                              const PagedCache* pg, char* ws, cudaStream_t st) {
  const Plan pl = make_plan(d, k);
  if (!pl.ok) return cudaErrorNotSupported;
  FusedParams prm;
  prm.q = q;
  prm.K = K;
  prm.V = V;
  prm.W = W;
  prm.Wk = Wk == W ? nullptr : Wk;
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
  prm.flags = d.flags;
  prm.stages = pl.stages;
  prm.lay = pl.lay;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.block_table = pg ? pg->block_table : nullptr;
  prm.block_shift = pg ? pg->block_shift : 0;
  prm.n_blocks = pg ? pg->n_blocks : 0;
  prm.max_blocks = pg ? pg->max_blocks : 0;
  return dispatch<LaunchFn>(d, pl, d, prm, st);
}

}  // namespace hata
