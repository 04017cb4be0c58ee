// The HATA decode step as three kernels chained by programmatic dependent launch
// ("HATA" paper notes, Decode 阶段算法 end to end, with the fusions of 硬件高效优化:
// projection + sign + bitpack + cache update in one kernel, XOR + popc Hamming
// scan with coalesced access, gather fused into the attention).
//
// Every (batch, KV head) unit's L cached tokens are cut into chunks of C tokens,
// and the chunks of all units are spread over all SMs.
//
// encode kernel (one small CTA per (unit, 32-column code word)):
//   0. the G query codes and the new key's code (written to cache slot L - 1),
//      fp32 FMAs in the order of warp_dot128, so the codes equal
//      hata_encode_append's decode form; the query codes go to the workspace.
// scan kernel (one CTA per SM, persistent over chunks; it starts once the encode
// kernel has passed its own wait on the preceding kernel).  Per chunk:
//   1. bulk-copy (TMA engine, no tensor map) the chunk's codes into shared
//      memory, all of it in flight at once, one mbarrier per 16 KB piece (slots
//      [0, L - 1) are final before the encode kernel ends, so this overlaps it);
//   2. wait for the encode kernel, then read the query codes (and patch slot L - 1
//      of a chunk that holds it with the new key's code);
//   3. score every token (xor + popc, the GQA sum folded into per-word
//      constants), keeping u16 scores and their histogram in shared memory;
//   4. write the chunk record: the cumulative histogram (u16 per score), and, in
//      token order, every token scoring below a bound Bc plus the first few
//      scoring exactly Bc, with Bc the first score whose cumulative count passes
//      about twice the chunk's fair share of the selection.
// tail kernel (one thread-block cluster per unit):
//   5. every CTA stages the unit's chunk records in shared memory and sums the
//      cumulative histograms to find the unit threshold T (the smallest score
//      with at least n = min(k, L) tokens at or below it); from the counts at T - 1
//      and T it derives each chunk's share of the selection: all of its tokens
//      below T and, of the ties at T, the quota left after earlier chunks (ties go
//      to the lower token index);
//   6. CTA r of the cluster takes the selected ranks [r n / CS, (r + 1) n / CS):
//      it reads those tokens from the candidate lists (a chunk whose list stops
//      short of T is rescored from the cache instead), gathers their K/V rows with
//      cp.async, and computes the flash-decode partial (max, sum, weighted V) of
//      the G query heads;
//   7. the partials go to the CTAs owning each output column through distributed
//      shared memory; after a cluster barrier each CTA merges its columns
//      (log-sum-exp) and writes them.
// The kernels exchange only the chunk records (and the query codes, for a
// rescore) through the workspace.  Every wait is a bounded wait on this CTA's own
// copies: on expiry the kernel records HATA_ERR_TIMEOUT, skips the remaining
// work, still reaches every cluster barrier, and drains its copies before exit.
#include <algorithm>
#include <climits>
#include <map>
#include <mutex>
#include <tuple>

#include "hata_kernels.cuh"
#include "hata_ptx.cuh"

namespace hata {

namespace {

constexpr int kSThreads = 512;                  // scan CTA
constexpr int kSWarp = kSThreads / 32;
constexpr int kTThreads = 512;                  // tail CTA
constexpr int kEThreads = 128;                  // encode CTA: 4 residues x the 32 columns of one code word
constexpr int kNWarp = 512 / 32;
constexpr int kRingBytes = 131072;              // one chunk's codes, all in flight at once
constexpr int kPieceBytes = 16384;              // one mbarrier per piece
constexpr int kMaxPieces = kRingBytes / kPieceBytes;
constexpr int kMinChunk = 256;
constexpr int kMaxB = 1024;                     // batches covered by the scan's chunk map
constexpr int kMaxChunkBlocks = 32768 / 16 + 1;  // (paged) blocks a chunk can span: C <= 32768, bs >= 16
constexpr int kXS = 36;                         // floats per residue row of an encoded vector
constexpr int kMaxCS = 16;                      // largest tail cluster
constexpr int kMaxGB = 256;                     // largest gather batch (rows)
constexpr uint32_t kWaitTries = 1u << 22;
constexpr uint32_t kTestWaitTries = 1u << 10;   // the test hook's wait on a barrier nothing completes
constexpr uint32_t kAbortBit = 0x80000000u;     // chunk record header: the scan gave up on this chunk

// Chunk record (one per chunk slot, unit u's slots u * P .. u * P + P - 1):
//   int32 hdr[4]     listed count, Bc, ties at Bc listed, chunk length (| kAbortBit)
//   u16   cum[nbp]   tokens of the chunk scoring <= v
//   u32   cand[cap]  listed tokens in token order: (score << 16) | offset in the chunk
struct StepGeom {
  int C, P, cap, nbp;
  uint32_t slot_bytes, cum_off, cand_off;
  uint32_t hist_bytes, unit_bytes;  // unit region: histogram [nbp] u32, then P chunk records
};

struct StepParams {
  const void* q;
  const void* K;
  const void* V;
  const float* Wq;
  const float* Wk;  // separate key encoder, or null: Wq encodes keys too
  uint32_t* codes;
  const int32_t* seq_lens;
  void* out;
  uint32_t* qcode_out;
  int32_t* idx_out;
  uint32_t* status;
  unsigned char* rec;  // chunk records [U * P][slot_bytes]
  uint32_t* qcode_ws;  // [B][Hq][NW] query codes (the tail's rescores read them)
  int B, Hq, Hkv, max_seq, k, flags;
  float scale_log2;
  StepGeom geo;
  int GB;  // tail gather batch (rows)
  // paged cache (K, V and codes are pools of blocks [n_blocks][Hkv][1 << block_shift][...])
  const int32_t* block_table;  // [B][max_blocks]
  int block_shift, n_blocks, max_blocks;
};

__host__ __device__ constexpr int nbins_padded(int G, int R) { return (G * R + 1 + 7) / 8 * 8; }

// Dynamic shared memory of the scan kernel: ring | scores (aliased by the encode's
// residue sums) | histogram | fp32 encode inputs | mbarriers.
struct ScanSmem {
  int ring, D, hist, mbar, total;
};
__host__ __device__ constexpr int round16(int x) { return (x + 15) / 16 * 16; }
__host__ __device__ inline ScanSmem scan_smem(int G, int NW) {
  const int R = NW * 32;
  const int cmax = kRingBytes / (NW * 4);
  const int nbp = nbins_padded(G, R);
  const int bpt = (nbp + kSThreads - 1) / kSThreads;
  ScanSmem s{};
  s.ring = 0;
  s.D = kRingBytes;
  s.hist = s.D + round16(cmax * 2 + 32);
  s.mbar = s.hist + bpt * kSThreads * 4;
  s.total = s.mbar + (kMaxPieces + 1) * 8;
  return s;
}

// Dynamic shared memory of the tail kernel.
struct TailSmem {
  int rec, Kr, Vr, lg, pb, rowtok, rowslot, xp, mslot, sst, qcs, mbar, total;
};
// Row stride (elements) of the gathered K and V rows: bf16 rows are padded by 16 bytes so
// that the tensor-core fragment loads of eight consecutive rows hit distinct banks.
__host__ __device__ constexpr int tail_row_stride(int esize) { return esize == 2 ? kHeadDim + 8 : kHeadDim; }
// Row stride (elements) of the bf16 probability tile [8 heads][GB + 8].
__host__ __device__ constexpr int tail_p_stride(int GB) { return GB + 8; }
__host__ __device__ inline TailSmem tail_smem(int G, int NW, int esize, const StepGeom& geo, int GB, int CS) {
  TailSmem s{};
  int o = 0;
  auto take = [&](int bytes) {
    const int r = o;
    o = round16(o + bytes);
    return r;
  };
  s.rec = take((int)geo.unit_bytes);
  // the K rows' buffer also holds the P.V partial sums [row groups][G][d] fp32
  s.Kr = take(std::max(GB * tail_row_stride(esize) * esize, (kTThreads / (kHeadDim / 2)) * G * kHeadDim * 4));
  s.Vr = take(GB * tail_row_stride(esize) * esize);
  s.lg = take(G * GB * 4);
  s.pb = take(esize == 2 ? 8 * tail_p_stride(GB) * 2 : 0);
  s.rowtok = take(GB * 4);
  s.rowslot = take(GB * 8);
  s.xp = take(G * kHeadDim * 4);
  s.mslot = take(CS * ((G * kHeadDim + CS - 1) / CS + 2 * G) * 4);
  s.sst = take(geo.P * 4 * 4);
  s.qcs = take(G * NW * 4);
  s.mbar = take(2 * 8);
  s.total = o;
  return s;
}

// D += A * B for a 16x16 bf16 A (row), a 16x8 bf16 B (col) and fp32 D, in the fragment
// layout of mma.m16n8k16 (g = lane / 4, c = lane % 4): a0 = A[g][2c..2c+1], a2 = A[g][2c+8..];
// rows 8-15 of A are zero (a1 = a3 = 0); b0 = B[2c..2c+1][g], b1 = B[2c+8..2c+9][g];
// d0 = D[g][2c], d1 = D[g][2c+1] (d2, d3: rows g + 8).
__device__ __forceinline__ void mma_16816_top(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// Two transposed 8x8 b16 tiles; lanes 0-7 address tile 0's rows, lanes 8-15 tile 1's.
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& r0, uint32_t& r1, const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r0), "=r"(r1)
               : "r"((unsigned)__cvta_generic_to_shared(row))
               : "memory");
}

// Order-preserving map of a float (not NaN) to an int, for integer atomicMax.
__device__ __forceinline__ int ord_of(float f) {
  const int i = __float_as_int(f);
  return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float float_of_ord(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

template <typename T>
struct Vec16;  // 16-byte vector of T as fp32
template <>
struct Vec16<__nv_bfloat16> {
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
  __device__ __forceinline__ static void convert(const uint4& v, float (&o)[4]) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
};

// Slot of token t of unit (b, g) in the K, V and code arrays: slot t of the unit's
// slab, or (paged) slot t mod bs of pool block block_table[b][t / bs].  A block
// number outside the pool is flagged and replaced by block 0.
template <bool PAGED>
__device__ __forceinline__ size_t token_slot(const StepParams& p, int b, int g, int t) {
  if constexpr (PAGED) {
    int pb = p.block_table[(size_t)b * p.max_blocks + (t >> p.block_shift)];
    if ((unsigned)pb >= (unsigned)p.n_blocks) {
      set_status(p.status, HATA_ERR_INVALID_ARG);
      pb = 0;
    }
    return (((size_t)pb * p.Hkv + g) << p.block_shift) | (size_t)(t & ((1 << p.block_shift) - 1));
  } else {
    return ((size_t)b * p.Hkv + g) * p.max_seq + t;
  }
}

__device__ __forceinline__ int clamp_seq(int L, int max_seq) { return L < 0 ? 0 : (L > max_seq ? max_seq : L); }

// ---------------------------------------------------------------------------
// encode kernel: the G query codes and the new key's code of every unit, one code
// word (32 columns of W_H) per CTA
// ---------------------------------------------------------------------------
template <typename T, int NW, int G, bool PAGED>
__global__ void __launch_bounds__(kEThreads) step_encode_kernel(const StepParams p) {
  constexpr int D = kHeadDim;
  constexpr int ESZ = (int)sizeof(T);
  constexpr int R = NW * 32;
  constexpr int NV = G + 1;                  // G queries + new key
  constexpr int XV = NV * D * ESZ / 16;      // 16-byte vectors of q + new key
  constexpr int QV = G * D * ESZ / 16;
  constexpr int EPV = 16 / ESZ;
  static_assert(kEThreads == 128, "4 residues x 32 columns");
  __shared__ __align__(16) float xr[NV * 4 * kXS];
  __shared__ float sb[NV * 4 * 32];

  // CTA (unit, code word jw): thread (residue s, column 32 jw + lane)
  const int tid = threadIdx.x, lane = tid & 31, s = tid >> 5;
  const int u = blockIdx.x / NW, jw = blockIdx.x % NW;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const int jc = jw * 32 + lane;
  const bool early = (p.flags & HATA_FLAG_EARLY_PREFETCH) != 0;
  // W_H rows s + 4a + 32u4 of column jc: y_jc of warp_dot128 is (S_0 + S_2) + (S_1 + S_3)
  // with S_s this thread's residue sum
  auto load_w = [&](const float* Wm, float (&w)[32]) {
    const float* Wg = Wm + (size_t)g * D * R + jc;
#pragma unroll
    for (int u4 = 0; u4 < 4; ++u4)
#pragma unroll
      for (int a = 0; a < 8; ++a) w[u4 * 8 + a] = __ldg(Wg + (size_t)(s + 4 * a + 32 * u4) * R);
  };
  float wq[32];
  if (early) {
    ptx::pdl_launch_dependents();  // the scan kernel may prefetch codes during the preceding kernel
    load_w(p.Wq, wq);              // the preceding kernel writes no W_H then
  }
  ptx::pdl_wait();  // q and the new K row come from the preceding kernel
  if (!early) {
    ptx::pdl_launch_dependents();  // the preceding kernel is complete: the scan kernel may read the cache
    load_w(p.Wq, wq);
  }
  const int L = clamp_seq(p.seq_lens[b], p.max_seq);
  const int nv = L > 0 ? NV : G;
  const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)g * G) * D;
  const T* kn = static_cast<const T*>(p.K) + (L > 0 ? token_slot<PAGED>(p, b, g, L - 1) : 0) * D;
  for (int t = tid; t < (L > 0 ? XV : QV); t += kEThreads) {
    const uint4 xv = t < QV ? reinterpret_cast<const uint4*>(qg)[t] : reinterpret_cast<const uint4*>(kn)[t - QV];
    float xe[EPV];
    Vec16<T>::convert(xv, xe);
    const int v = t * EPV / D;
#pragma unroll
    for (int e = 0; e < EPV; ++e) {
      const int i = (t * EPV + e) % D;
      xr[(v * 4 + (i & 3)) * kXS + (i >> 5) * 8 + ((i >> 2) & 7)] = xe[e];
    }
  }
  __syncthreads();
  auto residue_sum = [&](const float (&w)[32], int v) {
    const float* xs_ = xr + (v * 4 + s) * kXS;
    float P_[8];
#pragma unroll
    for (int u4 = 0; u4 < 4; ++u4) {
      const float4 x0 = reinterpret_cast<const float4*>(xs_ + u4 * 8)[0];
      const float4 x1 = reinterpret_cast<const float4*>(xs_ + u4 * 8)[1];
      const float xx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a) P_[a] = u4 == 0 ? xx[a] * w[u4 * 8 + a] : fmaf(xx[a], w[u4 * 8 + a], P_[a]);
    }
    const float q0 = P_[0] + P_[4], q1 = P_[1] + P_[5], q2 = P_[2] + P_[6], q3 = P_[3] + P_[7];
    sb[(v * 4 + s) * 32 + lane] = (q0 + q2) + (q1 + q3);
  };
#pragma unroll
  for (int v = 0; v < G; ++v) residue_sum(wq, v);
  if (L > 0) {
    if (p.Wk == nullptr) {
      residue_sum(wq, G);
    } else {
      float wk[32];
      load_w(p.Wk, wk);
      residue_sum(wk, G);
    }
  }
  __syncthreads();
  if (s == 0) {
    for (int v = 0; v < nv; ++v) {
      const float* sv = sb + v * 4 * 32;
      const float y = (sv[lane] + sv[2 * 32 + lane]) + (sv[32 + lane] + sv[3 * 32 + lane]);
      const unsigned bits = __ballot_sync(0xffffffffu, y > 0.f);
      if (lane == 0) {
        if (v < G) {
          const size_t o = ((size_t)b * p.Hq + (size_t)g * G + v) * NW + jw;
          p.qcode_ws[o] = bits;
          if (p.qcode_out) p.qcode_out[o] = bits;
        } else {
          p.codes[token_slot<PAGED>(p, b, g, L - 1) * NW + jw] = bits;  // the cache update
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// scan kernel
// ---------------------------------------------------------------------------
template <typename T, int NW, int G, bool PAGED>
__global__ void __launch_bounds__(kSThreads, 1) step_scan_kernel(const StepParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int R = NW * 32;
  constexpr int NB = G * R + 1;              // score values
  constexpr int NBP = nbins_padded(G, R);
  constexpr int BPT = (NBP + kSThreads - 1) / kSThreads;
  constexpr int PT = kPieceBytes / (NW * 4);  // tokens per piece
  constexpr int TPP = (PT + kSThreads - 1) / kSThreads;  // tokens per thread per piece
  constexpr int BULK_Q = NW >= 4 ? 1 : 4 / NW;  // tokens per 16 bytes
  static_assert(kMaxPieces <= 32, "one lane of warp 0 per piece");
  const ScanSmem S = scan_smem(G, NW);
  unsigned char* ring = smem + S.ring;
  uint32_t* lst = reinterpret_cast<uint32_t*>(smem + S.ring);  // the token-ordered list (the ring is free by then)
  uint16_t* Ds = reinterpret_cast<uint16_t*>(smem + S.D);
  int* hist = reinterpret_cast<int*>(smem + S.hist);  // counts, then each bin's exclusive prefix
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + S.mbar);  // pieces, then one nothing completes
  __shared__ int s_pre[kMaxB + 1];  // first chunk of batch b: Hkv * sum_{b' < b} ceil(L_b' / C)
  __shared__ int s_len[kMaxB];
  __shared__ int warp_sums[kSWarp];
  __shared__ __align__(16) uint32_t qc[(G + 1) * NW];  // the unit's query codes, then the new key's code
  __shared__ int s_abort, s_Bc, s_below;
  __shared__ int s_blk[PAGED ? kMaxChunkBlocks : 1];  // (paged) pool block of each block the chunk spans

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const StepGeom& geo = p.geo;
  const int C = geo.C;
  const bool test_expire = (p.flags & HATA_FLAG_TEST_EXPIRE_WAIT) != 0;

  if (tid == 0) {
    for (int i = 0; i < kMaxPieces + 1; ++i) ptx::mbar_init(&mbar[i], 1);
    ptx::fence_mbarrier_init();
    s_abort = 0;
  }
  // This kernel starts once the encode kernel has passed its own wait on the
  // preceding kernel (or, with early prefetch, at once): seq_lens and the cached
  // codes of slots [0, L - 1) are final, so they are read before this kernel waits
  // for the encode kernel; the query codes, the new key's code and every write come
  // after that wait.
  bool waited = false;

  // ---- chunk map: batch b holds Hkv * ceil(L_b / C) chunks, units b-major ----------
  {
    int cnt[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int b = 2 * tid + e;
      int L = 0;
      if (b < p.B) {
        const int raw = p.seq_lens[b];
        L = clamp_seq(raw, p.max_seq);
        s_len[b] = L;
        if (raw > p.max_seq) s_len[b] = -L - 1;  // flagged once the writes may start
      }
      cnt[e] = p.Hkv * ((L + C - 1) / C);
    }
    int total;
    const int ex = block_exclusive_scan<kSThreads>(cnt[0] + cnt[1], warp_sums, &total);
    if (2 * tid < p.B) s_pre[2 * tid] = ex;
    if (2 * tid + 1 < p.B) s_pre[2 * tid + 1] = ex + cnt[0];
    if (tid == 0) s_pre[p.B] = total;
  }
  __syncthreads();
  const int nchunks = s_pre[p.B];
  const uint64_t pol_stream = ptx::policy_evict_first();
  int enc_u = -1;         // unit whose query codes qc holds
  uint32_t par = 0u;      // bit pc: parity of the phase piece barrier pc completes next
  int last_np = 0;        // pieces issued for the latest chunk (drained on abort)
  uint32_t waited_mask = 0u;  // pieces of the latest chunk this thread has waited for

  for (int c = blockIdx.x; c < nchunks; c += gridDim.x) {
    // ---- locate the chunk: batch (largest b with s_pre[b] <= c), unit, index ---------
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= c) lo = mid;
      else hi = mid - 1;
    }
    const int b = lo, Ls = s_len[b], L = Ls < 0 ? -Ls - 1 : Ls;
    const int Pb = (L + C - 1) / C;
    const int loc = c - s_pre[b], g = loc / Pb, j = loc % Pb;
    const int u = b * p.Hkv + g;
    const int t0 = j * C, t1 = min(L, t0 + C), len = t1 - t0;
    const int np = (len + PT - 1) / PT;
    unsigned char* urec = p.rec + (size_t)u * geo.unit_bytes;  // unit histogram, then the chunk records
    unsigned char* rec = urec + geo.hist_bytes + (size_t)j * geo.slot_bytes;
    int32_t* rhdr = reinterpret_cast<int32_t*>(rec);
    const bool aborted_before = s_abort != 0;
    const bool own_last = L > 0 && t0 <= L - 1 && L - 1 < t1;

    // ---- 1. the chunk's codes into the ring: lane pc of warp 0 issues piece pc -------
    if constexpr (PAGED) {
      if (!aborted_before) {  // block-uniform: the chunk's block numbers, read in parallel
        const int blk0 = t0 >> p.block_shift, nblk = ((t1 - 1) >> p.block_shift) - blk0 + 1;
        for (int i = tid; i < nblk; i += kSThreads) {
          int pb = p.block_table[(size_t)b * p.max_blocks + blk0 + i];
          if ((unsigned)pb >= (unsigned)p.n_blocks) pb = -1;  // flagged below, block 0 used
          s_blk[i] = pb;
        }
        __syncthreads();
      }
    }
    if (warp == 0 && !aborted_before) {
      if (lane == 0) ptx::fence_proxy_async_smem();  // this CTA's earlier generic reads of the ring come first
      __syncwarp();
      const int pc = lane;
      if (pc < np) {
        const int ts = t0 + pc * PT, nt = min(PT, t1 - ts);
        const int nb = nt / BULK_Q * BULK_Q;  // tokens the copy moves (whole 16-byte units)
        ptx::mbar_arrive_expect_tx(&mbar[pc], (uint32_t)nb * NW * 4);
        if constexpr (PAGED) {
          // one copy per block segment; segments start on 16-token boundaries (bs >= 16)
          const int bsz = 1 << p.block_shift, blk0 = t0 >> p.block_shift;
          for (int x0 = 0; x0 < nb;) {
            const int t = ts + x0, seg = min(nb - x0, bsz - (t & (bsz - 1)));
            const size_t slot = (((size_t)max(0, s_blk[(t >> p.block_shift) - blk0]) * p.Hkv + g) << p.block_shift) |
                                (size_t)(t & (bsz - 1));
            ptx::bulk_g2s(ring + pc * kPieceBytes + (size_t)x0 * NW * 4, p.codes + slot * NW, (uint32_t)seg * NW * 4,
                          &mbar[pc], pol_stream);
            x0 += seg;
          }
        } else {
          if (nb)
            ptx::bulk_g2s(ring + pc * kPieceBytes, p.codes + token_slot<false>(p, b, g, ts) * NW,
                          (uint32_t)nb * NW * 4, &mbar[pc], pol_stream);
        }
      }
    }
    last_np = aborted_before ? last_np : np;
    waited_mask = aborted_before ? waited_mask : 0u;

    // ---- 2. the query codes (and the new key's code) from the encode kernel ---------
    if (!waited) {
      ptx::pdl_wait();  // the encode kernel is complete (and so is the kernel before it)
      ptx::pdl_launch_dependents();  // the tail kernel may read q and seq_lens before its own wait
      waited = true;
      if (blockIdx.x == 0 && tid < p.B && s_len[tid] < 0) set_status(p.status, HATA_ERR_INVALID_ARG);
    }
    if constexpr (PAGED) {
      if (!aborted_before) {
        const int blk0 = t0 >> p.block_shift, nblk = ((t1 - 1) >> p.block_shift) - blk0 + 1;
        for (int i = tid; i < nblk; i += kSThreads)
          if (s_blk[i] < 0) set_status(p.status, HATA_ERR_INVALID_ARG);
      }
    }
    if (!aborted_before && (u != enc_u || own_last)) {
      if (tid < G * NW) qc[tid] = p.qcode_ws[((size_t)b * p.Hq + (size_t)g * G) * NW + tid];
      if (own_last && tid >= G * NW && tid < (G + 1) * NW)
        qc[tid] = p.codes[token_slot<PAGED>(p, b, g, L - 1) * NW + (tid - G * NW)];
      enc_u = u;
    }
    for (int v = tid; v < BPT * kSThreads; v += kSThreads) hist[v] = 0;
    __syncthreads();

    // ---- 3. scores + histogram ------------------------------------------------------
    if (!aborted_before) {
      if (test_expire && !ptx::mbar_wait_bounded(&mbar[kMaxPieces], 0u, kTestWaitTries)) {
        set_status(p.status, HATA_ERR_TIMEOUT);  // test hook: the barrier nothing completes
        s_abort = 1;
      }
      GroupQuery<NW, G> gq;
      gq.init(qc);
      for (int pc = 0; pc < np; ++pc) {
        if (s_abort) break;
        if (!ptx::mbar_wait_spin(&mbar[pc], (par >> pc) & 1u, kWaitTries)) {
          set_status(p.status, HATA_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        par ^= 1u << pc;
        waited_mask |= 1u << pc;
        const int base = pc * PT, nt = min(PT, len - base), nb = nt / BULK_Q * BULK_Q;
        const uint32_t* buf = reinterpret_cast<const uint32_t*>(ring + pc * kPieceBytes);
        uint32_t kw[TPP][NW];
#pragma unroll
        for (int q = 0; q < TPP; ++q) {
          const int i = tid + q * kSThreads;
          if (i < nb) {
            if constexpr (NW >= 4) {
#pragma unroll
              for (int w4 = 0; w4 < NW / 4; ++w4) {
                const uint4 v4 = reinterpret_cast<const uint4*>(buf + (size_t)i * NW)[w4];
                kw[q][4 * w4] = v4.x;
                kw[q][4 * w4 + 1] = v4.y;
                kw[q][4 * w4 + 2] = v4.z;
                kw[q][4 * w4 + 3] = v4.w;
              }
            } else if constexpr (NW == 2) {
              const uint2 v2 = reinterpret_cast<const uint2*>(buf + (size_t)i * NW)[0];
              kw[q][0] = v2.x;
              kw[q][1] = v2.y;
            } else {
              kw[q][0] = buf[i];
            }
          } else if (i < nt) {  // the ragged end that a 16-byte copy cannot move
#pragma unroll
            for (int w = 0; w < NW; ++w) kw[q][w] = p.codes[token_slot<PAGED>(p, b, g, t0 + base + i) * NW + w];
          }
        }
#pragma unroll
        for (int q = 0; q < TPP; ++q) {
          const int i = tid + q * kSThreads;
          if (i < nt) {
            const int dv = gq.score(kw[q], qc, G);  // <= G * r by construction
            Ds[base + i] = (uint16_t)dv;
            atomicAdd(&hist[dv], 1);
          }
        }
      }
      __syncthreads();
      // the ring may hold the old code of slot L - 1 (the encode kernel writes the new
      // one while the copies run): rescore it with the new code
      if (own_last && tid == 0 && !s_abort) {
        uint32_t keyc[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) keyc[w] = qc[G * NW + w];
        const int d_new = gq.score(keyc, qc, G), d_old = Ds[L - 1 - t0];
        if (d_new != d_old) {
          Ds[L - 1 - t0] = (uint16_t)d_new;
          hist[d_old] -= 1;
          hist[d_new] += 1;
        }
      }
      if (tid < 16) Ds[len + tid] = (uint16_t)0xffffu;  // whole 16-score groups for the listing pass
      if (tid == 0) {
        s_Bc = NB;  // no crossing: every token is listed
        s_below = len;
      }
      __syncthreads();
    }

    // ---- 4. chunk record: cumulative histogram, bound, candidates sorted by score ----
    if (s_abort) {  // block-uniform (read after a barrier)
      if (tid == 0) {
        rhdr[0] = 0;
        rhdr[1] = 0;
        rhdr[2] = 0;
        rhdr[3] = (int32_t)((uint32_t)len | kAbortBit);
      }
      continue;  // no barrier inside: the next chunk only writes its header too
    }
    const int n = min(p.k, L);
    const long long fair = ((long long)n * len + L - 1) / L;
    const long long want_l = 2 * fair + 64;
    const int want = want_l < geo.cap ? (int)want_l : geo.cap;
    {
      uint16_t* rcum = reinterpret_cast<uint16_t*>(rec + geo.cum_off);
      uint32_t* uhist = reinterpret_cast<uint32_t*>(urec);
      int hv[BPT], local = 0;
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        hv[i] = hist[tid * BPT + i];
        local += hv[i];
      }
      int total;
      int run = block_exclusive_scan<kSThreads>(local, warp_sums, &total);
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        const int v = tid * BPT + i, before = run;
        run += hv[i];
        hist[v] = before;  // exclusive prefix: the first sorted position of score v
        if (v < NBP) {
          rcum[v] = (uint16_t)run;
          if (hv[i]) atomicAdd(&uhist[v], (uint32_t)hv[i]);  // the unit's histogram
        }
        if (before <= want && run > want) {  // the unique first bin whose count passes want
          s_Bc = v;
          s_below = before;
        }
      }
    }
    __syncthreads();
    const int Bc = s_Bc, below = s_below;
    const int tie_listed = Bc < NB ? want - below : 0;
    const int nlisted = below + tie_listed;
    {
      // token-ordered list (into the ring, free now): every score below Bc, and the
      // first tie_listed scores equal to Bc.  Each thread flags its 16 consecutive
      // scores as bit masks, one block scan places them.
      int lp_carry = 0, ep_carry = 0;
      for (int base = 0; base < len; base += 16 * kSThreads) {  // block-uniform trip count
        const int a = base + tid * 16;
        uint32_t mlt = 0u, meq = 0u;
        if (a < len) {  // a < len: both 16-byte loads stay inside the padded scores
          const uint4 v0 = reinterpret_cast<const uint4*>(Ds + a)[0];
          const uint4 v1 = reinterpret_cast<const uint4*>(Ds + a)[1];
          const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int d0 = (int)(w8[i] & 0xffffu), d1 = (int)(w8[i] >> 16);
            mlt |= (d0 < Bc ? 1u : 0u) << (2 * i) | (d1 < Bc ? 1u : 0u) << (2 * i + 1);
            meq |= (d0 == Bc ? 1u : 0u) << (2 * i) | (d1 == Bc ? 1u : 0u) << (2 * i + 1);
          }
        }
        int tot;
        const int pre = block_exclusive_scan<kSThreads>(__popc(mlt) | (__popc(meq) << 16), warp_sums, &tot);
        int lp = lp_carry + (pre & 0xffff), ep = ep_carry + (pre >> 16);
        uint32_t mm = mlt | meq;
        while (mm) {  // the thread's flagged scores, in token order
          const int i = __ffs(mm) - 1;
          mm &= mm - 1u;
          const int m_lt = __popc(mlt & ((1u << i) - 1u)), m_eq = __popc(meq & ((1u << i) - 1u));
          const int lpi = lp + m_lt, epi = ep + m_eq;
          const bool is_lt = (mlt >> i) & 1u;
          if (is_lt || epi < tie_listed)
            lst[lpi + min(epi, tie_listed)] = ((uint32_t)(is_lt ? 0 : 1) << 31) | (uint32_t)(a + i);
        }
        lp_carry += tot & 0xffff;
        ep_carry += tot >> 16;
      }
    }
    __syncthreads();
    {
      // sorted by score, equal scores in token order: each listed token first takes a
      // slot of its score's bin (any order), then its rank inside the bin by token index
      // (bins are small); the bin starts at the count of lower scores (hist, exclusive)
      uint32_t* rcand = reinterpret_cast<uint32_t*>(rec + geo.cand_off);
      uint32_t* tmp = lst + geo.cap;                         // bin slots: offsets, unordered in a bin
      int* fill = reinterpret_cast<int*>(tmp + geo.cap);     // next free slot of each bin
      for (int v = tid; v < NBP; v += kSThreads) fill[v] = hist[v];
      __syncthreads();
      for (int e = tid; e < nlisted; e += kSThreads) {
        const uint32_t ent = lst[e];
        const int off = (int)(ent & 0xffffu), d = (ent >> 31) ? Bc : (int)Ds[off];
        tmp[atomicAdd(&fill[d], 1)] = ((uint32_t)d << 16) | (uint32_t)off;
      }
      __syncthreads();
      for (int e = tid; e < nlisted; e += kSThreads) {
        const uint32_t me = tmp[e];
        const int d = (int)(me >> 16), b0 = hist[d], b1 = fill[d];
        int rk = 0;
        for (int x = b0; x < b1; ++x) rk += tmp[x] < me;  // same score: compares the offsets
        rcand[b0 + rk] = me;
      }
      if (tid == 0) {
        rhdr[0] = nlisted;
        rhdr[1] = Bc;
        rhdr[2] = tie_listed;
        rhdr[3] = len;
      }
    }
    __syncthreads();  // the ring, scores and histogram are free for the next chunk
  }

  if (!waited) ptx::pdl_launch_dependents();  // (no chunk here)
  if (s_abort && tid == 0) {
    // let the copies of the latest chunk that this thread did not wait for land (bounded)
    for (int pc = 0; pc < last_np; ++pc)
      if (!((waited_mask >> pc) & 1u)) ptx::mbar_wait_bounded(&mbar[pc], (par >> pc) & 1u, kWaitTries);
  }
}

// Selected tokens of a chunk whose candidate list stops short of the threshold T:
// every token scoring below T, then the first q scoring T, in token order, found by
// rescoring the chunk's codes from the cache (block-wide; 16 consecutive tokens a
// thread per pass, scored four at a time, once to count and once to place, which keeps
// the registers of this rare path low).  The token of selected rank rk in [lo, hi) goes
// to out[rk].
template <int NW, int G, bool PAGED>
__device__ __forceinline__ void rescore_chunk(const StepParams& p, int b, int g, int t0c, int lenc, int Tt, int q,
                                              int lo, int hi, int* out, const uint32_t* qcs, int* warp_sums) {
  const int tid = threadIdx.x;
  GroupQuery<NW, G> gq;
  gq.init(qcs);
  auto score_at = [&](int t) {  // score of chunk token t, or INT_MAX past the chunk
    if (t >= lenc) return INT_MAX;
    uint32_t kw[NW];
    load_code<NW>(p.codes + token_slot<PAGED>(p, b, g, t0c + t) * NW, kw);
    return gq.score(kw, qcs, G);
  };
  int lp_carry = 0, ep_carry = 0;
  for (int base = 0; base < lenc; base += 16 * kTThreads) {
    const int a = base + tid * 16;
    int lt = 0, eq = 0;
#pragma unroll 1
    for (int i0 = 0; i0 < 16; i0 += 4) {
      int dv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) dv[i] = score_at(a + i0 + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        lt += dv[i] < Tt;
        eq += dv[i] == Tt;
      }
    }
    int tot;
    const int pre = block_exclusive_scan<kTThreads>(lt | (eq << 16), warp_sums, &tot);
    int lp = lp_carry + (pre & 0xffff), ep = ep_carry + (pre >> 16);
#pragma unroll 1
    for (int i0 = 0; i0 < 16; i0 += 4) {
      int dv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) dv[i] = score_at(a + i0 + i);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (dv[i] < Tt || (dv[i] == Tt && ep < q)) {
          const int rk = lp + min(ep, q);
          if (rk >= lo && rk < hi) out[rk] = t0c + a + i0 + i;
        }
        lp += dv[i] < Tt;
        ep += dv[i] == Tt;
      }
    }
    lp_carry += tot & 0xffff;
    ep_carry += tot >> 16;
  }
}

// ---------------------------------------------------------------------------
// tail kernel
// ---------------------------------------------------------------------------
template <typename T, int NW, int G, bool PAGED>
__global__ void __launch_bounds__(kTThreads, 1) step_tail_kernel(const StepParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int D = kHeadDim;
  constexpr int ESZ = (int)sizeof(T);
  constexpr int R = NW * 32;
  constexpr int NB = G * R + 1;
  constexpr int NBP = nbins_padded(G, R);
  constexpr int BPT = (NBP + kTThreads - 1) / kTThreads;
  constexpr int EPV = 16 / ESZ;
  constexpr int RPR = D * ESZ / 16;          // 16-byte pieces per K or V row
  constexpr int RS = tail_row_stride(ESZ);  // row stride of the gathered rows (elements)
  constexpr int LT = 16;                     // lanes per row in the logits
  constexpr int LE = D / LT;                 // elements per lane in the logits (8)
  constexpr int PVG = kTThreads / (D / 2);   // row groups in P.V: thread = (column pair, row group)
  constexpr int OPT = (G * D + kTThreads - 1) / kTThreads;
  static_assert((2 * RPR) % 32 == 0, "a row's K and V pieces fill whole warps");

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CS = (int)ptx::cluster_nctarank();
  const int rank = (int)ptx::cluster_ctarank();
  const StepGeom& geo = p.geo;
  const int GB = p.GB;
  const TailSmem S = tail_smem(G, NW, ESZ, geo, GB, CS);
  unsigned char* urec = smem + S.rec;  // the unit's histogram, then its chunk records
  T* Kr = reinterpret_cast<T*>(smem + S.Kr);
  T* Vr = reinterpret_cast<T*>(smem + S.Vr);
  float* lg = reinterpret_cast<float*>(smem + S.lg);
  __nv_bfloat16* pbt = reinterpret_cast<__nv_bfloat16*>(smem + S.pb);  // (bf16) probabilities [8][GB + 8]
  int* rowtok = reinterpret_cast<int*>(smem + S.rowtok);
  long long* rowslot = reinterpret_cast<long long*>(smem + S.rowslot);  // (paged) cache slot of each row
  float* xp = reinterpret_cast<float*>(smem + S.xp);
  float* mslot = reinterpret_cast<float*>(smem + S.mslot);
  int* sst = reinterpret_cast<int*>(smem + S.sst);  // per chunk: selected before, selected, tie quota, covered
  uint32_t* qcs = reinterpret_cast<uint32_t*>(smem + S.qcs);
  uint64_t* mb = reinterpret_cast<uint64_t*>(smem + S.mbar);  // [0] records copy, [1] row gathers
  __shared__ int warp_sums[kNWarp];
  __shared__ int s_T, s_below, s_abort, s_uncovered;
  __shared__ float part[G * 2];

  const int u = blockIdx.x / CS;
  const int b = u / p.Hkv, g = u % p.Hkv;
  const uint32_t* uh = reinterpret_cast<const uint32_t*>(urec);
  auto rec = [&](int c) { return urec + geo.hist_bytes + (size_t)c * geo.slot_bytes; };
  auto hdr = [&](int c) { return reinterpret_cast<const int32_t*>(rec(c)); };
  auto cum = [&](int c) { return reinterpret_cast<const uint16_t*>(rec(c) + geo.cum_off); };
  auto cand = [&](int c) { return reinterpret_cast<const uint32_t*>(rec(c) + geo.cand_off); };

  // Before the wait: the scan kernel passed its own wait before it let this kernel
  // start, so seq_lens and q are final; only its records are not.
  ptx::cluster_arrive_relaxed();  // completed by the wait before the first remote store
  const int L = clamp_seq(p.seq_lens[b], p.max_seq);
  const int n = min(p.k, L);
  const int Pb = (L + geo.C - 1) / geo.C;
  if (tid == 0) {
    ptx::mbar_init(&mb[0], 1);
    ptx::mbar_init(&mb[1], kTThreads);
    ptx::fence_mbarrier_init();
    s_abort = 0;
  }
  for (int e = tid; e < G * D; e += kTThreads)
    xp[e] = to_f32<T>(static_cast<const T*>(p.q)[((size_t)b * p.Hq + (size_t)g * G) * D + e]);
  if (tid < G) {
    part[2 * tid] = -INFINITY;
    part[2 * tid + 1] = 0.f;
  }
  ptx::pdl_wait();  // the scan kernel's records are complete and visible
  ptx::pdl_launch_dependents();
  if (tid == 0 && Pb > 0) {
    const uint32_t bytes = geo.hist_bytes + (uint32_t)Pb * geo.slot_bytes;
    ptx::mbar_arrive_expect_tx(&mb[0], bytes);
    ptx::bulk_g2s(urec, p.rec + (size_t)u * geo.unit_bytes, bytes, &mb[0], ptx::policy_evict_first());
  }
  if (tid < G * NW) qcs[tid] = p.qcode_ws[((size_t)b * p.Hq + (size_t)g * G) * NW + tid];
  __syncthreads();  // the barrier initialisation is visible before anyone waits on it
  if (Pb > 0 && !ptx::mbar_wait_spin(&mb[0], 0u, kWaitTries)) {
    set_status(p.status, HATA_ERR_TIMEOUT);
    s_abort = 1;
  }
  __syncthreads();
  if (!s_abort)
    for (int c = tid; c < Pb; c += kTThreads)
      if ((uint32_t)hdr(c)[3] & kAbortBit) s_abort = 1;  // the scan gave up (its status is set)
  if (tid == 0) {
    s_T = NB - 1;
    s_below = 0;
    s_uncovered = 0;
  }
  __syncthreads();
  const bool active = !s_abort && n > 0;

  // ---- 5. threshold T (one scan of the unit histogram), each chunk's share ---------
  if (active) {
    int hv[BPT], local = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int v = tid * BPT + i;
      hv[i] = v < NBP ? (int)uh[v] : 0;
      local += hv[i];
    }
    int total;
    int run = block_exclusive_scan<kTThreads>(local, warp_sums, &total);
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      const int v = tid * BPT + i, before = run;
      run += hv[i];
      if (before < n && run >= n && v < NB) {  // the unique first score whose count reaches n
        s_T = v;
        s_below = before;
      }
    }
  }
  __syncthreads();
  const int Tt = s_T;
  if (active && warp == 0) {
    const int m = n - s_below;  // ties at T that are selected
    int tie_run = 0, sel_run = 0;
    for (int c0 = 0; c0 < Pb; c0 += 32) {  // lane c of each 32-chunk group
      const int c = c0 + lane;
      int bl = 0, te = 0;
      if (c < Pb) {
        bl = Tt > 0 ? (int)cum(c)[Tt - 1] : 0;
        te = (int)cum(c)[Tt] - bl;
      }
      int ti = te;  // inclusive scans of the ties and of the selected counts
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += y;
      }
      const int q = max(0, min(m - (tie_run + ti - te), te));
      const int sel = bl + q;
      int si = sel;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, si, o);
        if (lane >= o) si += y;
      }
      if (c < Pb) {
        // the list (sorted by score, ties in token order) holds the selection as its
        // first sel entries when T < Bc, or when T == Bc and the quota fits the ties listed
        const int32_t* h = hdr(c);
        const int Bc = h[1], tl = h[2];
        const bool covered = Tt < Bc || (Tt == Bc && q <= tl);
        sst[4 * c] = sel_run + si - sel;
        sst[4 * c + 1] = sel;
        sst[4 * c + 2] = q;
        sst[4 * c + 3] = covered ? 1 : 0;
        if (!covered && sel > 0) s_uncovered = 1;
      }
      tie_run += __shfl_sync(0xffffffffu, ti, 31);
      sel_run += __shfl_sync(0xffffffffu, si, 31);
    }
  }
  __syncthreads();

  // ---- 6. this CTA's selected ranks: rows, gather, attention partials ---------------
  const int r0 = active ? (int)((long long)rank * n / CS) : 0;
  const int r1 = active ? (int)((long long)(rank + 1) * n / CS) : 0;
  int32_t* ix = p.idx_out ? p.idx_out + (size_t)u * p.k : nullptr;
  float oacc[OPT];
#pragma unroll
  for (int q = 0; q < OPT; ++q) oacc[q] = 0.f;
  // Attention per gather batch, in the exp2 domain (logits scaled by scale * log2 e):
  // logits by LT lanes per row into lg, the batch's per-head maximum, p = 2^(logit - m)
  // in place, then P.V by (column pair, row group) threads whose partial sums meet in
  // shared memory and fold into oacc against the running per-head (maximum, sum).
  __shared__ int s_bmax[G];         // the batch's maximum logit per head (order-preserving int)
  __shared__ float s_wsum[kNWarp];  // (bf16) each warp's sum of its head's probabilities
  const int PS = tail_p_stride(GB);
  // (bf16) lane (gq, cq): Q fragments of head gq (zero beyond G) for the logits' A operand, and
  // the running weighted V sums of head gq, columns 8 w + 2 cq, 8 w + 2 cq + 1 (rows gq + 8 unused)
  const int gq = lane >> 2, cq = lane & 3;
  uint32_t qa0[ESZ == 2 ? D / 16 : 1], qa2[ESZ == 2 ? D / 16 : 1];
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (ESZ == 2) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      qa0[ks] = 0u;
      qa2[ks] = 0u;
      if (gq < G) {
        const float* xq_ = xp + gq * D + 16 * ks + 2 * cq;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(xq_[0], xq_[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(xq_[8], xq_[9]);
        qa0[ks] = *reinterpret_cast<const uint32_t*>(&lo);
        qa2[ks] = *reinterpret_cast<const uint32_t*>(&hi);
      }
    }
  }
  __shared__ float s_m[G], s_l[G];  // running maximum and sum per head
  __shared__ float s_redl[PVG * G];
  if (tid < G) {
    s_bmax[tid] = ord_of(-INFINITY);
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
  }
  uint32_t gphase = 0;
  const T* Kg = static_cast<const T*>(p.K);
  const T* Vg = static_cast<const T*>(p.V);
  // a row index outside [0, L) is never expected: it is flagged and row 0 used instead
  auto checked = [&](int t) {
    if ((unsigned)t >= (unsigned)L) {
      set_status(p.status, HATA_ERR_INVALID_ARG);
      t = 0;
    }
    return t;
  };
  for (int cur = r0; cur < r1; cur += GB) {  // block-uniform
    const int end = min(r1, cur + GB), nr = end - cur;
    // chunks whose list stops short of T: rescore from the cache (block-wide, in token order)
    for (int c = 0; s_uncovered && c < Pb; ++c) {
      const int sb0 = sst[4 * c], sel = sst[4 * c + 1], q = sst[4 * c + 2];
      if (sst[4 * c + 3] || sb0 + sel <= cur || sb0 >= end) continue;  // block-uniform
      rescore_chunk<NW, G, PAGED>(p, b, g, c * geo.C, min(geo.C, L - c * geo.C), Tt, q, max(0, cur - sb0),
                                  min(sel, end - sb0), rowtok + sb0 - cur, qcs, warp_sums);
    }
    // covered chunks: rank rk of chunk c is entry rk - sb0 of its sorted list
    for (int i = tid; i < nr; i += kTThreads) {
      const int rk = cur + i;
      int c = 0;  // the chunk holding selected rank rk (chunks of an empty share are skipped)
      for (int x = 1; x < Pb; ++x)
        if (sst[4 * x] <= rk) c = x;
      if (sst[4 * c + 3]) {
        const uint32_t ent = cand(c)[min(rk - sst[4 * c], geo.cap - 1)];
        rowtok[i] = c * geo.C + (int)(ent & 0xffffu);
      }
    }
    __syncthreads();
    // indices in ascending token order (selected ranks of a chunk follow its tokens)
    if (ix) {
      for (int i = tid; i < nr; i += kTThreads) {
        const int rk = cur + i;
        int c = 0;
        for (int x = 1; x < Pb; ++x)
          if (sst[4 * x] <= rk) c = x;
        int pos = rk;
        if (sst[4 * c + 3]) {  // a sorted list: the rank among the chunk's selected tokens by token index
          const uint32_t* lst = cand(c);
          const int sel = min(sst[4 * c + 1], geo.cap), me = rk - sst[4 * c];
          const uint32_t mo = lst[min(me, geo.cap - 1)] & 0xffffu;
          int before = 0;
          for (int e = 0; e < sel; ++e) before += (lst[e] & 0xffffu) < mo;
          pos = sst[4 * c] + before;
        }
        ix[pos] = rowtok[i];
      }
    }
    if constexpr (PAGED) {
      for (int i = tid; i < nr; i += kTThreads) rowslot[i] = (long long)token_slot<true>(p, b, g, checked(rowtok[i]));
      __syncthreads();
    }
    for (int e = tid; e < nr * 2 * RPR; e += kTThreads) {
      const int r = e / (2 * RPR), w = e % (2 * RPR);
      size_t slot;
      if constexpr (PAGED) slot = (size_t)rowslot[r];
      else slot = token_slot<false>(p, b, g, checked(rowtok[r]));
      const size_t row = slot * D;
      if (w < RPR) ptx::cp_async16(Kr + (size_t)r * RS + w * EPV, Kg + row + w * EPV);
      else ptx::cp_async16(Vr + (size_t)r * RS + (w - RPR) * EPV, Vg + row + (w - RPR) * EPV);
    }
    ptx::cp_async_mbar_arrive_noinc(&mb[1]);
    if (!ptx::mbar_wait_spin(&mb[1], gphase & 1u, kWaitTries)) {
      set_status(p.status, HATA_ERR_TIMEOUT);
      s_abort = 1;
    }
    ++gphase;
    __syncthreads();
    if (s_abort) break;  // block-uniform (read after the barrier)

    if constexpr (ESZ == 2) {
      // ---- tensor cores (bf16): S = Q K^T and O += P V as mma.m16n8k16, heads as the rows ----
      const int nr16 = (nr + 15) & ~15;
      // logits: warp w takes the 8-token groups w, w + 16, ...; lane (gq, cq) gets head gq's
      // logits of tokens 2 cq and 2 cq + 1 of the group
      float mxl = -INFINITY;
      for (int t0 = warp * 8; t0 < nr; t0 += kNWarp * 8) {  // warp-uniform
        const __nv_bfloat16* krow =
            reinterpret_cast<const __nv_bfloat16*>(Kr) + (size_t)min(t0 + gq, nr - 1) * RS + 2 * cq;
        float c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t b0 = *reinterpret_cast<const uint32_t*>(krow + 16 * ks);
          const uint32_t b1 = *reinterpret_cast<const uint32_t*>(krow + 16 * ks + 8);
          mma_16816_top(c4, qa0[ks], qa2[ks], b0, b1);
        }
        if (gq < G)
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            const int t = t0 + 2 * cq + tt;
            if (t < nr) {
              const float lv = c4[tt] * p.scale_log2;
              lg[gq * GB + t] = lv;
              mxl = fmaxf(mxl, lv);
            }
          }
      }
      mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, 1));
      mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, 2));
      if (cq == 0 && gq < G && mxl != -INFINITY) atomicMax(&s_bmax[gq], ord_of(mxl));
      // V rows [nr, nr16) enter the last k-step with p = 0: make them finite (zero)
      for (int e = tid; e < (nr16 - nr) * (D / 8); e += kTThreads)
        *reinterpret_cast<uint4*>(Vr + (size_t)(nr + e / (D / 8)) * RS + (e % (D / 8)) * 8) = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
      // probabilities: warp w takes head w % G, rows (w / G) * 32 + lane, ...; bf16 into the P
      // tile (zero for rows [nr, nr16)), and the head's sum of the rounded values
      {
        const int h = warp % G, wph = kNWarp / G;
        const float mn = fmaxf(s_m[h], float_of_ord(s_bmax[h]));
        float sm = 0.f;
        for (int t = (warp / G) * 32 + lane; t < nr16; t += 32 * wph) {
          const __nv_bfloat16 pv = __float2bfloat16_rn(t < nr ? exp2f(lg[h * GB + t] - mn) : 0.f);
          pbt[h * PS + t] = pv;
          sm += __bfloat162float(pv);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
        if (lane == 0) s_wsum[warp] = sm;
      }
      __syncthreads();
      // P.V into output columns 8 w .. 8 w + 7: the running output is rescaled first
      {
        const float m_old = gq < G ? s_m[gq] : 0.f;
        const float mn = gq < G ? fmaxf(m_old, float_of_ord(s_bmax[gq])) : 0.f;
        const float al = gq < G && m_old != -INFINITY ? exp2f(m_old - mn) : 0.f;
        acc[0] *= al;
        acc[1] *= al;
        const __nv_bfloat16* ph = pbt + min(gq, G - 1) * PS + 2 * cq;
        const __nv_bfloat16* vcol = reinterpret_cast<const __nv_bfloat16*>(Vr) + (size_t)(lane & 15) * RS + 8 * warp;
        for (int ks = 0; ks < nr16 / 16; ++ks) {
          const uint32_t a0 = gq < G ? *reinterpret_cast<const uint32_t*>(ph + 16 * ks) : 0u;
          const uint32_t a2 = gq < G ? *reinterpret_cast<const uint32_t*>(ph + 16 * ks + 8) : 0u;
          uint32_t b0, b1;
          ldsm_x2_trans(b0, b1, vcol + (size_t)16 * ks * RS);
          mma_16816_top(acc, a0, a2, b0, b1);
        }
      }
      __syncthreads();  // every thread has read the running maxima, the P tile and the V rows
      if (tid < G) {
        const int h = tid;
        const float m_old = s_m[h];
        const float mn = fmaxf(m_old, float_of_ord(s_bmax[h]));
        const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - mn);
        float ls = 0.f;
        for (int w = h; w < kNWarp; w += G) ls += s_wsum[w];
        s_l[h] = s_l[h] * alpha + ls;
        s_m[h] = mn;
        s_bmax[h] = ord_of(-INFINITY);
      }
    } else {
      // logits: LT lanes per row, LE consecutive elements each (xp is ready long before)
      {
        const int sgi = lane % LT;
        float xq[G][LE];
  #pragma unroll
        for (int h = 0; h < G; ++h)
  #pragma unroll
          for (int e = 0; e < LE; e += 4) {
            const float4 a = *reinterpret_cast<const float4*>(xp + h * D + sgi * LE + e);
            xq[h][e] = a.x;
            xq[h][e + 1] = a.y;
            xq[h][e + 2] = a.z;
            xq[h][e + 3] = a.w;
          }
        float mx[G];
  #pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
        for (int rb = warp * (32 / LT); rb < nr; rb += kNWarp * (32 / LT)) {  // warp-uniform trip count
          const int r = rb + lane / LT;
          const bool valid = r < nr;
          const T* kr = Kr + (size_t)(valid ? r : 0) * RS + sgi * LE;
          float kv[LE];
          if constexpr (ESZ == 2) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(kr);
            const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
              kv[2 * e] = f.x;
              kv[2 * e + 1] = f.y;
            }
          } else {
  #pragma unroll
            for (int e = 0; e < LE; e += 4) {
              const float4 f = *reinterpret_cast<const float4*>(kr + e);
              kv[e] = f.x;
              kv[e + 1] = f.y;
              kv[e + 2] = f.z;
              kv[e + 3] = f.w;
            }
          }
          float acc[G];
  #pragma unroll
          for (int h = 0; h < G; ++h) {
            float a = xq[h][0] * kv[0];
  #pragma unroll
            for (int e = 1; e < LE; ++e) a = fmaf(xq[h][e], kv[e], a);
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
  #pragma unroll
        for (int h = 0; h < G; ++h) {
          float m = mx[h];
  #pragma unroll
          for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0 && m != -INFINITY) atomicMax(&s_bmax[h], ord_of(m));
        }
      }
      __syncthreads();
      // probabilities against the new running maximum of each head
      for (int e = tid; e < G * nr; e += kTThreads) {
        const int h = e / nr, i = e - h * nr;
        const float mn = fmaxf(s_m[h], float_of_ord(s_bmax[h]));
        lg[h * GB + i] = exp2f(lg[h * GB + i] - mn);
      }
      __syncthreads();
      // P.V: thread (column pair cp, row group rg) over rows rg, rg + PVG, ...; the PVG partial
      // sums of each output meet in the K rows' buffer (free once the logits are done)
      {
        const int cp = tid % (D / 2), rg = tid / (D / 2);
        float pacc[G][2], lsum[G];
  #pragma unroll
        for (int h = 0; h < G; ++h) pacc[h][0] = pacc[h][1] = lsum[h] = 0.f;
  #pragma unroll 4
        for (int r = rg; r < nr; r += PVG) {
          float v0, v1;
          if constexpr (ESZ == 2) {
            const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Vr + (size_t)r * RS)[cp]);
            v0 = f.x;
            v1 = f.y;
          } else {
            const float2 f = reinterpret_cast<const float2*>(Vr + (size_t)r * RS)[cp];
            v0 = f.x;
            v1 = f.y;
          }
  #pragma unroll
          for (int h = 0; h < G; ++h) {
            const float pr = lg[h * GB + r];
            pacc[h][0] = fmaf(pr, v0, pacc[h][0]);
            pacc[h][1] = fmaf(pr, v1, pacc[h][1]);
            lsum[h] += pr;
          }
        }
        float* red = reinterpret_cast<float*>(Kr);  // [PVG][G][D]
  #pragma unroll
        for (int h = 0; h < G; ++h)
          reinterpret_cast<float2*>(red + ((size_t)rg * G + h) * D)[cp] = make_float2(pacc[h][0], pacc[h][1]);
        if (cp == 0)
  #pragma unroll
          for (int h = 0; h < G; ++h) s_redl[rg * G + h] = lsum[h];
        __syncthreads();
  #pragma unroll
        for (int q = 0; q < OPT; ++q) {
          const int e = tid + q * kTThreads;
          if (e < G * D) {
            const int h = e / D, i = e % D;
            const float m_old = s_m[h];
            const float mn = fmaxf(m_old, float_of_ord(s_bmax[h]));
            const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - mn);
            float sum = 0.f;
  #pragma unroll
            for (int j = 0; j < PVG; ++j) sum += red[((size_t)j * G + h) * D + i];
            oacc[q] = fmaf(oacc[q], alpha, sum);
          }
        }
        __syncthreads();  // every thread has read the running maxima and the partial sums
        if (tid < G) {
          const int h = tid;
          const float m_old = s_m[h];
          const float mn = fmaxf(m_old, float_of_ord(s_bmax[h]));
          const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - mn);
          float ls = 0.f;
  #pragma unroll
          for (int j = 0; j < PVG; ++j) ls += s_redl[j * G + h];
          s_l[h] = s_l[h] * alpha + ls;
          s_m[h] = mn;
          s_bmax[h] = ord_of(-INFINITY);
        }
      }
    }
  }
  __syncthreads();
  if constexpr (ESZ == 2) {  // the accumulators' columns into oacc's layout, through the K rows' buffer
    float* red = reinterpret_cast<float*>(Kr);  // [G][D]
    if (gq < G) {
      red[gq * D + 8 * warp + 2 * cq] = acc[0];
      red[gq * D + 8 * warp + 2 * cq + 1] = acc[1];
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < OPT; ++q) {
      const int e = tid + q * kTThreads;
      if (e < G * D) oacc[q] = red[e];
    }
    __syncthreads();
  }
  if (tid < G) {  // this CTA's partial: running maximum and sum per head (oacc holds the weighted V sums)
    part[2 * tid] = s_m[tid];
    part[2 * tid + 1] = s_l[tid];
  }
  __syncthreads();
  if (ix && rank == 0) {
    for (int jx = n + tid; jx < p.k; jx += kTThreads) ix[jx] = -1;
    if (!active)
      for (int jx = tid; jx < min(n, p.k); jx += kTThreads) ix[jx] = -1;
  }

  // ---- 7. partials to the CTAs owning each output column, then merge ---------------
  const int mc = (G * D + CS - 1) / CS, stride = mc + 2 * G;
  ptx::cluster_wait();  // every CTA of the cluster has started
  if (s_abort) {  // no partial from this CTA: an empty one
#pragma unroll
    for (int q = 0; q < OPT; ++q) oacc[q] = 0.f;
  }
#pragma unroll
  for (int q = 0; q < OPT; ++q) {
    const int e = tid + q * kTThreads;
    if (e < G * D) {
      const int owner = e / mc, col = e % mc;
      ptx::st_dsmem_f32(ptx::dsmem_addr(&mslot[rank * stride + 2 * G + col], owner), oacc[q]);
    }
  }
  for (int e = tid; e < 2 * G * CS; e += kTThreads) {
    const int owner = e / (2 * G), w = e % (2 * G);
    float v = part[w];
    if (s_abort) v = (w & 1) ? 0.f : -INFINITY;
    ptx::st_dsmem_f32(ptx::dsmem_addr(&mslot[rank * stride + w], owner), v);
  }
  ptx::cluster_sync();  // every CTA holds the partials of its columns; every records copy has landed
  if (rank == 0 && Pb > 0)  // the unit's histogram starts at zero for the next call
    for (int v = tid; v < NBP; v += kTThreads) reinterpret_cast<uint32_t*>(p.rec + (size_t)u * geo.unit_bytes)[v] = 0u;
  for (int col = tid; col < mc; col += kTThreads) {
    const int e = rank * mc + col;
    if (e < G * D) {
      const int h = e / D;
      // every source's (max, sum, column) first, then the log-sum-exp merge (no branches,
      // so the loads of all sources are in flight together)
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
#pragma unroll
      for (int c = 0; c < kMaxCS; ++c) {
        const float w = mv[c] == -INFINITY ? 0.f : exp2f(mv[c] - M);
        l = fmaf(lv[c], w, l);
        o = fmaf(ov[c], w, o);
      }
      static_cast<T*>(p.out)[((size_t)b * p.Hq + (size_t)g * G + h) * D + (e % D)] =
          from_f32<T>(l > 0.f ? o / l : 0.f);
    }
  }
  if (s_abort) {
    // nothing may land in shared memory after the CTA exits
    ptx::cp_async_wait_all();
    if (tid == 0 && Pb > 0) ptx::mbar_wait_bounded(&mb[0], 0u, kWaitTries);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct Plan {
  bool ok;
  StepGeom geo;
  int scan_grid, CS, GB;
  size_t scan_smem, tail_smem, ws_bytes;
};

int device_sms() {
  static std::mutex mu;
  static std::map<int, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    sms = 0;
  }
  cache[dev] = sms;
  return sms;
}

// Allow the largest dynamic shared memory (the device's opt-in limit minus the kernel's
// static shared memory) and non-portable cluster sizes, once per kernel and device.
// Returns the dynamic bytes allowed in *max_dyn.
cudaError_t configure(const void* kern, int* max_dyn) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, std::pair<cudaError_t, int>> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find({kern, dev});
  if (it == done.end()) {
    int optin = 0, dyn = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
    if (e == cudaSuccess) {
      dyn = optin - (int)fa.sharedSizeBytes;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    }
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    // every kernel of the step asks for the largest shared-memory carveout, so an SM that
    // runs one of them can take a CTA of the next one without reconfiguring
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) (void)cudaGetLastError();
    it = done.emplace(std::make_pair(kern, dev), std::make_pair(e, dyn)).first;
  }
  if (max_dyn) *max_dyn = it->second.second;
  return it->second.first;
}

int active_clusters(const void* kern, int CS, size_t smem) {
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
  cfg.blockDim = dim3(kTThreads, 1, 1);
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

template <typename T, int NW, int G>
Plan make_plan_t(const hata_dims_t& d, int k) {
  Plan pl{};
  const int sms = device_sms();
  if (sms < 1 || d.batch > kMaxB) return pl;
  const int R = NW * 32, esize = (int)sizeof(T);
  const long long U = (long long)d.batch * d.n_kv_heads;
  const int cmax = kRingBytes / (NW * 4);
  // chunk slots per unit: spread the units over every SM, chunks of at least kMinChunk
  // tokens and at most one ring
  const long long scan_sms = sms;  // the encode CTAs are small enough to share SMs with the scan
  long long P = (d.max_seq + cmax - 1) / cmax;
  if (U < scan_sms) P = std::max<long long>(P, scan_sms / U);
  P = std::min<long long>(P, std::max<long long>(1, (d.max_seq + kMinChunk - 1) / kMinChunk));
  P = std::max<long long>(P, (d.max_seq + cmax - 1) / cmax);
  long long C = ((d.max_seq + P - 1) / P + 15) / 16 * 16;
  if (C > cmax) C = cmax / 16 * 16;
  P = (d.max_seq + C - 1) / C;
  StepGeom geo{};
  geo.C = (int)C;
  geo.P = (int)P;
  geo.nbp = nbins_padded(G, R);
  // list capacity: the tokens a chunk can list (a list stopping short of the threshold
  // is rescored in the tail); the scan sorts it in its ring: two lists and a bin counter each
  geo.cap = (int)((std::min<long long>(C, (long long)k + 64) + 3) / 4 * 4);
  geo.cap = std::min(geo.cap, (kRingBytes - geo.nbp * 4) / 8 / 4 * 4);
  geo.cum_off = 16;
  geo.cand_off = (uint32_t)(16 + geo.nbp * 2);
  geo.slot_bytes = (uint32_t)(geo.cand_off + geo.cap * 4);
  geo.hist_bytes = (uint32_t)(geo.nbp * 4);
  geo.unit_bytes = geo.hist_bytes + (uint32_t)P * geo.slot_bytes;
  if ((long long)P * geo.slot_bytes > 0x7fffffffLL || U > 0x7fffffffLL / geo.unit_bytes) return pl;
  pl.geo = geo;
  pl.scan_grid = (int)std::min<long long>(U * P, scan_sms);
  pl.scan_smem = (size_t)scan_smem(G, NW).total;
  int dyn_scan = 0, dyn_scan_p = 0, dyn_tail = 0, dyn_tail_p = 0;
  if (configure((const void*)step_scan_kernel<T, NW, G, false>, &dyn_scan) != cudaSuccess ||
      configure((const void*)step_scan_kernel<T, NW, G, true>, &dyn_scan_p) != cudaSuccess)
    return pl;
  if (pl.scan_smem > (size_t)std::min(dyn_scan, dyn_scan_p)) return pl;
  // tail: the largest cluster (<= 16) that puts every unit in one wave, else the
  // largest that fits at all; the gather batch takes the shared memory that is left
  const void* tail = (const void*)step_tail_kernel<T, NW, G, false>;
  if (configure(tail, &dyn_tail) != cudaSuccess ||
      configure((const void*)step_tail_kernel<T, NW, G, true>, &dyn_tail_p) != cudaSuccess)
    return pl;
  const int tail_limit = std::min(dyn_tail, dyn_tail_p);
  int bestCS = 0, bestGB = 0;
  size_t best_smem = 0;
  for (int CS = kMaxCS; CS >= 1; --CS) {
    if (CS > 1 && (long long)CS * 2 > std::max<long long>(2, std::min<long long>(k, d.max_seq))) continue;
    int GB = kMaxGB;
    while (GB >= 32 && tail_smem(G, NW, esize, geo, GB, CS).total > tail_limit) GB -= 32;
    if (GB < 32) continue;
    const size_t sm = (size_t)tail_smem(G, NW, esize, geo, GB, CS).total;
    const int act = active_clusters(tail, CS, sm);
    if (act < 1) continue;
    if (act >= U || CS == 1) {
      bestCS = CS;
      bestGB = GB;
      best_smem = sm;
      break;
    }
  }
  if (!bestCS) return pl;
  pl.CS = bestCS;
  pl.GB = bestGB;
  pl.tail_smem = best_smem;
  pl.ws_bytes = align_up((size_t)U * geo.unit_bytes, kAlign) + align_up((size_t)d.batch * d.n_q_heads * NW * 4, kAlign);
  pl.ok = true;
  return pl;
}

template <template <typename, int, int> class F, typename... A>
auto dispatch(const hata_dims_t& d, A&&... a) -> decltype(F<float, 1, 1>::run(a...)) {
  const int G = d.n_q_heads / d.n_kv_heads, NW = d.hash_bits / 32;
#define HATA_G(T, NW_)                      \
  switch (G) {                              \
    case 1: return F<T, NW_, 1>::run(a...); \
    case 2: return F<T, NW_, 2>::run(a...); \
    case 4: return F<T, NW_, 4>::run(a...); \
    case 8: return F<T, NW_, 8>::run(a...); \
  }                                         \
  break;
#define HATA_NW(T)       \
  switch (NW) {          \
    case 1: HATA_G(T, 1) \
    case 2: HATA_G(T, 2) \
    case 4: HATA_G(T, 4) \
    case 8: HATA_G(T, 8) \
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

template <typename T, int NW, int G, bool PAGED>
cudaError_t launch_t(const Plan& pl, const hata_dims_t& d, const StepParams& prm, cudaStream_t st) {
  auto enc = step_encode_kernel<T, NW, G, PAGED>;
  auto scan = step_scan_kernel<T, NW, G, PAGED>;
  auto tail = step_tail_kernel<T, NW, G, PAGED>;
  cudaError_t e = configure((const void*)enc, nullptr);
  if (e == cudaSuccess) e = configure((const void*)scan, nullptr);
  if (e == cudaSuccess) e = configure((const void*)tail, nullptr);
  if (e != cudaSuccess) return e;
  // all three are launched with programmatic dependent launch: each may start while
  // the kernel before it runs and waits (griddepcontrol.wait) before using its results
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(d.batch * d.n_kv_heads * NW), 1, 1);
  cfg.blockDim = dim3(kEThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, enc, prm);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)pl.scan_grid, 1, 1);
  cfg.blockDim = dim3(kSThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.scan_smem;
  e = cudaLaunchKernelEx(&cfg, scan, prm);
  if (e != cudaSuccess) return e;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = pl.CS;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(d.batch * d.n_kv_heads * pl.CS), 1, 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.tail_smem;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, tail, prm);
}

template <typename T, int NW, int G>
struct LaunchFn {
  static cudaError_t run(const Plan& pl, const hata_dims_t& d, const StepParams& prm, cudaStream_t st) {
    return prm.block_table ? launch_t<T, NW, G, true>(pl, d, prm, st) : launch_t<T, NW, G, false>(pl, d, prm, st);
  }
  static cudaError_t fail() { return cudaErrorNotSupported; }
};

Plan make_plan_uncached(const hata_dims_t& d, int k) {
  const int G = d.n_q_heads / d.n_kv_heads, NW = d.hash_bits / 32;
  if (G != 1 && G != 2 && G != 4 && G != 8) return Plan{};
  if ((long long)d.max_seq * NW % 4 != 0) return Plan{};  // 16-byte aligned per-unit code slabs
  return dispatch<PlanFn>(d, d, k);
}

// Plans are cached per (device, shape, budget): the first call for a shape sets kernel
// attributes and queries cluster occupancy; later calls (including ones made while a
// stream is being captured into a CUDA graph) only look it up.
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

bool split_step_applies(const hata_dims_t& d, int k) { return make_plan(d, k).ok; }

size_t split_step_ws_bytes(const hata_dims_t& d, int k) {
  const Plan pl = make_plan(d, k);
  return pl.ok ? pl.ws_bytes : 0;
}

cudaError_t launch_split_step(const hata_dims_t& d, const WsLayout& L, const void* q, const void* K, const void* V,
                              const float* W, const float* Wk, uint32_t* codes, const int32_t* seq_lens, int k,
                              float scale, void* out, uint32_t* qcode_out, int32_t* idx_out, const PagedCache* pg,
                              char* ws, cudaStream_t st) {
  const Plan pl = make_plan(d, k);
  if (!pl.ok || L.fused_bytes < pl.ws_bytes) return cudaErrorNotSupported;
  StepParams prm{};
  prm.q = q;
  prm.K = K;
  prm.V = V;
  prm.Wq = W;
  prm.Wk = Wk == W ? nullptr : Wk;
  prm.codes = codes;
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.qcode_out = qcode_out;
  prm.idx_out = idx_out;
  prm.status = reinterpret_cast<uint32_t*>(ws + L.status);
  prm.rec = reinterpret_cast<unsigned char*>(ws + L.fused);
  prm.qcode_ws = reinterpret_cast<uint32_t*>(ws + L.fused + align_up((size_t)d.batch * d.n_kv_heads *
                                                                        pl.geo.unit_bytes, kAlign));
  prm.B = d.batch;
  prm.Hq = d.n_q_heads;
  prm.Hkv = d.n_kv_heads;
  prm.max_seq = d.max_seq;
  prm.k = k;
  prm.flags = d.flags;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.geo = pl.geo;
  prm.GB = pl.GB;
  prm.block_table = pg ? pg->block_table : nullptr;
  prm.block_shift = pg ? pg->block_shift : 0;
  prm.n_blocks = pg ? pg->n_blocks : 0;
  prm.max_blocks = pg ? pg->max_blocks : 0;
  return dispatch<LaunchFn>(d, pl, d, prm, st);
}

}  // namespace hata
