// Causal prefill attention on the 5th-generation tensor cores, with the key
// HashEncode fused in ("HATA" paper notes, 整体框架: in the prefill phase the
// prompt is processed with full attention while every key is hashed and its code
// cached, so that decode can select by Hamming distance; 实验: that encode costs
// under 1% of the time).
//
//   out[b][h][t] = sum_{s <= t} softmax_s(scale * q[b][h][t] . K[b][g][s]) V[b][g][s]
//   codes[b][g][s] = pack(K[b][g][s] . W_H[g] > 0)        (when codes != NULL)
// for t, s < L_b, with g = h / G.
//
// One CTA of ten warps per (query tile of 128 positions, query head, batch),
// heaviest tiles launched first.  For key tiles j = 0 .. i (i = the query tile):
//   * warp 9 (one lane) streams Q once and K / V tiles through 3-deep rings (TMA,
//     128-byte swizzle), refilling a stage once the MMAs reading it are done;
//   * warp 8 (one lane) issues S_j = Q K_j^T (M = N = 128, K = 16 per MMA) into one
//     of three TMEM score buffers and, once P_j is written, O += P_j V_j into the
//     TMEM output accumulator, with P_j read from TMEM and V as an MN-major operand
//     (no transpose);
//   * warps 0-7 are two softmax warpgroups over the same 128 query rows (TMEM lane =
//     row).  Warpgroup w reads keys 64 w .. 64 w + 63 of S_j, finds their maximum and
//     exchanges it with the other warpgroup through a TMEM column (both then hold the
//     same row maximum m), computes p = 2^(s * scale * log2 e - m) for its keys,
//     stores it as bf16 pairs over the first half of the scores it read (the A operand
//     of PV_j), and sums it.  A buffer is
//     reused three tiles later, after PV_j has read it, so the softmax of tile j
//     never waits for PV_{j-1}.  The running maximum m used for O moves only when a
//     row's maximum exceeds it by more than 2^8; then each warpgroup rescales its half
//     of O's row in TMEM once PV_{j-1} has landed (PV_j is issued after).  The
//     diagonal tile masks keys after the row.
// On the diagonal tile the key tile K_i is already in shared memory: the CTA of
// the group's first query head copies W_H^T (three bf16 parts, split once per
// call into the workspace) into the freed V ring and runs Y = K_i W_H as
// three accumulating MMAs of N = r into TMEM; warpgroup 0 turns Y into code words
// after writing its output columns.  Only the summation order differs from an
// fp32 dot product, so a code bit can differ from the exact sign only where |y|
// is within fp32 rounding of zero.
//
// Every wait is bounded; on expiry the kernel records HATA_ERR_TIMEOUT in the
// workspace's status word, stops issuing work, waits (bounded) for the copies and
// MMAs it issued, frees its TMEM and returns.
#include <algorithm>
#include <map>
#include <mutex>

#include "hata_kernels.cuh"
#include "hata_tc.cuh"

namespace hata {

namespace {

constexpr int kPfThreads = 320;  // warps 0-7: two softmax / epilogue warpgroups, 8: MMA issue, 9: TMA
constexpr int kPfSoftmax = 256;
constexpr int kPfMmaWarp = 8, kPfTmaWarp = 9;
constexpr int kPfTile = 128;
constexpr int kPfTileBytes = kPfTile * kHeadDim * 2;  // 32 KB of bf16
constexpr int kPfKStages = 3, kPfVStages = 3;
constexpr int kPfSBufs = 3;  // TMEM score buffers; P_j overwrites the first 64 columns of S_j
constexpr uint32_t kPfQ = 0;
constexpr uint32_t kPfK = kPfQ + kPfTileBytes;
constexpr uint32_t kPfV = kPfK + kPfKStages * kPfTileBytes;
constexpr uint32_t kPfEnd = kPfV + kPfVStages * kPfTileBytes;
constexpr uint32_t kPfW = kPfV;  // W_H^T parts on the diagonal: the V ring, 96 KB
constexpr int kPfSmem = (int)kPfEnd + 1024;  // + alignment to 1024 bytes
constexpr uint32_t kPfTmemCols = 512;  // S0 [0,128) S1 [128,256) S2 [256,384) O [384,512); Y in S0
constexpr uint32_t kColO = 384, kColY = 0;
constexpr uint32_t kPfWaitTries = 1u << 22;
constexpr uint32_t kPfTestWaitTries = 1u << 10;
constexpr float kRescaleSlack = 8.f;  // log2 units: p <= 2^8 between rescales

static_assert(kPfW + 3 * 128 * kHeadDim * 2 <= kPfEnd, "W_H^T parts fit the V ring");

struct PfParams {
  int B, Hq, Hkv, G, max_seq, n_qt;
  const int32_t* seq_lens;
  const __nv_bfloat16* wparts;  // [Hkv][3][r x 128] core-matrix layout, or null
  void* codes;                  // [B][Hkv][max_seq][r/32] uint32 (uint16 for r = 16), or null
  __nv_bfloat16* out;           // [B][Hq][max_seq][128]
  float scale_log2;             // scale * log2(e), > 0
  uint32_t* status;
  int test_expire;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of the 16-byte chunk (row, k .. k + 7) in the core-matrix layout of a [rows][128] bf16 operand
__host__ __device__ __forceinline__ uint32_t cm_off128(int row, int k) {
  return (uint32_t)((((row >> 3) * (kHeadDim / 8) + (k >> 3)) << 7) + ((row & 7) << 4));
}

// W_H^T as three bf16 parts w1 + w2 + w3 (w1 = bf16(w), w2 = bf16(w - w1),
// w3 = bf16(w - w1 - w2)) in the core-matrix layout, one (column n, 8
// consecutive k) chunk per thread and step; grid.x = KV group
template <int R>
__global__ void __launch_bounds__(256) split_w_kernel(const float* __restrict__ W, __nv_bfloat16* __restrict__ parts) {
  const int g = blockIdx.x;
  const float* Wg = W + (size_t)g * kHeadDim * R;
  unsigned char* dst = reinterpret_cast<unsigned char*>(parts) + (size_t)g * 3 * R * kHeadDim * 2;
  constexpr int WPART = R * kHeadDim * 2;
  for (int it = threadIdx.x; it < R * (kHeadDim / 8); it += blockDim.x) {
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
    const uint32_t off = cm_off128(n, k0);
    *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(p1);
    *reinterpret_cast<uint4*>(dst + WPART + off) = *reinterpret_cast<const uint4*>(p2);
    *reinterpret_cast<uint4*>(dst + 2 * WPART + off) = *reinterpret_cast<const uint4*>(p3);
  }
}

// scores of keys after row m (column col0 + e > m) set to -inf: the causal mask of the diagonal tile
__device__ __forceinline__ void mask_after_row(uint32_t (&va)[32], uint32_t (&vb)[32], int col0, int m) {
  const uint32_t ninf = 0xff800000u;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    va[e] = col0 + e <= m ? va[e] : ninf;
    vb[e] = col0 + 32 + e <= m ? vb[e] : ninf;
  }
}

// sum of 64 values by a tree of additions (consumes va)
__device__ __forceinline__ float tree_sum64(uint32_t (&va)[32], const uint32_t (&vb)[32]) {
#pragma unroll
  for (int e = 0; e < 32; ++e) va[e] = __float_as_uint(__uint_as_float(va[e]) + __uint_as_float(vb[e]));
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
    for (int e = 0; e < w; ++e) va[e] = __float_as_uint(__uint_as_float(va[e]) + __uint_as_float(va[e + w]));
  return __uint_as_float(va[0]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
  const __nv_bfloat162 pb = __floats2bfloat162_rn(__uint_as_float(lo), __uint_as_float(hi));
  return *reinterpret_cast<const uint32_t*>(&pb);
}

template <int R>  // R = 0: attention only
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const PfParams p) {
  extern __shared__ __align__(1024) unsigned char pf_smem[];
  __shared__ __align__(8) uint64_t q_full, k_full[kPfKStages], k_free[kPfKStages], v_full[kPfVStages],
      v_free[kPfVStages], s_full[kPfSBufs], s_free[kPfSBufs], p_full, pv_done, w_full, y_done, drain, never,
      mx_bar[2];
  __shared__ uint32_t tmem_s;
  __shared__ volatile int abort_s;
  __shared__ int k_issued_s, v_issued_s, w_issued_s;
  __shared__ float l_part[2][kPfTile];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbh = p.B * p.Hq;
  const int item = (int)blockIdx.x;
  const int i = p.n_qt - 1 - item / nbh;  // query tile: the heaviest first
  const int b = (item % nbh) / p.Hq, h = (item % nbh) % p.Hq;
  int L = p.seq_lens[b];
  L = L > p.max_seq ? p.max_seq : (L < 0 ? 0 : L);
  if (i < 0 || kPfTile * i >= L) return;
  if (tid == 0 && i == 0 && h == 0 && p.seq_lens[b] > p.max_seq) set_status(p.status, HATA_ERR_INVALID_ARG);
  const int g = h / p.G;
  const int n = i + 1;  // key tiles 0 .. i
  const bool enc = R > 0 && p.codes != nullptr && (h % p.G) == 0;
  const uint32_t base = (tc::smem_u32(pf_smem) + 1023u) & ~1023u;
  const int q_row = (b * p.Hq + h) * p.max_seq + kPfTile * i;
  const int kv_row = (b * p.Hkv + g) * p.max_seq;

  if (warp == 0) tc::tmem_alloc(&tmem_s, kPfTmemCols);
  if (tid == kPfSoftmax) {
    tc::mbar_init(&q_full, 1);
    for (int s = 0; s < kPfKStages; ++s) {
      tc::mbar_init(&k_full[s], 1);
      tc::mbar_init(&k_free[s], 1);
    }
    for (int s = 0; s < kPfVStages; ++s) {
      tc::mbar_init(&v_full[s], 1);
      tc::mbar_init(&v_free[s], 1);
    }
    for (int s = 0; s < kPfSBufs; ++s) {
      tc::mbar_init(&s_full[s], 1);
      tc::mbar_init(&s_free[s], 1);
    }
    tc::mbar_init(&p_full, kPfSoftmax);
    tc::mbar_init(&pv_done, 1);
    tc::mbar_init(&w_full, 1);
    tc::mbar_init(&y_done, 1);
    tc::mbar_init(&drain, 1);
    tc::mbar_init(&never, 1);
    tc::mbar_init(&mx_bar[0], kPfSoftmax);
    tc::mbar_init(&mx_bar[1], kPfSoftmax);
    tc::mbar_init_fence();
    abort_s = 0;
    k_issued_s = 0;
    v_issued_s = 0;
    w_issued_s = 0;
  }
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = tmem_s;

  // bounded wait; on expiry record the timeout once and tell every role to stop
  // (polls the abort flag every 64 tries, so that the other roles stop soon after one gives up)
  auto wait_ok = [&](uint64_t* bar, uint32_t parity) -> bool {
    for (uint32_t it = 0; it < kPfWaitTries; it += 64) {
      if (abort_s) return false;
      if (tc::mbar_wait(bar, parity, 64)) return true;
    }
    set_status(p.status, HATA_ERR_TIMEOUT);
    abort_s = 1;
    return false;
  };

  if (warp == kPfTmaWarp) {
    if (lane == 0) {
      // ---------------- loader: Q once, then K_t / V_t into 3-deep rings ----------------
      auto load_k = [&](int t) {
        const uint32_t dst = base + kPfK + (uint32_t)(t % kPfKStages) * kPfTileBytes;
        tc::mbar_expect(&k_full[t % kPfKStages], (uint32_t)kPfTileBytes);
        tc::tma_load_2d(dst, &kmap, 0, kv_row + kPfTile * t, &k_full[t % kPfKStages]);
        tc::tma_load_2d(dst + kPfTileBytes / 2, &kmap, 64, kv_row + kPfTile * t, &k_full[t % kPfKStages]);
        k_issued_s = t + 1;
      };
      auto load_v = [&](int t) {
        const uint32_t dst = base + kPfV + (uint32_t)(t % kPfVStages) * kPfTileBytes;
        tc::mbar_expect(&v_full[t % kPfVStages], (uint32_t)kPfTileBytes);
        tc::tma_load_2d(dst, &vmap, 0, kv_row + kPfTile * t, &v_full[t % kPfVStages]);
        tc::tma_load_2d(dst + kPfTileBytes / 2, &vmap, 64, kv_row + kPfTile * t, &v_full[t % kPfVStages]);
        v_issued_s = t + 1;
      };
      tc::mbar_expect(&q_full, (uint32_t)kPfTileBytes);
      tc::tma_load_2d(base + kPfQ, &qmap, 0, q_row, &q_full);
      tc::tma_load_2d(base + kPfQ + kPfTileBytes / 2, &qmap, 64, q_row, &q_full);
      // K_t once S_{t-3} is done with its stage, V_t once PV_{t-3} is
      for (int t = 0; t < n; ++t) {
        if (t >= kPfKStages && !wait_ok(&k_free[t % kPfKStages], (uint32_t)(((t - kPfKStages) / kPfKStages) & 1)))
          break;
        load_k(t);
        if (t >= kPfVStages && !wait_ok(&v_free[t % kPfVStages], (uint32_t)(((t - kPfVStages) / kPfVStages) & 1)))
          break;
        load_v(t);
      }
      // drain: every copy still in flight lands before the CTA leaves
      const int kl = k_issued_s, vl = v_issued_s;
      for (int t = max(0, kl - kPfKStages); t < kl; ++t)
        tc::mbar_wait(&k_full[t % kPfKStages], (uint32_t)((t / kPfKStages) & 1), kPfWaitTries);
      for (int t = max(0, vl - kPfVStages); t < vl; ++t)
        tc::mbar_wait(&v_full[t % kPfVStages], (uint32_t)((t / kPfVStages) & 1), kPfWaitTries);
      tc::mbar_wait(&q_full, 0, kPfWaitTries);
    }
  } else if (warp == kPfMmaWarp) {
    if (lane == 0) {
      // ---------------- MMA issue: S_j, then PV_{j-1} ----------------
      bool ok = true;
      if (p.test_expire && !tc::mbar_wait(&never, 0, kPfTestWaitTries)) {  // test hook: this wait runs out
        set_status(p.status, HATA_ERR_TIMEOUT);
        abort_s = 1;
        ok = false;
      }
      ok = ok && wait_ok(&q_full, 0);
      constexpr uint32_t idS = tc::idesc_bf16(kPfTile, kPfTile, false);
      constexpr uint32_t idPV = tc::idesc_bf16(kPfTile, kHeadDim, true);
      auto issue_pv = [&](int t) {  // O (+)= P_t V_t, P_t read from TMEM (8 columns per 16 keys)
        tc::fence_after();
        const uint32_t vb = base + kPfV + (uint32_t)(t % kPfVStages) * kPfTileBytes;
        const uint32_t pa = tmem + (uint32_t)((t % kPfSBufs) * kPfTile);
#pragma unroll
        for (int ks = 0; ks < kPfTile / 16; ++ks)  // keys 64 w .. 64 w + 63 of P at columns 64 w ..
          tc::mma_ts(tmem + kColO, pa + (uint32_t)((ks >> 2) * 64 + (ks & 3) * 8),
                     tc::desc_mnmajor_sw128(vb + (uint32_t)ks * 2048u, (uint32_t)(kPfTileBytes / 2)), idPV,
                     (t > 0 || ks > 0) ? 1u : 0u);
        tc::commit(&pv_done);
        tc::commit(&v_free[t % kPfVStages]);
        tc::commit(&s_free[t % kPfSBufs]);
      };
      for (int j = 0; ok && j < n; ++j) {
        if (!(ok = wait_ok(&k_full[j % kPfKStages], (uint32_t)((j / kPfKStages) & 1)))) break;
        // score buffer j % 3 is free once PV_{j-3} (which read P_{j-3} from it) is done
        if (j >= kPfSBufs &&
            !(ok = wait_ok(&s_free[j % kPfSBufs], (uint32_t)(((j - kPfSBufs) / kPfSBufs) & 1))))
          break;
        tc::fence_after();
        // S_j = Q K_j^T
        const uint32_t kb = base + kPfK + (uint32_t)(j % kPfKStages) * kPfTileBytes;
#pragma unroll
        for (int ks = 0; ks < kHeadDim / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * (kPfTileBytes / 2) + (ks & 3) * 32);
          tc::mma(tmem + (uint32_t)((j % kPfSBufs) * kPfTile), tc::desc_kmajor_sw128(base + kPfQ + off),
                  tc::desc_kmajor_sw128(kb + off), idS, ks > 0 ? 1u : 0u);
        }
        tc::commit(&s_full[j % kPfSBufs]);
        tc::commit(&k_free[j % kPfKStages]);
        if (j >= 1) {
          if (!(ok = wait_ok(&p_full, (uint32_t)((j - 1) & 1)))) break;
          if (!(ok = wait_ok(&v_full[(j - 1) % kPfVStages], (uint32_t)(((j - 1) / kPfVStages) & 1)))) break;
          issue_pv(j - 1);
        }
      }
      if (ok) ok = wait_ok(&p_full, (uint32_t)((n - 1) & 1));
      if (ok) ok = wait_ok(&v_full[(n - 1) % kPfVStages], (uint32_t)(((n - 1) / kPfVStages) & 1));
      if (ok) issue_pv(n - 1);
      if constexpr (R > 0) {
        if (ok && enc) {
          // Y = K_i W_H: the W_H^T parts into the V ring once the last PV has read it
          ok = wait_ok(&pv_done, (uint32_t)((n - 1) & 1));
          if (ok) {
            constexpr uint32_t wbytes = 3u * R * kHeadDim * 2u;
            tc::mbar_expect(&w_full, wbytes);
            tc::bulk_load(base + kPfW, p.wparts + (size_t)g * 3 * R * kHeadDim, wbytes, &w_full);
            w_issued_s = 1;
            ok = wait_ok(&w_full, 0);
          }
          if (ok) {
            tc::fence_after();
            constexpr uint32_t idY = tc::idesc_bf16(kPfTile, R, false);
            const uint32_t kb = base + kPfK + (uint32_t)((n - 1) % kPfKStages) * kPfTileBytes;
#pragma unroll
            for (int part = 0; part < 3; ++part)
#pragma unroll
              for (int ks = 0; ks < kHeadDim / 16; ++ks)
                tc::mma(tmem + kColY,
                        tc::desc_kmajor_sw128(kb + (uint32_t)((ks >> 2) * (kPfTileBytes / 2) + (ks & 3) * 32)),
                        tc::desc_kmajor_cm(base + kPfW + (uint32_t)(part * R * kHeadDim * 2 + ks * 256)), idY,
                        (part | ks) ? 1u : 0u);
            tc::commit(&y_done);
          }
        }
      }
      // drain: every MMA issued above completes before the CTA leaves
      tc::commit(&drain);
      tc::mbar_wait(&drain, 0, kPfWaitTries);
      if (w_issued_s) tc::mbar_wait(&w_full, 0, kPfWaitTries);
    }
  } else {
    // ---------------- softmax warpgroups: query row m = tid % 128 ----------------
    // Both warpgroups find the full row maximum (identical arithmetic, so identical m);
    // warpgroup w then owns keys 64 w .. 64 w + 63 of each tile (exponentials, P, its
    // part of the row sum) and columns 64 w .. 64 w + 63 of O (rescale, output).
    const int wg = warp >> 2;
    const int m = tid & 127;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const float c = p.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // warp-uniform outcome, so that the warp-collective TMEM loads below run with every lane or none
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = wait_ok(bar, parity);
      return __all_sync(0xffffffffu, r);
    };
    for (int j = 0; j < n; ++j) {
      if (!(ok = wait_warp(&s_full[j % kPfSBufs], (uint32_t)((j / kPfSBufs) & 1)))) break;
      tc::fence_after();
      const uint32_t sa = lane_base + (uint32_t)((j % kPfSBufs) * kPfTile);
      const bool diag = j == i;
      // pass 1 (this warpgroup's 64 keys, kept in registers for pass 2): the maximum over its
      // visible keys (scale > 0, so of the raw scores; the diagonal tile's keys after the row
      // set to -inf first), then the other warpgroup's half.  The halves meet in TMEM: column
      // 64 w + 32 of this score buffer (read already; P only takes the first 32 of each half)
      // on the row's lane, ordered by mx_bar; two barrier slots suffice, since a warpgroup
      // reaches tile j + 2 only after both have finished tile j.
      const int cc = 2 * wg;
      uint32_t va[32], vb[32];
      tc::ld32_nowait(sa + 32 * cc, va);
      tc::ld32_nowait(sa + 32 * cc + 32, vb);
      tc::ld_wait();
      if (diag) mask_after_row(va, vb, 32 * cc, m);
      float m8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m8[e] = fmaxf(__uint_as_float(va[e]), __uint_as_float(vb[e]));
#pragma unroll
      for (int e = 8; e < 32; ++e) m8[e & 7] = fmaxf(m8[e & 7], fmaxf(__uint_as_float(va[e]), __uint_as_float(vb[e])));
      const float mown = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      tc::st1(sa + 64 * wg + 32, __float_as_uint(mown));
      tc::st_wait();
      tc::fence_before();
      tc::mbar_arrive(&mx_bar[j & 1]);
      if (!(ok = wait_warp(&mx_bar[j & 1], (uint32_t)((j >> 1) & 1)))) break;
      tc::fence_after();
      const float mx = fmaxf(mown, __uint_as_float(tc::ld1(sa + 64 * (wg ^ 1) + 32)));
      const float m_tile = mx * c;
      if (j == 0) {
        m_used = m_tile;
      } else if (__any_sync(0xffffffffu, m_tile > m_used + kRescaleSlack)) {
        // O is rescaled once the previous PV has landed (PV_j is issued only after this tile's P)
        if (!(ok = wait_warp(&pv_done, (uint32_t)((j - 1) & 1)))) break;
        tc::fence_after();
        const float m_new = fmaxf(m_used, m_tile);
        const float alpha = ex2(m_used - m_new);
#pragma unroll 1
        for (int cc = 2 * wg; cc < 2 * wg + 2; ++cc) {
          uint32_t o[32];
          tc::ld32(lane_base + kColO + 32 * cc, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tc::st32(lane_base + kColO + 32 * cc, o);
        }
        tc::st_wait();
        l *= alpha;
        m_used = m_new;
      }
      // pass 2 (this warpgroup's 64 keys, from pass 1's registers): p = 2^(s c - m_used) (0 for
      // masked keys), packed as bf16 pairs over the first half of the scores it read (columns
      // 64 w .. 64 w + 31 of this buffer), and its part of the row sum
      float sum = 0.f;
      {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          va[e] = __float_as_uint(ex2(fmaf(__uint_as_float(va[e]), c, -m_used)));
          vb[e] = __float_as_uint(ex2(fmaf(__uint_as_float(vb[e]), c, -m_used)));
        }
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pk[e] = pack_bf16x2(va[2 * e], va[2 * e + 1]);
          pk[16 + e] = pack_bf16x2(vb[2 * e], vb[2 * e + 1]);
        }
        tc::st32(sa + 32 * cc, pk);
        sum += tree_sum64(va, vb);
      }
      l += sum;
      tc::st_wait();
      // the last tile of the sequence: value rows at or beyond L_b (never visible, possibly not finite)
      // are zeroed so that 0 * V stays 0 in PV
      if (j == n - 1 && kPfTile * n > L) {
        if (!(ok = wait_warp(&v_full[j % kPfVStages], (uint32_t)((j / kPfVStages) & 1)))) break;
        if (kPfTile * j + m >= L) {  // warpgroup w: the row's half in box w (elements 64 w ..)
          unsigned char* vrow = pf_smem + (base - tc::smem_u32(pf_smem)) + kPfV + (j % kPfVStages) * kPfTileBytes +
                                wg * (kPfTileBytes / 2) + (m >> 3) * 1024 + (m & 7) * 128;
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) *reinterpret_cast<uint4*>(vrow + qq * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      tc::fence_async_smem();
      tc::fence_before();
      tc::mbar_arrive(&p_full);
    }
    // the row sum of both halves (every softmax thread reaches this barrier, also after an abort)
    l_part[wg][m] = l;
    asm volatile("bar.sync 1, %0;\n" ::"n"(kPfSoftmax) : "memory");
    l = l_part[0][m] + l_part[1][m];
    // output rows: O / l once the last PV is done (warpgroup w: columns 64 w .. 64 w + 63)
    if (ok) ok = wait_warp(&pv_done, (uint32_t)((n - 1) & 1));
    if (ok) {
      tc::fence_after();
      const int t = kPfTile * i + m;
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.out + ((size_t)(b * p.Hq + h) * p.max_seq + t) * kHeadDim;
#pragma unroll
      for (int cc = 2 * wg; cc < 2 * wg + 2; ++cc) {
        uint32_t o[32];
        tc::ld32(lane_base + kColO + 32 * cc, o);
        if (t < L) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 ob = __floats2bfloat162_rn(__uint_as_float(o[8 * qq + 2 * e]) * inv,
                                                              __uint_as_float(o[8 * qq + 2 * e + 1]) * inv);
              w4[e] = *reinterpret_cast<const uint32_t*>(&ob);
            }
            *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * qq) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
    }
    if constexpr (R > 0) {
      if (ok && enc && wg == 0) {
        ok = wait_warp(&y_done, 0);
        if (ok) {
          tc::fence_after();
          const int key = kPfTile * i + m;
          constexpr int NWd = R < 32 ? 1 : R / 32;
          uint32_t word[NWd];
#pragma unroll
          for (int cw = 0; cw < NWd; ++cw) {
            uint32_t y[32];
            tc::ld32(lane_base + kColY + 32 * cw, y);
            uint32_t bits = 0u;
#pragma unroll
            for (int e = 0; e < (R < 32 ? R : 32); ++e) bits |= (__uint_as_float(y[e]) > 0.f ? 1u : 0u) << e;
            word[cw] = bits;
          }
          if (key < L) {
            const size_t slot = (size_t)(b * p.Hkv + g) * p.max_seq + key;
            if constexpr (R == 16) {
              reinterpret_cast<uint16_t*>(p.codes)[slot] = (uint16_t)word[0];
            } else if constexpr (NWd == 4) {
              reinterpret_cast<uint4*>(p.codes)[slot] = make_uint4(word[0], word[1], word[2], word[3]);
            } else if constexpr (NWd == 2) {
              reinterpret_cast<uint2*>(p.codes)[slot] = make_uint2(word[0], word[1]);
            } else {
              reinterpret_cast<uint32_t*>(p.codes)[slot] = word[0];
            }
          }
        }
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::tmem_dealloc(tmem, kPfTmemCols);
  }
}

template <int R>
cudaError_t configure_prefill() {
  static std::mutex mu;
  static std::map<int, cudaError_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  auto it = done.find(dev);
  if (it != done.end()) return it->second;
  e = cudaFuncSetAttribute(prefill_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmem);
  if (e != cudaSuccess) (void)cudaGetLastError();
  done[dev] = e;
  return e;
}

template <int R>
cudaError_t launch_r(const hata_dims_t& d, const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                     PfParams& prm, const float* W, unsigned grid, cudaStream_t st) {
  cudaError_t e = configure_prefill<R>();
  if (e != cudaSuccess) return e;
  if constexpr (R > 0) {
    if (prm.codes) {
      split_w_kernel<R><<<d.n_kv_heads, 256, 0, st>>>(W, const_cast<__nv_bfloat16*>(prm.wparts));
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  prefill_kernel<R><<<grid, kPfThreads, kPfSmem, st>>>(qm, km, vm, prm);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_ws_bytes(const hata_dims_t& d) {
  const size_t parts = (size_t)d.n_kv_heads * 3 * (size_t)std::max(d.hash_bits, 0) * kHeadDim * 2;
  return kStatusBytes + (parts + 15) / 16 * 16;
}

cudaError_t launch_prefill(const hata_dims_t& d, const void* q, const void* K, const void* V, const float* W,
                           void* codes, const int32_t* seq_lens, float scale, void* out, char* ws,
                           cudaStream_t st) {
  const long long n_qt = (d.max_seq + kPfTile - 1) / kPfTile;
  const long long grid = n_qt * d.batch * d.n_q_heads;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  CUtensorMap qm, km, vm;
  if (!make_bf16_rows_map(&qm, q, (long long)d.batch * d.n_q_heads * d.max_seq, kPfTile) ||
      !make_bf16_rows_map(&km, K, (long long)d.batch * d.n_kv_heads * d.max_seq, kPfTile) ||
      !make_bf16_rows_map(&vm, V, (long long)d.batch * d.n_kv_heads * d.max_seq, kPfTile))
    return cudaErrorNotSupported;
  PfParams prm;
  prm.B = d.batch;
  prm.Hq = d.n_q_heads;
  prm.Hkv = d.n_kv_heads;
  prm.G = d.n_q_heads / d.n_kv_heads;
  prm.max_seq = d.max_seq;
  prm.n_qt = (int)n_qt;
  prm.seq_lens = seq_lens;
  prm.wparts = reinterpret_cast<const __nv_bfloat16*>(ws + kStatusBytes);
  prm.codes = codes;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.status = reinterpret_cast<uint32_t*>(ws);
  prm.test_expire = (d.flags & HATA_FLAG_TEST_EXPIRE_WAIT) ? 1 : 0;
  const unsigned g = (unsigned)grid;
  if (!codes) return launch_r<0>(d, qm, km, vm, prm, W, g, st);
  switch (d.hash_bits) {
    case 16: return launch_r<16>(d, qm, km, vm, prm, W, g, st);
    case 32: return launch_r<32>(d, qm, km, vm, prm, W, g, st);
    case 64: return launch_r<64>(d, qm, km, vm, prm, W, g, st);
    case 128: return launch_r<128>(d, qm, km, vm, prm, W, g, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace hata
