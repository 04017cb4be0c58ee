/*
 * hata.h -- C ABI of libhata, the B200 (sm_100a) decode-step hot path of HATA,
 * Hash-Aware Top-k Attention.
 *
 * Method source: "HATA: Trainable and Hardware-Efficient Hash-Aware Top-k
 * Attention for Scalable Large Model Inference" (paper notes, ACL 2025).
 *   - section 方法详解 > 关键设计: the hash h(x) = 2*Sigmoid(sigma * x W_H) - 1 with
 *     one trainable W_H per attention head; its sign is the code.
 *   - section 方法详解 > Decode 阶段算法: per decode step, HashEncode the new query
 *     and key (matrix multiply + Sign + BitPack), append the key code to the
 *     hash-code cache, Hamming distance bitcount(xor(Q_H, K_H_cache)) against all
 *     cached codes, aggregate the scores of the query heads that share a KV
 *     cache (GQA), select top-k, gather those K/V rows and run exact attention.
 *   - section 硬件高效优化: projection + sign + bitpack + cache update fused in one
 *     kernel; XOR + popc Hamming operator with coalesced access; gather fused
 *     into the flash-attention kernel.
 *
 * Readings this library fixes where the pages are silent:
 *   - bit j of a code is [y_j > 0] with y = x . W_H computed in fp32; bit j sits
 *     in 32-bit word j / 32 at position j % 32 (least significant first);
 *   - W_H is one [d][r] fp32 matrix per KV head, shared by the G = Hq / Hkv
 *     query heads of that group and by its keys; query head h is in group h / G;
 *   - the GQA aggregate is the sum of the G per-head distances, so a score lies
 *     in [0, G * r]; lower is more similar;
 *   - top-k keeps the min(k, L_b) tokens with the smallest score; ties go to the
 *     lower token index; indices are reported in ascending order;
 *   - attention is softmax(scale * q . K_t) V_t over the selected rows only, fp32
 *     accumulation, one rounding to the output type; scale <= 0 means 1/sqrt(d);
 *   - an empty selection (L_b <= 0) gives an all-zero output row.
 *
 * Conventions for every call:
 *   - All tensor arguments are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory.  Scratch space and the device status word are
 *     a caller-provided workspace (hata_workspace_size); the one exception is
 *     hata_topk_noalloc, whose scratch is a fixed array inside the library.
 *   - Every call only enqueues work on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and never synchronises, except
 *     hata_read_device_status.
 *   - Host-visible argument errors are reported before anything is launched
 *     (HATA_ERR_INVALID_ARG / HATA_ERR_UNSUPPORTED); a failed launch reports
 *     HATA_ERR_CUDA.  Errors that only the device can see (a sequence length
 *     beyond max_seq, an index outside the cache, a bounded wait that ran out)
 *     are recorded in the workspace's status word, read with
 *     hata_read_device_status.  No kernel traps or asserts.
 *   - Layouts are C-contiguous:
 *       q, out      [B][Hq][d]            (dtype)
 *       K, V        [B][Hkv][max_seq][d]  (dtype), one contiguous row per token
 *       W_H         [Hkv][d][r]           fp32, used as x . W_H
 *       codes       [B][Hkv][max_seq][r/32] uint32 (the hash-code cache);
 *                   for r = 16, [B][Hkv][max_seq] uint16, one code per token
 *       qcode       [B][Hq][r/32]         uint32 ([B][Hq] uint16 for r = 16)
 *       seq_lens    [B]                   int32, cached length incl. the new token
 *       scores      [B][Hkv][max_seq]     int32
 *       idx         [B][Hkv][k]           int32, ascending, -1 padded
 *       n_sel       [B]                   int32, min(k, L_b)
 *   - Pointers must be 16-byte aligned.
 */
#ifndef HATA_H_
#define HATA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HATA_API __attribute__((visibility("default")))
#else
#define HATA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HATA_OK = 0,
  HATA_ERR_INVALID_ARG = 1, /* bad pointer, size or shape */
  HATA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim != 128) */
  HATA_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
  HATA_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up */
  HATA_ERR_WORKSPACE = 5    /* workspace missing or smaller than hata_workspace_size */
} hata_status_t;

typedef enum { HATA_F32 = 0, HATA_BF16 = 1 } hata_dtype_t;

/* Problem shape, shared by every call. */
typedef struct {
  int batch;      /* B >= 1 */
  int n_q_heads;  /* Hq >= 1, a multiple of n_kv_heads */
  int n_kv_heads; /* Hkv >= 1 */
  int head_dim;   /* d; this version supports 128 */
  int hash_bits;  /* r in {16, 32, 64, 128, 256}; 16 needs an even max_seq */
  int max_seq;    /* token capacity of each (b, kv head) cache slab, >= 1 */
  int dtype;      /* hata_dtype_t of q, K, V and out */
  int flags;      /* HATA_FLAG_* bits, 0 for none */
} hata_dims_t;

/* hata_decode_step is launched with programmatic dependent launch: it waits for
 * the kernel before it on the stream to finish before reading anything.  With
 * HATA_FLAG_EARLY_PREFETCH it instead starts reading seq_lens, W_H and the
 * cached codes of slots [0, L_b - 1) while that kernel is still running, and
 * waits only before it reads q, the new K/V row or writes anything.  Set the
 * flag only when the preceding kernel writes none of seq_lens, W_H and those
 * code slots -- e.g. when it is the projection that produces q and the new
 * K/V row.  It must not be set when the preceding kernel is a decode step or an
 * encode of the same cache. */
#define HATA_FLAG_EARLY_PREFETCH 1

/* Test hook for the timeout path of hata_decode_step (and its _qk and _paged
 * forms): the call's first bounded device-side wait is made on a barrier that
 * nothing completes, with a short limit, so it runs out; the call then records
 * HATA_ERR_TIMEOUT in the workspace's status word, skips its remaining work
 * without touching memory outside its arguments, and its outputs are
 * undefined.  Never set it outside tests; after it, re-initialise the
 * workspace (hata_workspace_init). */
#define HATA_FLAG_TEST_EXPIRE_WAIT 2

/* The decode step has two fused forms with identical results.  The cluster form
 * (one launch; a thread-block cluster of up to 16 SMs per (batch, KV head) unit,
 * every exchange on chip) is used while the units are few.  The all-SM form (an
 * encode kernel, a scan kernel that spreads every unit's cache over all SMs, and
 * a tail kernel with one cluster per unit, chained by programmatic dependent
 * launch) is used for 64 or more units, for 32 or more units that select at least
 * 32768 rows in all (units x min(k, max_seq)), and for paged caches.  This flag
 * selects the all-SM form for any shape it covers. */
#define HATA_FLAG_ALL_SM_SCAN 4

/* Bytes of workspace that every call below needs for these dims and budget k
 * (one size serves all calls).  Returns HATA_OK and writes *bytes. */
HATA_API hata_status_t hata_workspace_size(const hata_dims_t* dims, int k, size_t* bytes);

/* Zero a workspace before its first use (enqueued memset).  Every call leaves
 * the workspace's counters back at zero, so this is needed once, and again
 * only after a call reported HATA_ERR_TIMEOUT. */
HATA_API hata_status_t hata_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * KV cache update of a decode step (Decode 阶段算法: the new token's key and
 * value enter the cache before it is scored): for every batch b with
 * 1 <= L_b = seq_lens[b] <= max_seq and every KV head g,
 *     K[b][g][L_b - 1][:] = new_k[b][g][:]     V[b][g][L_b - 1][:] = new_v[b][g][:]
 * Batches with L_b outside [1, max_seq] are left unchanged.  hata_decode_step
 * then encodes K[b][g][L_b - 1] and appends its code.
 *   new_k, new_v  device [B][Hkv][d], dims->dtype, 16-byte aligned
 *   K, V          device [B][Hkv][max_seq][d], dims->dtype, 16-byte aligned
 *   seq_lens      device [B] int32
 * No workspace.  Enqueued on `stream`; the caller owns every buffer.
 */
HATA_API hata_status_t hata_append_kv(const hata_dims_t* dims, const void* new_k, const void* new_v, void* K, void* V,
                             const int32_t* seq_lens, void* stream);

/*
 * The same cache update for the paged pools of hata_decode_step_paged: the new
 * rows go to slot (L_b - 1) mod bs of pool block block_table[b][(L_b - 1) / bs]
 * of K_pool / V_pool ([n_blocks][Hkv][bs][d], dims->dtype, 16-byte aligned).
 * block_table is device [B][ceil(max_seq / bs)] int32; block_size bs is a power
 * of two in [16, 65536].  Batches with L_b outside [1, max_seq], or whose block
 * number lies outside [0, n_blocks), are left unchanged.  No workspace.
 */
HATA_API hata_status_t hata_append_kv_paged(const hata_dims_t* dims, const void* new_k, const void* new_v, void* K_pool,
                                   void* V_pool, const int32_t* block_table, int block_size, int n_blocks,
                                   const int32_t* seq_lens, void* stream);

/*
 * HashEncode + cache update (Decode 阶段算法, first two steps; 硬件高效优化,
 * fused projection -> sign -> bitpack -> cache update).  For every batch b,
 * head h < x_heads and token t in [end_b - n_tok, end_b) that also lies in
 * [0, min(x_len, codes_len)):
 *     codes[b][h][t][:] = pack(x[b][h][t][:] . W_H[h / (x_heads / Hkv)] > 0)
 * with end_b = seq_end[b] if seq_end is not NULL, else x_len.
 *   x         device [B][x_heads][x_len][d], dims->dtype
 *   x_heads   Hq to encode queries, Hkv to encode keys (a multiple of Hkv)
 *   seq_end   device [B] int32 or NULL
 *   codes     device [B][x_heads][codes_len][r/32] uint32
 * Typical uses: query codes (x = q, x_heads = Hq, x_len = codes_len = 1,
 * n_tok = 1, seq_end = NULL); appending the new key (x = K, x_heads = Hkv,
 * x_len = codes_len = max_seq, n_tok = 1, seq_end = seq_lens); prefill
 * (same with n_tok = max_seq).  For n_tok <= 4 the projection is fp32 FMA in
 * the same fixed order as hata_decode_step, so both give the same codes bit for
 * bit.  The prefill form of bf16 keys with r <= 128 runs on the tensor cores
 * with W_H split into three bf16 parts (exact products, fp32 accumulation in
 * another order); other prefill forms are fp32 FMA.  Codes of the different
 * forms can differ only where |x . W_H| is within fp32 rounding of zero.
 *   workspace  device, 16-byte aligned, at least 16 bytes (any workspace from
 *              hata_workspace_size qualifies, and can be shared with the other
 *              calls on the same stream): only its status word is used.  If a
 *              bounded wait of the tensor-core kernel runs out, HATA_ERR_TIMEOUT
 *              is recorded there (the codes are then incomplete); read it with
 *              hata_read_device_status.  Missing or too small:
 *              HATA_ERR_WORKSPACE.
 */
HATA_API hata_status_t hata_encode_append(const hata_dims_t* dims, const void* x, int x_heads, int x_len, int n_tok,
                                 const int32_t* seq_end, const float* W_H, uint32_t* codes, int codes_len,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * Hamming scan with the GQA sum (Decode 阶段算法, Hamming and GQA steps;
 * 硬件高效优化, XOR + popc operator):
 *     scores[b][g][t] = sum over h in group g of popcount(qcode[b][h] ^ codes[b][g][t])
 * for t < L_b = min(seq_lens[b], max_seq); entries t >= L_b are not written.
 */
HATA_API hata_status_t hata_hamming_scores(const hata_dims_t* dims, const uint32_t* qcode, const uint32_t* codes,
                                  const int32_t* seq_lens, int32_t* scores, void* stream);

/*
 * Top-k select (Decode 阶段算法, top-k step): for each (b, g), the min(k, L_b)
 * tokens t < L_b with the smallest scores[b][g][t], ties to the lower t, written
 * in ascending t to idx[b][g][0 .. n-1]; idx[b][g][n .. k-1] = -1.  n_sel[b]
 * (nullable) receives n.  Scores must lie in [0, G * r] (values outside are
 * clamped and flagged in the workspace status word).
 */
HATA_API hata_status_t hata_topk(const hata_dims_t* dims, const int32_t* scores, const int32_t* seq_lens, int k,
                        int32_t* idx, int32_t* n_sel, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Gather-fused sparse flash-decode (Decode 阶段算法, gather + sparse attention;
 * 硬件高效优化, gather fused into flash attention): for each b and query head h
 * in group g,
 *     out[b][h] = sum_j softmax_j(scale * q[b][h] . K[b][g][t_j]) V[b][g][t_j]
 * over the entries t_j = idx[b][g][j], j < k, with t_j >= 0 (negative entries
 * are padding).  Entries >= max_seq are skipped and flagged in the workspace
 * status word.  scale <= 0 selects 1/sqrt(d).
 */
HATA_API hata_status_t hata_sparse_decode(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                 const int32_t* idx, int k, float scale, void* out, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * The whole decode step in one call (Decode 阶段算法 end to end, with the
 * fusions of 硬件高效优化): encode the queries; encode the new key K[b][g][L_b-1]
 * and write its code to codes[b][g][L_b-1]; Hamming scan with the GQA sum over
 * t < L_b; top-k; gather + attention into out.  The new token is a candidate
 * like any other.  Results equal the chain hata_encode_append ->
 * hata_hamming_scores -> hata_topk -> hata_sparse_decode bit for bit in codes
 * and indices.  qcode_out ([B][Hq][r/32]) and idx_out ([B][Hkv][k]) are
 * optional copies of the intermediates (NULL to skip).
 */
HATA_API hata_status_t hata_decode_step(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                               const float* W_H, uint32_t* codes, const int32_t* seq_lens, int k, float scale,
                               void* out, uint32_t* qcode_out, int32_t* idx_out, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * The decode step with separate query and key encoders, the form of
 * "HashAttention: Semantic Sparsity for Faster Inference" (its summary's
 * Approach: independent key and query mappings into Hamming space, pivotal
 * tokens found by XOR + popcount): queries are encoded with W_q, the new key
 * with W_k ([Hkv][d][r] fp32 each, 16-byte aligned), and the cache must hold
 * codes made with W_k (hata_encode_append with W_H = W_k).  Everything else,
 * including layouts, outputs and errors, is as in hata_decode_step, which is
 * this call with W_q = W_k.
 */
HATA_API hata_status_t hata_decode_step_qk(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                  const float* W_q, const float* W_k, uint32_t* codes, const int32_t* seq_lens,
                                  int k, float scale, void* out, uint32_t* qcode_out, int32_t* idx_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The decode step over a paged cache (the block layout of vLLM PagedAttention,
 * which the HashAttention summary lists among its foundations; a growing cache
 * appends one token per step).  K_pool and V_pool are [n_blocks][Hkv][bs][d]
 * (dims->dtype), codes_pool is [n_blocks][Hkv][bs][r/32] uint32, block_size bs is
 * a power of two in [16, 65536].  Sequence b's logical token t lives in slot
 * t mod bs of pool block block_table[b][t / bs]; block_table is device
 * [B][ceil(max_seq / bs)] int32, with dims->max_seq the logical capacity of a
 * sequence.  The new token's K/V row must already be in its slot, and its code is
 * written there.  Queries are encoded with W_q and keys with W_k (pass the same
 * matrix twice for HATA's single encoder).  Indices in idx_out are logical token
 * indices; everything else is as in hata_decode_step.  A block number outside
 * [0, n_blocks) is replaced by block 0 and flagged in the status word.  Returns
 * HATA_ERR_UNSUPPORTED for shapes the fused kernel does not cover (G not in
 * {1, 2, 4, 8}).  The prefill encode of a paged cache is hata_encode_append over
 * the pool seen as a batch of blocks: dims with batch = n_blocks, max_seq = bs,
 * x = K_pool, x_heads = Hkv, x_len = n_tok = codes_len = bs, seq_end = NULL.
 */
HATA_API hata_status_t hata_decode_step_paged(const hata_dims_t* dims, const void* q, const void* K_pool,
                                     const void* V_pool, const float* W_q, const float* W_k, uint32_t* codes_pool,
                                     const int32_t* block_table, int block_size, int n_blocks,
                                     const int32_t* seq_lens, int k, float scale, void* out, uint32_t* qcode_out,
                                     int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dense flash-decode, the comparison baseline: exact attention of every query
 * head over all cached tokens (the dense attention that the "HATA" paper notes'
 * 实验 section times HATA against, at 32K-128K context):
 *     out[b][h] = sum_{t < L_b} softmax_t(scale * q[b][h] . K[b][g][t]) V[b][g][t]
 * with g = h / G and L_b = min(seq_lens[b], max_seq) (seq_lens NULL: max_seq).
 * Same layouts as hata_decode_step; bf16 only, G <= 8, d = 128 (else
 * HATA_ERR_UNSUPPORTED).  Logits and P.V run on tensor-core tiles (bf16 in,
 * fp32 accumulate, probabilities rounded to bf16 for P.V), so results agree
 * with exact attention within the bf16 tolerance.  The workspace
 * (hata_dense_workspace_size bytes, 16-byte aligned) holds per-split partials
 * and arrival counters; zero it once with hata_workspace_init before the first
 * call; every call leaves the counters at zero.  L_b > max_seq is clamped and
 * flagged in the workspace's status word (hata_read_device_status).
 */
HATA_API hata_status_t hata_dense_workspace_size(const hata_dims_t* dims, size_t* bytes);
HATA_API hata_status_t hata_dense_decode(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                         const int32_t* seq_lens, float scale, void* out, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * Causal prefill attention with the key HashEncode fused in (整体框架, prefill
 * phase: the prompt runs full attention while every key is hashed and its code
 * cached for decode; 实验: the encode costs under 1%).  For every batch b, query
 * head h (KV group g = h / G) and position t < L_b = seq_lens[b]:
 *     out[b][h][t][:] = sum_{s <= t} softmax_s(scale * q[b][h][t] . K[b][g][s]) V[b][g][s][:]
 * and, when codes is not NULL, for every s < L_b:
 *     codes[b][g][s] = pack(K[b][g][s][:] . W_H[g] > 0)      (as hata_encode_append)
 *   q, out      device [B][Hq][max_seq][d] bf16; rows t >= L_b of out are not written
 *   K, V        device [B][Hkv][max_seq][d] bf16
 *   W_H         device [Hkv][d][r] fp32 (ignored when codes is NULL)
 *   codes       device [B][Hkv][max_seq][r/32] uint32 ([..][max_seq] uint16 for
 *               r = 16), or NULL for plain prefill attention; r <= 128
 *   scale       softmax scale, > 0; 0 selects 1/sqrt(d)
 * bf16 only (HATA_ERR_UNSUPPORTED otherwise).  Logits and P.V run on tcgen05
 * tensor-core tiles (bf16 in, fp32 accumulate, probabilities rounded to bf16),
 * so outputs agree with exact attention within the bf16 tolerance; code bits
 * can differ from the exact sign only where |x . W_H| is within fp32 rounding
 * of zero.  The workspace (hata_prefill_workspace_size bytes, 16-byte aligned)
 * holds the status word and W_H split into bf16 parts; no initialisation is
 * needed.  L_b > max_seq is clamped and flagged in the status word; a bounded
 * wait that runs out records HATA_ERR_TIMEOUT there (hata_read_device_status).
 */
HATA_API hata_status_t hata_prefill_workspace_size(const hata_dims_t* dims, size_t* bytes);
HATA_API hata_status_t hata_prefill_attention(const hata_dims_t* dims, const void* q, const void* K, const void* V,
                                     const float* W_H, void* codes, const int32_t* seq_lens, float scale, void* out,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * hata_topk without a workspace, for callers that cannot allocate device memory
 * (no counterpart on the pages: it only changes where scratch lives).  Same
 * inputs, outputs and results as hata_topk.  Its scratch is one 8 MiB array of
 * device memory owned by the library, present on every GPU that loads it until
 * the process exits.  Problems whose scratch would exceed it return
 * HATA_ERR_WORKSPACE before any launch.  The first call on a device looks up
 * the array's address (that device current): make it before any stream
 * capture.  All calls on a device share the array, so calls whose work
 * overlaps on the GPU race; each call clears the counters it needs.  Device-side
 * argument errors of this call are not reported.  Allocates nothing.
 */
HATA_API hata_status_t hata_topk_noalloc(const hata_dims_t* dims, const int32_t* scores, const int32_t* seq_lens,
                                         int k, int32_t* idx, int32_t* n_sel, void* stream);

/* Number of kernels one hata_decode_step call with these dims and k enqueues:
 * 1 for the cluster form, 3 for the all-SM form (see HATA_FLAG_ALL_SM_SCAN), 6
 * for the granular chain (r = 16, or shapes neither fused form covers), or -1
 * for invalid dims. */
HATA_API int hata_decode_step_kernel_count(const hata_dims_t* dims, int k);

/* Wait for `stream`, then return the workspace's device status word (a
 * hata_status_t recorded by a kernel, HATA_OK if none) in *device_status and
 * clear it.  The only call that synchronises. */
HATA_API hata_status_t hata_read_device_status(void* workspace, void* stream, int* device_status);

/* Static description of a status code. */
HATA_API const char* hata_status_string(hata_status_t status);

/* Library version as 10000 * major + 100 * minor + patch. */
HATA_API int hata_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HATA_H_ */
