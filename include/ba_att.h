/*
 * ba_att.h — C ABI of the BA-Att hot path on NVIDIA B200 (sm_100a).
 *
 * Block Approximate Sparse Attention (BA-Att) has two stages:
 *   1. a block-wise pre-downsample selector: per-block means and diagonal
 *      variances of Q and K, a covariance-compensated block-score map, and
 *      norm sorting that keeps the top fraction of key blocks per query block;
 *   2. block-sparse bidirectional attention over the kept blocks, emitting the
 *      output O and the per-row log-sum-exp (LSE).
 * A companion call merges two partial attentions (O, LSE) in log space.
 *
 * Sources: "Efficient Long-Context Modeling in Diffusion Language Models via
 * Block Approximate Sparse Attention" (abstract, "Core claim", "What carries
 * the argument", Figure 4) and "FlashBlock: Attention Caching for Efficient
 * Long-Context Block Diffusion" (Eq. 5, Eq. 9). The pages give the method in
 * prose only; the formulas stated below are the plain reading of that prose.
 *
 * Conventions shared by every call
 *  - Tensors are dense, row-major, head-major: Q is [B, Hq, N_alloc, d];
 *    K and V are [B, Hkv, N_alloc, d]. Only rows n < N of each head are
 *    tokens; rows N..N_alloc-1 are padding that is never read as a token and
 *    never written.
 *  - Blocks: block size b for queries and keys alike; nq = nk = ceil(N / b);
 *    block i covers rows [i*b, min(N, (i+1)*b)) (the last may be ragged).
 *  - Grouped-query attention: query head h uses KV head h / (Hq / Hkv).
 *  - Memory: the caller allocates and owns every buffer. Device pointers are
 *    CUDA device (or managed) memory, 16-byte aligned. No call allocates
 *    device memory; the global state is one device-side error word, per
 *    device the two copy streams and events of ba_att_forward_host, and the
 *    static scratch of ba_att_forward_host_noalloc: a __device__ array of
 *    BA_ATT_STATIC_SCRATCH_BYTES (512 MiB) that the library's device code
 *    reserves on every device where it is loaded, whichever calls are made.
 *  - Streams: every call is asynchronous on `stream` (NULL = legacy default
 *    stream) and never synchronises, except ba_att_get_device_error.
 *  - Errors: arguments are checked on the host before anything is launched;
 *    a bad argument returns a status and launches nothing. A failed launch
 *    returns BA_ERR_CUDA. Inconsistent data discovered on the device (an
 *    out-of-range block index, a count above kmax, a list not strictly
 *    ascending) never traps: the offending entry is skipped, a bit is set in
 *    the device error word, and ba_att_get_device_error reports it later.
 */
#ifndef BA_ATT_H
#define BA_ATT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so the header needs no CUDA. */
typedef struct CUstream_st *ba_stream_t;

typedef enum {
  BA_OK = 0,
  BA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, keep outside (0,1], ... */
  BA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d = 96)        */
  BA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned               */
  BA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
  BA_ERR_DEVICE = 5,        /* device-side data check failed (see error word) */
  BA_ERR_TIMEOUT = 6        /* a bounded device-side wait ran out             */
} ba_status;

typedef enum { BA_DTYPE_F32 = 0, BA_DTYPE_BF16 = 1 } ba_dtype;

/* Device error word bits (ba_att_get_device_error). */
#define BA_DEVERR_BAD_INDEX     0x1u  /* block index outside [0, nk)          */
#define BA_DEVERR_BAD_COUNT     0x2u  /* count outside [0, kmax]              */
#define BA_DEVERR_NOT_ASCENDING 0x4u  /* list entries not strictly ascending  */
#define BA_DEVERR_WAIT_TIMEOUT  0x8u  /* a bounded barrier wait gave up       */

typedef struct {
  int32_t B;        /* batch                                   >= 1          */
  int32_t Hq;       /* query heads                             >= 1          */
  int32_t Hkv;      /* key/value heads, divides Hq             >= 1          */
  int32_t N;        /* valid tokens per head                   >= 1          */
  int32_t N_alloc;  /* rows allocated per head                 >= N          */
  int32_t d;        /* head dimension: 64 or 128                             */
  int32_t block;    /* block size b: a multiple of 16 in [16, 256]           */
  int32_t dtype;    /* ba_dtype of Q, K and V (and of O unless stated)      */
  float sm_scale;   /* softmax scale s; <= 0 selects d^-1/2                  */
  int32_t block_k;  /* key block size b_k when it differs from b (asymmetric
                       blocks): a multiple of 16 in [16, 256]; 0 = b          */
} ba_att_shape;

/* Block geometry: query blocks have b = block rows, key blocks b_k rows
 * (b_k = block_k, or block when block_k is 0); nq = ceil(N / b) and
 * nk = ceil(N / b_k). Query-side arrays (statistics of Q, lists, counts,
 * score rows) have nq blocks, key-side ones (statistics of K, score
 * columns, list entries) nk. The pages use one block size for both; unequal
 * sizes are an extension. */

/* Library version string, e.g. "0.1.0 sm_100a". Never NULL. */
const char *ba_att_version(void);

/* Human-readable name of a status. Never NULL. */
const char *ba_att_status_string(ba_status status);

/* nq = ceil(N / block), query blocks; -1 if the shape is invalid. */
int32_t ba_att_num_blocks(const ba_att_shape *shape);

/* nk = ceil(N / b_k), key blocks; -1 if the shape is invalid. */
int32_t ba_att_num_key_blocks(const ba_att_shape *shape);

/* Kept blocks per query block: max(1, ceil(keep * nk)) (the selector keeps
 * the top fraction of key blocks; "Core claim"). -1 if keep is outside (0,1]
 * or the shape is invalid. */
int32_t ba_att_keep_count(const ba_att_shape *shape, double keep);

/*
 * ba_att_stats — stage one, block-wise pre-downsample statistics
 * (BA-Att abstract: Q and K are pooled per block before any scoring;
 * "Core claim": the correction uses per-dimension Q/K variances).
 *
 * For every block i and head h, over the valid rows r of the block:
 *   mean[i, m] = (1/n_i) sum_r x[r, m]
 *   var [i, m] = (1/n_i) sum_r (x[r, m] - mean[i, m])^2     (population)
 * computed in fp32 from the per-column sums of the deviations from the
 * block's first row c: mean = c + S1/n, var = (S2 - S1^2/n)/n, at least 0
 * (S1 = sum (x - c), S2 = sum (x - c)^2, rows summed in order). A column
 * that does not vary within a block has variance exactly 0.
 *
 * Q, K      device, [B,Hq|Hkv,N_alloc,d] of shape->dtype; read once.
 * q_mean, q_var   device fp32 [B, Hq,  nq, d]  (written)
 * k_mean, k_var   device fp32 [B, Hkv, nk, d]  (written)
 */
ba_status ba_att_stats(const ba_att_shape *shape, const void *Q, const void *K,
                       float *q_mean, float *q_var, float *k_mean, float *k_var,
                       ba_stream_t stream);

/*
 * ba_att_select — covariance-compensated block scores + norm sorting
 * (BA-Att abstract and "Core claim": score blocks in the downsampled space,
 * correct the pooled score with diagonal Q/K variances, sort, keep the top
 * fraction; Figure 2 names the sorted metric).
 *
 *   S~[i, j] = s * qbar_i . kbar_j
 *            + (s^2/2) * sum_m ( vq_i,m kbar_j,m^2 + qbar_i,m^2 vk_j,m + vq_i,m vk_j,m )
 *            + ln m_j
 * i.e. ln E[e^x] for the Gaussian model x = s q.k with q, k independent with
 * the block means and diagonal variances, summed over the m_j keys of block j.
 * Per (batch, query head, query block) the key blocks are ranked by S~
 * descending (ties: lower j first) and the first k = ba_att_keep_count(keep)
 * are kept and written in ascending order.
 *
 * q_mean..k_var   device fp32, as written by ba_att_stats.
 * kv_idx          device int32 [B, Hq, nq, kmax]: kept key-block indices,
 *                 ascending; entries at positions >= count are set to -1.
 * kv_cnt          device int32 [B, Hq, nq]: number kept (= k).
 * kmax            row stride of kv_idx; must be >= k.
 * block_scores    device fp32 [B, Hq, nq, nk], caller-owned, required: the
 *                 full S~ map is written there first and the top-k pass
 *                 reads it back, so on return it holds the score map.
 *                 NULL -> BA_ERR_INVALID_ARG; misaligned (not 16 B) ->
 *                 BA_ERR_MISALIGNED.
 * Requires nk <= 4096 (BA_ERR_UNSUPPORTED above).
 */
ba_status ba_att_select(const ba_att_shape *shape, double keep,
                        const float *q_mean, const float *q_var,
                        const float *k_mean, const float *k_var,
                        int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax,
                        float *block_scores, ba_stream_t stream);

/*
 * ba_att_topk — the norm sorting step alone, on a score map the caller gives
 * (BA-Att "The pith", abstract, Figure 2: the downsampled blocks are ranked
 * and the top fraction is kept). Per row of `block_scores`, the k columns
 * with the largest scores are kept (ranking by score descending, equal
 * scores to the lower column, NaN last) and written ascending. This is the
 * step ba_att_select runs after its score GEMM.
 *
 * block_scores  device fp32 [rows, nk], 16-byte aligned.
 * kv_idx        device int32 [rows, kmax]: kept columns, ascending; entries
 *               at positions >= k are -1.
 * kv_cnt        device int32 [rows]: k (nk when k >= nk).
 * 1 <= k, k <= kmax, 1 <= nk <= 4096, rows >= 1 (else BA_ERR_INVALID_ARG or,
 * for nk, BA_ERR_UNSUPPORTED).
 */
ba_status ba_att_topk(const float *block_scores, int64_t rows, int32_t nk, int32_t k,
                      int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax, ba_stream_t stream);

/*
 * ba_att_selector_workspace — device workspace bytes that ba_att_selector
 * needs for this shape: the augmented score features of every block
 * (6 planes (3 parts x {hi, lo}) x (B*Hq*nq + B*Hkv*nk) rows x d bf16), then
 * room for the score map [B, Hq, nq, nk] fp32 for callers that pass no
 * block_scores; each part rounded up to 256 bytes. -1 for an invalid shape.
 */
int64_t ba_att_selector_workspace(const ba_att_shape *shape);

/*
 * ba_att_selector — the whole selector stage in one call: ba_att_stats,
 * then the scores and norm sorting of ba_att_select (default ranking, no
 * variant flags). The pages give the two steps as one stage (BA-Att
 * abstract, "Core claim": pooled means and diagonal variances, the corrected
 * block score, sort and keep); there is no separate counterpart for the
 * feature workspace, which is a layout of this implementation.
 *
 * The statistics pass also writes, per block, the augmented features of the
 * score dot product (S~ = sum over parts p of q~_p . k~_p + ln m_j):
 *   q~ = [ s*qbar, (s^2/2)*vq, (s^2/2)*qbar^2 ],  k~ = [ kbar, kbar^2 + vk, vk ]
 * each split x = hi + lo into two bf16s (hi = RN(x), lo = RN(x - hi)), into
 * `workspace`; the score GEMM reads them instead of deriving them per tile.
 * Outputs are bit-identical to ba_att_stats followed by ba_att_select.
 *
 * Q, K, q_mean..k_var, kv_idx, kv_cnt, kmax: as for ba_att_stats and
 * ba_att_select.
 * block_scores  nullable: device fp32 [B, Hq, nq, nk], 16-byte aligned,
 *             which then holds the score map on return; NULL keeps the map
 *             inside the workspace (it is not returned).
 * workspace   device, caller-owned, >= ba_att_selector_workspace(shape)
 *             bytes, 16-byte aligned; its contents on return are unspecified.
 * Shapes with more than 2^31 - 129 feature rows (B*Hq*nq) run ba_att_stats
 * and ba_att_select instead (the score map then still goes to block_scores or
 * the workspace). NULL pointers other than block_scores ->
 * BA_ERR_INVALID_ARG; misaligned -> BA_ERR_MISALIGNED; nk > 4096 ->
 * BA_ERR_UNSUPPORTED.
 */
ba_status ba_att_selector(const ba_att_shape *shape, double keep,
                          const void *Q, const void *K,
                          float *q_mean, float *q_var, float *k_mean, float *k_var,
                          void *workspace, float *block_scores,
                          int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax,
                          ba_stream_t stream);

/*
 * ba_att_split_lists — partition every kept-block list at a key-block
 * boundary into a block-external span (blocks < split_block) and a
 * block-internal span (blocks >= split_block) (FlashBlock Eq. 5: the two
 * parts are attended separately and merged with ba_att_merge_lse).
 *
 * kv_idx, kv_cnt        device int32 input lists, layout as ba_att_select.
 * lo_idx/lo_cnt, hi_idx/hi_cnt   device int32 outputs, same layouts and kmax;
 *                       unused entries are -1. Input entries that are out of
 *                       range are dropped and flagged in the error word.
 * 0 <= split_block <= nk.
 */
ba_status ba_att_split_lists(const ba_att_shape *shape, int32_t split_block,
                             const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax,
                             int32_t *lo_idx, int32_t *lo_cnt,
                             int32_t *hi_idx, int32_t *hi_cnt, ba_stream_t stream);

/* Selection variants for ba_att_select_ex (bit flags; the pages fix none of
 * them, they are options around the ranking of "The pith" / "Core claim"). */
#define BA_SELECT_NO_VAR_PRODUCT  0x1u  /* drop the var_q * var_k term of the correction   */
#define BA_SELECT_FORCE_DIAGONAL  0x2u  /* query block i always keeps key block i           */
#define BA_SELECT_SHARED_GQA      0x4u  /* one selection per KV group: mean S~ of its heads */
#define BA_SELECT_BY_MASS         0x8u  /* keep the shortest top prefix with softmax share >= keep */

/*
 * ba_att_select_ex — ba_att_select with selection variants (flags, above).
 *  - NO_VAR_PRODUCT: S~ without the (s^2/2) sum_m vq_i,m vk_j,m term; the
 *    score map holds this S~.
 *  - FORCE_DIAGONAL: block i of every query block i is kept and ranked
 *    first; the other k-1 follow the usual ranking.
 *  - SHARED_GQA: the Hq/Hkv query heads of each KV group rank key blocks by
 *    the mean of their S~ (fp32, summed in head order) and all receive the
 *    same list; the score map still holds each head's own S~.
 *  - BY_MASS: keep is a target share tau in (0, 1]: per query block, the
 *    shortest prefix of the ranking (S~ descending, ties to the lower j)
 *    whose share of softmax_j S~ (fp32) reaches tau, at least one block;
 *    counts vary per row, so kmax must be >= nk (BA_ERR_INVALID_ARG
 *    otherwise). Not combined with FORCE_DIAGONAL (BA_ERR_UNSUPPORTED).
 * flags = 0 is ba_att_select. FORCE_DIAGONAL, SHARED_GQA and BY_MASS require
 * nk <= 1024 (BA_ERR_UNSUPPORTED above); unknown bits -> BA_ERR_INVALID_ARG.
 * Other arguments as for ba_att_select.
 */
ba_status ba_att_select_ex(const ba_att_shape *shape, double keep, uint32_t flags,
                           const float *q_mean, const float *q_var,
                           const float *k_mean, const float *k_var,
                           int32_t *kv_idx, int32_t *kv_cnt, int32_t kmax,
                           float *block_scores, ba_stream_t stream);

/*
 * ba_att_complement_lists — for every kept-block list, the key blocks of
 * [0, nk) it leaves out, ascending ("FlashBlock", review of Fig. 6: sparse
 * attention plus a cached residual over the unselected blocks; by Eq. 5 and
 * Eq. 9, attention over a list merged with attention over its complement is
 * dense attention). Pairs with ba_att_sparse_fwd / ba_att_sparse_fwd_merge.
 *
 * kv_idx, kv_cnt, kmax   device int32 lists as written by ba_att_select;
 *                        entries outside [0, nk) are ignored and flagged in
 *                        the device error word.
 * c_idx   device int32 [B, Hq, nq, c_kmax]: the complement, ascending,
 *         -1 padded; c_kmax >= nk (BA_ERR_INVALID_ARG otherwise).
 * c_cnt   device int32 [B, Hq, nq]: its length, nk minus the distinct valid
 *         entries. Requires nk <= 4096 (BA_ERR_UNSUPPORTED above).
 */
ba_status ba_att_complement_lists(const ba_att_shape *shape, const int32_t *kv_idx, const int32_t *kv_cnt,
                                  int32_t kmax, int32_t *c_idx, int32_t *c_cnt, int32_t c_kmax,
                                  ba_stream_t stream);

/*
 * ba_att_sparse_fwd — block-sparse bidirectional attention forward
 * (BA-Att abstract and Figure 4: attention evaluated only over the kept
 * blocks, no causal mask).
 *
 * For every valid row r of query block i, with C_i the valid keys of blocks
 * kv_idx[i, 0..kv_cnt[i]):
 *   LSE[r] = ln sum_{c in C_i} exp(s q_r . k_c)
 *   O[r]   = sum_{c in C_i} exp(s q_r . k_c - LSE[r]) v_c
 * computed with an online softmax over the kept blocks, fp32 accumulation,
 * O rounded to nearest-even into shape->dtype. An empty list gives O[r] = 0
 * and LSE[r] = -inf. Rows >= N are not written.
 *
 * Q, K, V   device, shape->dtype, layouts as above.
 * kv_idx, kv_cnt, kmax   device int32 lists as written by ba_att_select
 *           (any strictly ascending lists in [0, nk) are accepted).
 * O         device [B, Hq, N_alloc, d] of o_dtype (written).
 * o_dtype   shape->dtype, or BA_DTYPE_F32 to keep a partial output in fp32
 *           (one rounding in total when partials are merged later).
 * LSE       device fp32 [B, Hq, N_alloc], natural log (written).
 * Paths: bf16 with d = 64 or 128, block = 64, 128 or 256 and key blocks of
 * 64, 128 or 256 rows runs the tcgen05/TMEM tensor-core kernel (key blocks
 * are taken as 64-key halves). A 256-row block with d = 128 runs on a pair
 * of CTAs (a 2-CTA cluster, cta_group::2 MMAs of 256 rows) that share each
 * K/V half; with d = 64 it is two 128-row tiles sharing its list. Two
 * 64-row blocks share one 128-row tile, which attends the union of their
 * lists, each row masking the key blocks its own list leaves out. Every
 * other supported shape runs an fp32 CUDA-core kernel.
 */
ba_status ba_att_sparse_fwd(const ba_att_shape *shape,
                            const void *Q, const void *K, const void *V,
                            const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax,
                            void *O, int32_t o_dtype, float *LSE, ba_stream_t stream);

/*
 * ba_att_sparse_fwd_merge — ba_att_sparse_fwd over the listed blocks, merged
 * in the epilogue with an earlier partial over a disjoint key set
 * (FlashBlock Eq. 5 and Eq. 9: attention over X u Y from the parts over X
 * and Y). The result equals ba_att_sparse_fwd into an fp32 partial followed
 * by ba_att_merge_lse(O_prev, LSE_prev, that partial) bit for bit (the same
 * rounding steps), without writing or reading the second partial.
 *
 * O_prev    device fp32 [B, Hq, N_alloc, d]: the earlier partial, e.g. a
 *           ba_att_sparse_fwd with o_dtype = BA_DTYPE_F32 over another span.
 * LSE_prev  device fp32 [B, Hq, N_alloc]: its log-sum-exp.
 * O, LSE    as for ba_att_sparse_fwd (o_dtype = shape dtype or fp32); with
 *           fp32 output O may be O_prev and LSE may be LSE_prev (in place).
 * Other arguments and paths as for ba_att_sparse_fwd. NULL O_prev or
 * LSE_prev -> BA_ERR_INVALID_ARG.
 */
ba_status ba_att_sparse_fwd_merge(const ba_att_shape *shape,
                                  const void *Q, const void *K, const void *V,
                                  const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax,
                                  const float *O_prev, const float *LSE_prev,
                                  void *O, int32_t o_dtype, float *LSE, ba_stream_t stream);

/*
 * ba_att_sparse_fwd_rows — block-sparse attention for one range of query
 * rows only, optionally merged with a cached partial of those rows
 * (FlashBlock "Core claim" and "What carries the argument": during block
 * diffusion the attention of the current block's queries to the tokens
 * outside the block changes little between steps, so its (O, LSE) is cached
 * and only the attention inside the current block is recomputed, then merged
 * in log space by Eq. 9; the key access per step then scales with the block,
 * not with the sequence).
 *
 * Query side: q_rows valid rows per (batch, query head), at a stride of
 * q_stride rows (q_stride >= q_rows), cut into nqr = ceil(q_rows / block)
 * query blocks of shape->block rows (the last may be ragged). Q is
 * [B, Hq, q_stride, d] of shape->dtype; O, LSE, O_prev and LSE_prev use the
 * same row stride. Q may be a compact buffer of the range (q_stride = q_rows)
 * or point at row r0 of a full [B, Hq, N_alloc, d] tensor (Q + r0*d, with
 * q_stride = N_alloc; r0 a multiple of 8 keeps the 16-byte alignment).
 * Key side: K, V, N, N_alloc, Hkv, block_k and sm_scale as in shape.
 * kv_idx  device int32 [B, Hq, nqr, kmax], kv_cnt [B, Hq, nqr]: per query
 *         block of the range, its key blocks in [0, nk), strictly ascending.
 * O_prev, LSE_prev   nullable (both or neither): fp32 [B, Hq, q_stride, d]
 *         and [B, Hq, q_stride], the cached partial of these rows over a key
 *         set disjoint from the listed blocks; the epilogue merges it exactly
 *         as ba_att_sparse_fwd_merge does. With o_dtype = BA_DTYPE_F32, O may
 *         be O_prev and LSE may be LSE_prev (in place).
 * O       device [B, Hq, q_stride, d] of o_dtype (shape->dtype or fp32);
 *         LSE device fp32 [B, Hq, q_stride]. Rows >= q_rows are not written.
 * One CTA (or CUDA-core block) is launched per query tile of the range only,
 * B * Hq * nqr tiles in all. Results equal ba_att_sparse_fwd (or _merge) on
 * the same rows bit for bit. Paths as for ba_att_sparse_fwd. q_rows < 1 or
 * q_stride < q_rows -> BA_ERR_INVALID_ARG; one of O_prev, LSE_prev NULL ->
 * BA_ERR_INVALID_ARG.
 */
ba_status ba_att_sparse_fwd_rows(const ba_att_shape *shape, int32_t q_rows, int32_t q_stride,
                                 const void *Q, const void *K, const void *V,
                                 const int32_t *kv_idx, const int32_t *kv_cnt, int32_t kmax,
                                 const float *O_prev, const float *LSE_prev,
                                 void *O, int32_t o_dtype, float *LSE, ba_stream_t stream);

/*
 * ba_att_merge_lse — log-space merge of two partial attentions over disjoint
 * key sets (FlashBlock Eq. 9, decomposition of Eq. 5):
 *   m = max(L1, L2), w_k = exp(L_k - m),
 *   O = (w1 O1 + w2 O2) / (w1 + w2),  L = m + ln(w1 + w2);
 * both L = -inf gives O = 0, L = -inf.
 *
 * rows      number of rows (e.g. B*Hq*N_alloc); d in {64, 128}.
 * O1, O2    device [rows, d] of in_dtype; O device [rows, d] of out_dtype;
 *           L1, L2, L device fp32 [rows]. Math in fp32, one rounding to
 *           out_dtype.
 * When in_dtype == out_dtype, O may alias O1 or O2 and L may alias L1 or L2
 * (in-place merge).
 */
ba_status ba_att_merge_lse(int64_t rows, int32_t d, int32_t in_dtype, int32_t out_dtype,
                           const void *O1, const float *L1,
                           const void *O2, const float *L2,
                           void *O, float *L, ba_stream_t stream);

/*
 * ba_att_forward_host_workspace — device workspace bytes that
 * ba_att_forward_host needs for this shape, keep, split and chunking; -1 for
 * arguments ba_att_forward_host would reject.
 */
int64_t ba_att_forward_host_workspace(const ba_att_shape *shape, double keep, int32_t split_block,
                                      int32_t kv_heads_per_chunk);

/*
 * ba_att_forward_host — the whole BA-Att forward from HOST buffers to HOST
 * buffers: H2D of Q, K, V; ba_att_stats; ba_att_select; then either one
 * ba_att_sparse_fwd (split_block < 0), or (split_block >= 0) the key set split
 * at that key block (FlashBlock Eq. 5), ba_att_sparse_fwd over the first span
 * into an fp32 partial and ba_att_sparse_fwd_merge over the second (the
 * FlashBlock Eq. 9 merge in its epilogue); D2H of O and LSE.
 * The pages define the operator only; the pipelining is this library's.
 *
 * The work is cut into chunks of kv_heads_per_chunk KV heads (with their
 * Hq/Hkv query heads each) of one batch entry; <= 0 picks the fewest KV heads
 * that give about 1024 (query head, query block) tiles per chunk. Chunk c+1's inputs are copied in, and chunk c-1's outputs
 * copied out, on two internal non-blocking streams while chunk c computes
 * on `stream`; every result equals that of the device-resident calls above
 * bit for bit, as each chunk runs the same kernels on the same heads.
 *
 * Q, K, V   host [B, Hq|Hkv, N_alloc, d] of shape->dtype; pinned (page-locked)
 *           memory lets the copies overlap compute, pageable memory works
 *           but serialises them.
 * O         host [B, Hq, N_alloc, d] of shape->dtype; LSE host fp32
 *           [B, Hq, N_alloc]. Rows n < N of each head are written, padding
 *           rows are left untouched.
 * workspace device memory of at least ba_att_forward_host_workspace(...)
 *           bytes, 256-byte aligned, owned by the caller and not used by
 *           anything else until `stream` has passed this call.
 * Returns once everything is enqueued; results are on the host when
 * `stream` reaches the point of the call (e.g. after cudaStreamSynchronize).
 * Calls for one device are enqueued one at a time (an internal lock), since
 * they share the two copy streams. A status other than BA_OK may leave part
 * of the work enqueued; `stream` still waits for all of it.
 */
ba_status ba_att_forward_host(const ba_att_shape *shape, double keep, int32_t split_block,
                              int32_t kv_heads_per_chunk,
                              const void *Q, const void *K, const void *V,
                              void *O, float *LSE,
                              void *workspace, int64_t workspace_bytes, ba_stream_t stream);

/* Size of the library's static device scratch (ba_att_forward_host_noalloc). */
#define BA_ATT_STATIC_SCRATCH_BYTES (512ull << 20)

/*
 * ba_att_forward_host_noalloc — ba_att_forward_host without a workspace
 * argument. The pages have no counterpart: this is a deployment variant of
 * the same computation.
 *
 * The workspace is a static __device__ array of BA_ATT_STATIC_SCRATCH_BYTES
 * inside the library (reserved on every device where the library's device
 * code is loaded, at load time, whether or not this call is ever made;
 * nothing is allocated at call time). The chunk is the one
 * ba_att_forward_host picks for kv_heads_per_chunk <= 0 (about 1024 query
 * tiles, so that copies overlap compute), narrowed until its workspace
 * (ba_att_forward_host_workspace) fits the scratch; BA_ERR_UNSUPPORTED when
 * one KV head per chunk does not fit (e.g. 32 query heads per KV head at
 * N = 128K with a split). Results are bit-identical to
 * ba_att_forward_host. The scratch is shared by all calls on a device: each
 * call starts on `stream` only after the previous call on the scratch has
 * ended, whatever stream that call used.
 * Arguments as for ba_att_forward_host.
 */
ba_status ba_att_forward_host_noalloc(const ba_att_shape *shape, double keep, int32_t split_block,
                                      const void *Q, const void *K, const void *V,
                                      void *O, float *LSE, ba_stream_t stream);

/*
 * ba_att_get_device_error — synchronise `stream`, read the device error word
 * of the current device, clear it, and return BA_OK (word 0), BA_ERR_TIMEOUT
 * (timeout bit set) or BA_ERR_DEVICE (any other bit). *word_out (nullable)
 * receives the raw bits.
 */
ba_status ba_att_get_device_error(ba_stream_t stream, uint32_t *word_out);

/*
 * ba_att_selftest_bounded_wait — launch one CTA that waits on a shared-memory
 * barrier no thread ever arrives on, giving up after timeout_us microseconds
 * (1 <= timeout_us <= 2000000). It exercises the bounded-wait path every
 * pipelined kernel here uses: the wait must end, set BA_DEVERR_WAIT_TIMEOUT
 * and leave the context usable. No counterpart on the pages.
 */
ba_status ba_att_selftest_bounded_wait(uint32_t timeout_us, ba_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BA_ATT_H */
