/*
 * hs2.h - C ABI of the HySparse2 hybrid-block attention path on NVIDIA B200 (sm_100a).
 *
 * One Hybrid Block = one Full Attention layer followed by several Sparse
 * Attention layers.  The full-attention layer reads the whole KV cache and also
 * decides which tokens matter; the sparse layers reuse that cache and that
 * token selection (KV Reuse).  Sources, by page title and section:
 *   [HT]  "Xiaomi Unveils HySparse2 for Faster Long-Context AI",
 *         sections "Two-Level KV Sharing" and "Token-Level Selection and
 *         Unified Local Access".
 *   [OH]  "Xiaomi Releases HySparse2, Targeting Long-Horizon Reasoning for
 *         Agents", section "From Hybrid SWA to HySparse2, Xiaomi Continues to
 *         Refine the Attention Structure".
 *   [BB]  "Xiaomi discloses MiMo-V3 plans to adopt HySparse2 architecture",
 *         section "Article".
 *   [LF]  "MiMo-V3 Architecture Revealed: HySparse2 ...", section
 *         "Token-Level Sparse Selection and Deployment Optimization".
 *
 * The four calls of one decode or chunk step, in order:
 *   hs2_full_attn_scores  full attention of the query tokens + per-key scores
 *   hs2_topk_select       token-level top-k outside the window, plus the window
 *   hs2_sparse_attn       one sparse layer over the selected rows (call once
 *                         per reuse layer, each with its own queries)
 *   hs2_block_select      (comparison path) first-generation block selection
 * and, before them in a decode step, hs2_kv_append (the new tokens' K/V rows
 * written into the cache).  A decode step whose cache is split by position
 * across GPUs uses the hs2_cp_* calls instead (context parallelism, below).
 *
 * Conventions shared by every call
 * --------------------------------
 * Layout.  Token-major and packed over the batch.  For B sequences with query
 *   lengths Tq_b and cache lengths N_b:
 *     Q, O        [total_q,  Hq,  D]   total_q  = sum_b Tq_b
 *     K, V        [total_kv, Hkv, D]   total_kv = sum_b N_b
 *   contiguous, row-major, element type ``dtype`` (HS2_BF16 or HS2_F32; all
 *   of Q, K, V and O share it).  Query head h reads KV head h / (Hq / Hkv).
 *   D must be 128.  Query row i (0-based) of sequence b sits at absolute
 *   position t = N_b - Tq_b + i and sees cache positions 0..t (causal).  The
 *   query's own key is already in the cache.
 * Rows.  A selection row is one (query row, KV head) pair:
 *   row = query_row * Hkv + kv_head, R = total_q * Hkv rows.
 * Scores.  float32 [R, score_stride]: entry j of a row is the score of cache
 *   position j of that row's sequence.  Only entries 0..t are defined.
 * Indices.  int32 positions relative to the start of the row's sequence.
 * Pointers.  Every tensor pointer is a DEVICE pointer, 16-byte aligned.  The
 *   offsets in hs2_problem are device pointers too; their host copies
 *   total_q / total_kv / max_q_len / max_kv_len must agree with them.
 * Ownership.  The caller owns every buffer, including the workspace.  The
 *   library allocates no memory, never synchronises (except
 *   hs2_get_last_device_error) and launches only on ``stream``
 *   (a cudaStream_t; NULL is the legacy default stream).  Calls that use the
 *   same workspace must not overlap.
 * Workspace.  Query the size with the matching *_workspace_size call; pass at
 *   least that many bytes, 256-byte aligned.  Its contents on entry do not
 *   matter; on return they are unspecified - except that hs2_cp_scores reads
 *   the logits hs2_cp_attn_partial left in the same workspace.
 * Empty steps.  When total_q = 0 (no query rows) a call checks the problem
 *   and its scalar arguments, launches nothing and returns HS2_OK; its tensor
 *   and workspace pointers are not used and may be null.
 * Errors.  Arguments are checked on the host before any launch; a failed check
 *   returns an error code and launches nothing.  A CUDA launch failure returns
 *   HS2_ERR_CUDA.  Conditions only the device can see (offsets that disagree
 *   with the host totals, an index outside 0..t) are recorded in a device error
 *   word, the offending work is skipped, and hs2_get_last_device_error reports
 *   them.  Inputs must be finite; NaN / Inf give unspecified results.
 */
#ifndef HS2_H
#define HS2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARG = -1,  /* bad pointer, size, stride or shape                */
  HS2_ERR_UNSUPPORTED = -2,  /* valid but not built (D != 128, group size, ...)     */
  HS2_ERR_WORKSPACE = -3,    /* workspace missing, too small or misaligned          */
  HS2_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed          */
  HS2_ERR_TIMEOUT = -5,      /* a bounded device-side wait ran out                   */
  HS2_ERR_DEVICE_INPUT = -6  /* the device found inputs that break the contract      */
} hs2_status;

typedef enum { HS2_F32 = 0, HS2_BF16 = 1 } hs2_dtype;

/* Shapes of one batch.  All fields are read on the host; the two offset
 * arrays are device pointers read by the kernels. */
typedef struct {
  int32_t B;                 /* sequences in the batch, >= 1                        */
  int32_t Hq;                /* query heads                                         */
  int32_t Hkv;               /* KV heads; Hq % Hkv == 0                             */
  int32_t D;                 /* head dimension; must be 128                         */
  int32_t dtype;             /* hs2_dtype of Q, K, V, O                             */
  int32_t reserved;          /* must be 0                                           */
  const int64_t* q_offsets;  /* device [B+1], prefix sums of Tq_b, q_offsets[0] = 0  */
  const int64_t* kv_offsets; /* device [B+1], prefix sums of N_b,  kv_offsets[0] = 0 */
  int64_t total_q;           /* = q_offsets[B]                                      */
  int64_t total_kv;          /* = kv_offsets[B]                                     */
  int64_t max_q_len;         /* >= every Tq_b; 1 selects the decode kernels          */
  int64_t max_kv_len;        /* >= every N_b; every N_b must be >= Tq_b             */
  float scale;               /* softmax scale applied to q.k, e.g. 1/sqrt(D)        */
} hs2_problem;

/* ---------------------------------------------------------------------------
 * hs2_full_attn_scores - the Full Attention layer of a Hybrid Block, which
 * both produces the attention output over the whole KV cache and decides
 * which tokens are important ([OH]; [HT] "Two-Level KV Sharing", KV Reuse).
 *
 * For every query row (position t) and query head h:
 *   x_j = scale * q_h . k_{g(h), j}   for j = 0..t
 *   P_hj = exp(x_j - max x) / sum_j exp(x_j - max x),   O_h = sum_j P_hj v_j
 * and, for every KV head g, the selection score of position j
 *   scores[row(query, g)][j] = sum over the G query heads h of group g of P_hj
 * (the pages do not define the score; this sum of the group's probabilities is
 * the reading this library implements).  Scores are float32; O has ``dtype``.
 *
 * Q [total_q, Hq, D], K / V [total_kv, Hkv, D]: inputs.  O [total_q, Hq, D]:
 * output.  scores [R, score_stride] float32: output, score_stride >= max_kv_len
 * (any value; rows need not be 16-byte aligned).  Entries 0..t of a row are
 * written; entries past t are left as they were.
 * Decode (max_q_len == 1) streams the cache once; chunks (max_q_len > 1) make a
 * second pass over K to write the scores.
 * Returns HS2_OK, or INVALID_ARG / UNSUPPORTED / WORKSPACE / CUDA.
 */
hs2_status hs2_full_attn_workspace_size(const hs2_problem* p, size_t* bytes);
/* The number of kernels one hs2_full_attn_scores call launches for ``p`` on
 * the current device (*n = 0 when total_q = 0): decode 2 (the pass, then the
 * O merge and score finalize); bf16 chunks 1, or 3 when the visible keys are
 * split over several CTAs per query tile (statistics, then scores and O
 * shares, then the O sum); float32 chunks 2.  Returns HS2_OK or INVALID_ARG. */
hs2_status hs2_full_attn_launches(const hs2_problem* p, int32_t* n);
hs2_status hs2_full_attn_scores(const hs2_problem* p, const void* Q, const void* K,
                                const void* V, void* O, float* scores, int64_t score_stride,
                                void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_topk_select - token-level selection ([HT] "Token-Level Selection and
 * Unified Local Access"; [BB]; [LF]).  For each row with query position t:
 *   window     = positions [max(0, t-window+1), t]          (always kept)
 *   candidates = positions [0, t-window]                    (outside the window)
 *   global     = the k candidates with the highest score; equal scores are
 *                ordered by lower position (deterministic, independent of
 *                the launch shape); all candidates if there are at most k.
 * idx [R, k+window] int32: output, global positions ascending, then the window
 * ascending, then -1 padding.  count [R] int32: output, number of valid
 * entries = min(#candidates, k) + min(t+1, window).
 * Scores are compared as float32 values (-0.0 == +0.0).  1 <= k, window.
 * Results are bit-identical to a full sort by (score desc, position asc).
 */
hs2_status hs2_topk_workspace_size(const hs2_problem* p, int32_t k, int32_t window,
                                   size_t* bytes);
hs2_status hs2_topk_select(const hs2_problem* p, const float* scores, int64_t score_stride,
                           int32_t k, int32_t window, int32_t* idx, int32_t* count,
                           void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_block_select - the first-generation HySparse block-level selection, kept
 * as a comparison path ([BB]: groups of 64 tokens kept whole).  Candidates as
 * in hs2_topk_select.  Block b covers positions [block*b, block*b+block-1];
 * its score is the maximum score of its candidate positions; blocks without a
 * candidate are not eligible.  The n_blocks best blocks (equal scores: lower
 * block index first) contribute all their candidate positions, ascending,
 * followed by the window.
 * idx [R, n_blocks*block + window] int32 (-1 padded), count [R] int32.
 * A row whose offsets give more candidates than score_stride is recorded as
 * HS2_ERR_DEVICE_INPUT and gets count 0 and all -1.
 */
hs2_status hs2_block_select_workspace_size(const hs2_problem* p, int32_t n_blocks,
                                           int32_t block, int32_t window, size_t* bytes);
hs2_status hs2_block_select(const hs2_problem* p, const float* scores, int64_t score_stride,
                            int32_t n_blocks, int32_t block, int32_t window, int32_t* idx,
                            int32_t* count, void* workspace, size_t workspace_bytes,
                            void* stream);

/* ---------------------------------------------------------------------------
 * hs2_sparse_attn - one Sparse Attention layer that reuses the full-attention
 * layer's KV cache and index set ([HT] "Two-Level KV Sharing", KV Reuse, and
 * "Token-Level Selection and Unified Local Access": local and global tokens in
 * one sparse computation over the shared cache).  For every query row and
 * query head h of KV group g, with I = idx[row(query, g)][0 .. count-1]:
 *   O_l,h = sum_{j in I} softmax_I(scale * q_l,h . k_{g,j}) v_{g,j}
 * Q_l [total_q, Hq, D]: this layer's queries.  K / V: the same cache as the
 * full-attention call.  idx [R, idx_stride], count [R]: from a select call
 * (0 <= count <= idx_stride).  O_l [total_q, Hq, D]: output.  A row with
 * count 0 gives O = 0.  An index outside 0..t is recorded as
 * HS2_ERR_DEVICE_INPUT and skipped.
 */
hs2_status hs2_sparse_attn_workspace_size(const hs2_problem* p, int32_t idx_stride,
                                          size_t* bytes);
hs2_status hs2_sparse_attn(const hs2_problem* p, const void* Q_l, const void* K,
                           const void* V, const int32_t* idx, const int32_t* count,
                           int32_t idx_stride, void* O_l, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_swa_attn - the sliding-window attention layer of the Hybrid SWA baseline
 * that the pages compare HySparse2 against ([OH] "From Hybrid SWA to
 * HySparse2 ...": the MiMo-V2 models mixed a few full-attention layers with
 * layers that attend only to a local neighbourhood).  For every query row at
 * position t and query head h of KV group g:
 *   O_h = sum_{j = max(0, t-window+1)}^{t} softmax_j(scale * q_h . k_{g,j}) v_{g,j}
 * The pages give no window size; it is an argument (window >= 1).  Q, O
 * [total_q, Hq, D]; K, V the layer's cache [total_kv, Hkv, D].  No workspace.
 * It runs the sparse-attention kernels with the window in place of an index
 * list; the result equals hs2_sparse_attn given the window positions.
 */
hs2_status hs2_swa_attn(const hs2_problem* p, const void* Q, const void* K, const void* V,
                        int32_t window, void* O, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_kv_bridge - KV Bridging ([HT] "Two-Level KV Sharing"): the KV cache of
 * a Cross-Decoder full-attention layer computed from the hidden states of the
 * matching Self-Decoder full-attention layer, one GEMM per matrix:
 *   K[n, g, :] = sum_i H[n, i] Wk_t[g*D + :, i]    (K = H Wk, with Wk_t = Wk^T)
 *   V[n, g, :] = sum_i H[n, i] Wv_t[g*D + :, i]
 * for every cache row n < total_kv.  The pages give neither the hidden size
 * nor the weights: both are arguments.  bf16 only (HS2_ERR_UNSUPPORTED
 * otherwise), fp32 accumulation, outputs rounded to bf16.
 * H [total_kv, hidden], Wk_t and Wv_t [Hkv*D, hidden] (row-major: one output
 * column's weights contiguous); hidden a positive multiple of 64.  K, V
 * [total_kv, Hkv, D]: written (all rows).  Only total_kv, Hkv, D and dtype of
 * the problem are used.  No workspace.
 */
hs2_status hs2_kv_bridge(const hs2_problem* p, const void* H, int32_t hidden, const void* Wk_t,
                         const void* Wv_t, void* K, void* V, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_kv_append - writes the K/V rows of a step's new tokens into the KV cache
 * that the full-attention layer produces and its sparse layers reuse ([HT]
 * "Two-Level KV Sharing"; [OH]: decoding extends the cache a token at a time).
 * Each new token's key goes to its own cache position: query row i of sequence
 * b (position t = N_b - Tq_b + i) writes K[kv_offsets[b] + t] and
 * V[kv_offsets[b] + t], all Hkv heads, which is where the attention calls of
 * the same step read it (the query's own key is in the cache).
 * K_new, V_new [total_q, Hkv, D]: the new rows (dtype of the problem).
 * K, V [total_kv, Hkv, D]: the cache, updated in place; no other row changes.
 * Needs no workspace.  A position outside the cache (offsets that disagree
 * with the host totals) is recorded as HS2_ERR_DEVICE_INPUT and skipped.
 */
hs2_status hs2_kv_append(const hs2_problem* p, const void* K_new, const void* V_new, void* K,
                         void* V, void* stream);

/* ---------------------------------------------------------------------------
 * hs2_block_select_noalloc - hs2_block_select for callers that cannot give
 * the library device memory (the pages have no counterpart: this is a
 * deployment convenience, not part of the method).  Some hosts cannot
 * allocate on the library's behalf: an engine or plugin interface that owns
 * every device allocation and passes no workspace pointer, or a caller that
 * must avoid cudaMalloc because it may synchronise the device and fragment a
 * memory pool the engine manages.  This call takes its scratch (block maxima
 * and chosen block ids) from a fixed 16 MiB array that the library keeps in
 * device memory; every GPU that loads the library holds that array until the
 * process exits.  It allocates nothing.
 *   - Arguments, outputs and results are those of hs2_block_select.
 *   - Limit: the scratch hs2_block_select_workspace_size reports for the same
 *     arguments must be at most 16 MiB (16,777,216 bytes); larger problems
 *     return HS2_ERR_WORKSPACE and launch nothing.
 *   - The first call on a device looks up the array's device address (a CUDA
 *     runtime query, no allocation).
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents.  Nothing in it needs to start at zero: every scratch entry
 *     whose value reaches idx or count was written earlier in the same call
 *     (a row the device rejects with HS2_ERR_DEVICE_INPUT gets count 0 and
 *     all -1, whatever the array held).  Calls that overlap on the GPU
 *     (different streams, or host threads without ordering) race on it:
 *     serialise them.
 */
hs2_status hs2_block_select_noalloc(const hs2_problem* p, const float* scores,
                                    int64_t score_stride, int32_t n_blocks, int32_t block,
                                    int32_t window, int32_t* idx, int32_t* count, void* stream);

/* ---------------------------------------------------------------------------
 * Context parallelism for decode (max_q_len == 1): the KV cache of every
 * sequence is split by position across R ranks (one process per GPU).  Rank r
 * holds the contiguous global positions [pos0[b], pos0[b] + n_b) of sequence
 * b, where n_b is the sequence length in the rank's own ("local") problem;
 * the ranks' ranges of a sequence are disjoint, cover it, and are ordered by
 * rank.  The pages describe one device ([OH], [HT] as above); the split and
 * these calls are this library's.  Each step computes the unsplit definition
 * of hs2_full_attn_scores / hs2_topk_select / hs2_sparse_attn exactly, up to
 * floating-point rounding order; between the steps the caller all-gathers the
 * small partials (e.g. NCCL over NVLink), stacking them in rank order.
 *
 * Per step and rank:
 *   1. hs2_cp_attn_partial (local problem) -> O_part, ml_part; all-gather;
 *      hs2_cp_merge -> O and the global (m, 1/l) of every (query, head).
 *   2. hs2_cp_scores (local problem, global ml) -> this rank's scores.
 *   3. hs2_cp_topk_local -> (score, global position) pairs; all-gather;
 *      hs2_cp_topk_merge (global problem) -> idx, count, identical on every
 *      rank and equal to hs2_topk_select on the unsplit scores.
 *   4. per sparse layer: hs2_cp_sparse_partial -> O_part, ml_part;
 *      all-gather; hs2_cp_merge -> O_l.
 * Partials: O_part [total_q, Hq, D] float32, each (query, head) normalised by
 * its own softmax sum; ml_part [total_q, Hq, 2] float32 = (m, 1/l), with
 * 1/l = 0 where the rank saw no key.  Stacked: [R, ...] in rank order.
 * Returns as the unsplit calls; HS2_ERR_UNSUPPORTED for max_q_len > 1.
 */

/* Full-attention pass over the rank's rows: partials O_part / ml_part; the
 * logits stay in ``workspace`` (hs2_full_attn_workspace_size bytes of the same
 * local problem) for hs2_cp_scores, which must get the same workspace. */
hs2_status hs2_cp_attn_partial(const hs2_problem* p, const void* Q, const void* K, const void* V,
                               float* O_part, float* ml_part, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Merge of R stacked partials of ``rows`` (query, head) rows: O [rows, D] of
 * ``dtype`` (HS2_BF16 or HS2_F32) and, if ml is not null, the merged (m, 1/l)
 * [rows, 2].  M = max_r m_r, w_r = l_r exp(m_r - M), O = sum_r w_r O_r / sum_r w_r. */
hs2_status hs2_cp_merge(int64_t rows, int32_t R, const float* O_parts, const float* ml_parts, int32_t dtype,
                        void* O, float* ml, void* stream);

/* Selection scores of the rank's own keys (local positions, as
 * hs2_full_attn_scores writes them) from the logits kept by
 * hs2_cp_attn_partial and the merged global ml [total_q, Hq, 2]. */
hs2_status hs2_cp_scores(const hs2_problem* p, const float* ml, float* scores, int64_t score_stride,
                         void* workspace, size_t workspace_bytes, void* stream);

/* The rank's top-(k + window) keys over all its positions (window positions
 * included: at most ``window`` of them can be), as pairs pair_score /
 * pair_pos [rows, k + window] (float32 score, int32 global position = pos0[b]
 * + local position; unused entries have position -1).  pos0: device [B].
 * idx_tmp [rows, k + window] and count_tmp [rows]: scratch. */
hs2_status hs2_cp_topk_local(const hs2_problem* p, const float* scores, int64_t score_stride, int32_t k,
                             int32_t window, const int64_t* pos0, int32_t* idx_tmp, int32_t* count_tmp,
                             float* pair_score, int32_t* pair_pos, void* stream);

/* Global selection from R stacked pair sets [R, rows, k + window] with the
 * GLOBAL problem (global kv offsets): positions <= t - window compete, the k
 * best by (score desc, position asc) ascending, then the window, then -1;
 * idx [rows, k + window], count [rows], as hs2_topk_select.  R (k + window)
 * <= 16384 and k <= 2048, else HS2_ERR_UNSUPPORTED. */
hs2_status hs2_cp_topk_merge(const hs2_problem* p, int32_t R, int32_t k, int32_t window, const float* pair_score,
                             const int32_t* pair_pos, int32_t* idx, int32_t* count, void* stream);

/* One sparse layer over the entries of the global list idx / count (global
 * positions, from hs2_cp_topk_merge) that fall in the rank's rows: partials
 * O_part / ml_part.  Entries outside the rank's rows are skipped silently
 * (so an invalid global position is not reported here). */
hs2_status hs2_cp_sparse_partial(const hs2_problem* p, const void* Q_l, const void* K, const void* V,
                                 const int32_t* idx, const int32_t* count, int32_t idx_stride,
                                 const int64_t* pos0, float* O_part, float* ml_part, void* stream);

/* ---------------------------------------------------------------------------
 * Device error word.  Synchronises ``stream``, returns the first error any
 * kernel of this library recorded on the current device since the last call
 * (HS2_OK if none) and clears it.  HS2_ERR_CUDA if the synchronisation fails.
 */
hs2_status hs2_get_last_device_error(void* stream);

/* ---------------------------------------------------------------------------
 * Failure-detection self-test.  The pages have no counterpart: this call
 * exists so that a test can watch one of the library's bounded device waits
 * run out without faulting or hanging the GPU.  It launches one 32-thread
 * block on ``stream`` whose single waiting thread waits for an event that
 * nothing ever produces:
 *   - mode 0: phase 0 of a shared-memory mbarrier that expects one arrival
 *     and never gets it (the form of every pipeline wait in the kernels);
 *   - mode 1: a device word that no code writes (the form of a flag wait).
 * The wait gives up after ``limit_cycles`` SM clock cycles (values above the
 * library's own wait limit, about 4e9 cycles, are clamped to it) and records
 * HS2_ERR_TIMEOUT in the device error word, which hs2_get_last_device_error
 * then returns and clears.  The context stays usable.
 *   - Returns HS2_OK once the launch is queued; HS2_ERR_INVALID_ARG for a
 *     mode other than 0 or 1 or a negative limit (nothing launched);
 *     HS2_ERR_CUDA if the launch fails.
 *   - Reads and writes no caller memory.
 */
hs2_status hs2_wait_selftest(int32_t mode, int64_t limit_cycles, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* hs2_status_string(hs2_status s);

/* Library version, (major << 16) | minor. */
int32_t hs2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HS2_H */
