/*
 * dsa.h -- C ABI of libdsa.so, the B200 (sm_100a) GQA-adapted DeepSeek Sparse
 * Attention (DSA) layer: lightning indexer -> causal top-k -> sparse GQA
 * attention, for prefill and for decode over a paged KV cache.
 *
 * Sources (web pages on the Kwai Keye-VL-2.0 technical report):
 *   [REVIEW]  "Kwai Keye-VL-2.0 Technical Report" paper review
 *             (xllm-io.github.io), section 三 "技术架构", "核心公式".
 *   [REPORT]  "快手开源 Kwai Keye-VL-2.0-30B-A3B：面向长视频理解与智能体智能的
 *             MoE 多模态模型" (translation of the report), sections 2.3.1,
 *             2.3.2, 5.1.2, 5.2.1 and 5.3.
 *
 * Conventions for every call
 * --------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller.  Layouts are
 *    row-major and dense unless a leading dimension is passed.  Shapes below
 *    use [a, b, c] with c fastest.
 *  - The library never allocates, frees or synchronises.  Temporary memory
 *    comes from a caller-provided workspace whose size a *_workspace_size()
 *    query returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and keep no state between calls, so separate calls on separate
 *    streams with separate buffers may run concurrently.
 *  - Arguments are validated on the host before any CUDA call.  On an error
 *    nothing is launched and no output is touched.  DSA_ERR_CUDA means a
 *    launch failed; the CUDA error string is available from
 *    dsa_last_error_string() on the calling thread.
 *  - FP8 means OCP e4m3fn bytes; the real value of a stored byte is
 *    e4m3(byte) * scale, one float scale per token.  bf16 tensors are passed
 *    as uint16_t bit patterns.  NaN / Inf inputs give unspecified results.
 *  - Index tensors are int32.  Selected-index rows are ascending and padded
 *    with -1.  Entries of an index row that fall outside the causally visible
 *    range are skipped by the attention kernels, so a corrupt row cannot make
 *    them read out of bounds.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#define DSA_VERSION 100      /* 1.0.0 */
#define DSA_PAGE_SIZE 64     /* tokens per KV-cache page */

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad range */
    DSA_ERR_UNSUPPORTED_SHAPE = 2, /* a head count or head dim this build has no kernel for */
    DSA_ERR_WORKSPACE = 3,         /* workspace missing or smaller than the size query */
    DSA_ERR_CUDA = 4,              /* a kernel launch failed */
    DSA_ERR_TIMEOUT = 5            /* a bounded device-side wait gave up (dsa_check_device_error) */
} dsa_status_t;

/* Human-readable name of a status code (static storage). */
DSA_API const char *dsa_status_string(dsa_status_t s);
/* DSA_VERSION of the loaded library. */
DSA_API int dsa_version(void);
/* Text of the last CUDA error seen by a dsa_* call on this thread ("" if none). */
DSA_API const char *dsa_last_error_string(void);
/* Diagnostic, not for the hot path: synchronises the current device, then
 * returns DSA_ERR_TIMEOUT if a kernel's bounded wait on an on-chip barrier
 * expired since the last call (the kernel then wrote incomplete results and
 * exited cleanly), DSA_OK otherwise.  Clears the flag. */
DSA_API dsa_status_t dsa_check_device_error(void);
/* Diagnostic, for tests of the failure path: sets, on the current device,
 * the time after which the prefill indexer's on-chip pipeline waits (between
 * its TMA, tensor-core and epilogue roles) give up, in nanoseconds; 0
 * restores the default of 2 s.  A wait that gives up sets the flag that
 * dsa_check_device_error reports, every role of the kernel unwinds (copies in
 * flight are drained, tensor memory is freed) and the scores are incomplete.
 * Synchronous; not for the hot path. */
DSA_API dsa_status_t dsa_set_wait_limit_ns(unsigned long long ns);

/* ------------------------------------------------------------------------
 * Lightning-indexer scores (prefill), one chunk of query rows.
 *
 * [REVIEW] 核心公式, indexer score; [REPORT] 2.3.1 (one key head shared by all
 * indexer heads, FP8, ReLU scoring):
 *     I[t,s] = sum_{j<HI} w[t,j] * ReLU( qI[t,j] . kI[s] ),   0 <= s <= t,
 *     qI[t,j,c] = e4m3(q8[t,j,c]) * q_scale[t],  kI[s,c] = e4m3(k8[s,c]) * k_scale[s].
 * The score matrix is produced one chunk of query rows at a time ([REPORT]
 * 5.2.1: the chunked indexer bounds peak memory).
 *
 *   q8       [L, HI, dI] e4m3      q_scale [L] float     w [L, HI] float
 *   k8       [L, dI]     e4m3      k_scale [L] float
 *   rows     t in [row_begin, row_begin + n_rows), 0 <= row_begin, row_begin + n_rows <= L
 *   scores   [n_rows, ld_scores] float; row r holds query t = row_begin + r;
 *            columns 0..t are written, columns > t are left unspecified.
 *            ld_scores >= row_begin + n_rows and ld_scores % 4 == 0.
 *   q8, k8 must be 16-byte aligned (they are read by the tensor-memory
 *   accelerator).
 *   row_stats  optional (NULL to skip): device buffer of
 *            dsa_row_stats_bytes(n_rows) bytes that receives, per row, the
 *            range of the scores just written.  Its layout is private to the
 *            library; passing it to dsa_topk for the same rows lets the top-k
 *            skip its own pass over the row to find that range.
 * Supported: dI in {32, 64, 128}; HI in {4, 8, 16, 32, 64}.
 * All scale factors must be positive (they commute with the ReLU).
 * ------------------------------------------------------------------------ */
DSA_API size_t dsa_row_stats_bytes(int n_rows);
DSA_API dsa_status_t dsa_indexer_scores(const uint8_t *q8, const float *q_scale, const float *w,
                                const uint8_t *k8, const float *k_scale,
                                int L, int HI, int dI, int row_begin, int n_rows,
                                float *scores, int64_t ld_scores, void *row_stats, void *stream);

/* ------------------------------------------------------------------------
 * Per-row top-k selection.
 *
 * [REVIEW] 核心公式, Omega_t = { s | I[t,s] in Top-k(I[t,:]) }; [REPORT] 2.3.1;
 * [REPORT] 5.1.2 (a row with fewer than k visible entries keeps all of them);
 * [REPORT] 5.2.1 (the selection must be deterministic).
 * Row r has n_r candidates scores[r * ld_scores + 0 .. n_r-1]:
 *   row_len == NULL: n_r = row_begin + r + 1 (causal prefill rows),
 *   row_len != NULL: n_r = row_len[r] (device int32 [n_rows]), clamped to [0, max_len].
 * Output idx [n_rows, k]: if n_r <= k, the indices 0..n_r-1; otherwise the k
 * indices of the largest scores, ties broken toward the lower index, -0.0 and
 * +0.0 equal.  Indices ascending, padded with -1.
 *   max_len  upper bound of every n_r (the host sizes grids with it);
 *            ld_scores >= max_len and ld_scores % 4 == 0; scores 16-byte aligned.
 * Supported: 1 <= k <= 40000 (a row's winners are staged in shared memory).
 *   row_stats  NULL, or the buffer dsa_indexer_scores filled for exactly
 *            these rows (same row_begin / n_rows, scores unchanged since).
 *   ws       device workspace of at least dsa_topk_workspace_size() bytes
 *            (may be NULL when that size is 0).
 * ------------------------------------------------------------------------ */
DSA_API size_t dsa_topk_workspace_size(int n_rows, int max_len, int k);
DSA_API dsa_status_t dsa_topk(const float *scores, int64_t ld_scores, int row_begin, int n_rows,
                      const int32_t *row_len, int max_len, int k, int32_t *idx,
                      const void *row_stats, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * Fused lightning indexer + causal top-k (prefill), one chunk of query rows:
 * the same Omega_t as dsa_indexer_scores followed by dsa_topk, without
 * writing the score matrix.
 *
 * [REVIEW] 核心公式 (indexer score and Omega_t); [REPORT] 2.3.1; [REPORT]
 * 5.1.2 (rows with t+1 <= k keep all of 0..t); [REPORT] 5.2.1 (deterministic
 * top-k; the score matrix is what bounds memory, which the report handles by
 * chunking -- here it is not materialised at all).
 * Steps, on `stream`: the indexer scores every 32nd key of each row; a
 * threshold per row is read off those samples (about 2k keys of a row lie at
 * or above it); the indexer then scores every causal key and keeps only the
 * (index, score) pairs at or above the threshold; the exact top-k of those
 * candidates is taken.  A row whose candidates cannot decide it (fewer than
 * k of them, or more than fit) is scored again in full and selected exactly,
 * so the result never depends on the sample: it is the top-k of the row's
 * fp32 scores, ties to the lower index, -0.0 == +0.0.
 *
 *   q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows: as for
 *            dsa_indexer_scores (q8, k8 16-byte aligned; positive scales).
 *   k        the top-k budget, >= 1.
 *   idx      [n_rows, k] int32: row r = query t = row_begin + r; ascending,
 *            -1 padded when t + 1 < k.
 *   ws       device workspace of dsa_indexer_topk_workspace_size(row_begin,
 *            n_rows, k, HI, dI) bytes, 256-byte aligned (sampled scores,
 *            thresholds, candidate lists, the repair list and its scratch
 *            rows).
 *   stats    optional (NULL to skip): device int64[2] that receives the
 *            number of rows of this call that were scored again in full and
 *            the number of candidates the indexer kept for the selection.
 * Supported: HI in {8, 16, 32, 64}, dI in {32, 64, 128} (the tensor-core
 * indexer's shapes), L * HI < 2^31; DSA_ERR_UNSUPPORTED_SHAPE otherwise
 * (use dsa_indexer_scores + dsa_topk there).
 * ------------------------------------------------------------------------ */
DSA_API size_t dsa_indexer_topk_workspace_size(int row_begin, int n_rows, int k, int HI, int dI);
DSA_API dsa_status_t dsa_indexer_topk(const uint8_t *q8, const float *q_scale, const float *w,
                              const uint8_t *k8, const float *k_scale,
                              int L, int HI, int dI, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream);
/* Packed (varlen) form of dsa_indexer_topk: several sequences packed along
 * the token axis, each its own causal prefill ([REPORT] 5.1.2: per-sample
 * causal regions in one launch).  Sequence b holds tokens
 * cu_seqlens[b] .. cu_seqlens[b+1]-1; query token t of sequence b scores and
 * selects only the keys cu_seqlens[b] .. t, and idx row r (t = row_begin +
 * r) holds positions within that sequence (0 = its first token), ascending,
 * -1 padded; a row with t - cu_seqlens[b] + 1 <= k keeps all of them.
 *   cu_seqlens  device int32 [nseq + 1], ascending, cu_seqlens[0] = 0,
 *               cu_seqlens[nseq] = L (empty sequences allowed); read on the
 *               device (a malformed array gives wrong rows, never reads
 *               outside the tokens 0..t).
 *   L           total packed tokens; every other argument as for
 *               dsa_indexer_topk, with the same workspace size query. */
DSA_API dsa_status_t dsa_indexer_topk_varlen(const uint8_t *q8, const float *q_scale, const float *w,
                              const uint8_t *k8, const float *k_scale, int L, int HI, int dI,
                              const int32_t *cu_seqlens, int nseq, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream);
/* The three stages of dsa_indexer_topk, same arguments, for callers that time
 * or schedule them separately; called in this order on one stream, with the
 * same workspace and arguments, they are dsa_indexer_topk:
 *   _threshold   sampled scores (every 32nd key) and one threshold per row;
 *   _candidates  every causal score, keeping the (index, score) pairs at or
 *                above the row's threshold (the tensor-core indexer);
 *   _select      the exact top-k of the candidates into idx, and the full
 *                re-scoring and selection of any row they cannot decide. */
DSA_API dsa_status_t dsa_indexer_topk_threshold(const uint8_t *q8, const float *q_scale, const float *w,
                              const uint8_t *k8, const float *k_scale,
                              int L, int HI, int dI, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream);
DSA_API dsa_status_t dsa_indexer_topk_candidates(const uint8_t *q8, const float *q_scale, const float *w,
                              const uint8_t *k8, const float *k_scale,
                              int L, int HI, int dI, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream);
DSA_API dsa_status_t dsa_indexer_topk_select(const uint8_t *q8, const float *q_scale, const float *w,
                              const uint8_t *k8, const float *k_scale,
                              int L, int HI, int dI, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream);

/* ------------------------------------------------------------------------
 * Indexer distillation losses (forward), one chunk of query rows.
 *
 * [REVIEW] 核心公式, dense warm-up loss and sparse adaptation loss;
 * [REPORT] 2.3.3 (the target of group g is its aggregated dense attention,
 * normalised; in the sparse stage it is truncated to the selected set S_t and
 * renormalised, and the indexer softmax runs over S_t):
 *     loss_rows[r] = sum_{g<G} KL( p[r,g,S] / sum_S p[r,g,S]  ||  Softmax(I[t,S]) )
 *     KL(a||b) = sum_s a_s ln(a_s / b_s),  0 ln 0 = 0,   t = row_begin + r.
 *   idx == NULL: S = [0, t] (dense warm-up); otherwise S = the entries of idx
 *   row r that lie in [0, t] (sparse adaptation; entries must be distinct,
 *   -1 padding and out-of-range entries are skipped).
 *
 *   scores     [n_rows, ld_scores] float: I[t, s] for s <= t (e.g. from
 *              dsa_indexer_scores); ld_scores >= row_begin + n_rows.
 *   p          [n_rows, G, ld_p] float, non-negative target weights for keys
 *              0..t (they are normalised over S here); ld_p >= row_begin + n_rows.
 *   idx        NULL, or [n_rows, k] int32 (e.g. from dsa_topk).
 *   loss_rows  [n_rows] double: the loss of each row; a group with no target
 *              mass on S contributes 0, a row whose S is empty gets 0.
 *   loss_total optional (NULL to skip): one double, the sum of loss_rows
 *              (fixed summation order: bitwise reproducible).
 * Sums are accumulated in double precision from the float inputs.
 * ------------------------------------------------------------------------ */
DSA_API dsa_status_t dsa_indexer_kl(const float *scores, int64_t ld_scores, int row_begin, int n_rows,
                            const float *p, int G, int64_t ld_p, const int32_t *idx, int k,
                            double *loss_rows, double *loss_total, void *stream);

/* ------------------------------------------------------------------------
 * Sparse GQA attention (prefill), one chunk of query rows.
 *
 * [REVIEW] 核心公式, u[t,g] = Attn(h[t,g], { c[s,g] | s in Omega_t });
 * [REPORT] 2.3.2: one index set Omega_t serves every KV group g; the group
 * outputs are concatenated.  Head h reads group g = h / (Hq / Hkv):
 *     O[t,h] = sum_{s in Omega_t} softmax_s( sm_scale * Q[t,h] . K[s,g] ) V[s,g]
 *     lse[t,h] = log sum_{s in Omega_t} exp( sm_scale * Q[t,h] . K[s,g] )
 * Only the first min(k, t+1) entries of an index row are visited ([REPORT]
 * 5.1.2); entries outside [0, t] are skipped.
 *
 *   Q    [n_rows, Hq, D] bf16 (row r is query t = row_begin + r)
 *   K, V [>= row_begin + n_rows, Hkv, D] bf16
 *   idx  [n_rows, k] int32 (from dsa_topk)
 *   O    [n_rows, Hq, D] bf16;  lse [n_rows, Hq] float, may be NULL.
 * Supported: D in {64, 128}; Hq % Hkv == 0 with Hq / Hkv <= 8;
 * n_rows * Hkv < 2^31 (one CTA per (row, group)).
 * A row with no valid index writes O = 0 and lse = -inf.
 * ------------------------------------------------------------------------ */
DSA_API dsa_status_t dsa_sparse_gqa_prefill(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                    const int32_t *idx, int row_begin, int n_rows,
                                    int Hq, int Hkv, int D, int k, float sm_scale,
                                    uint16_t *O, float *lse, void *stream);
/* Packed (varlen) form: sequence b holds tokens cu_seqlens[b] ..
 * cu_seqlens[b+1]-1 (cu_seqlens as for dsa_indexer_topk_varlen, device int32
 * [nseq + 1]); idx row r (query t = row_begin + r of sequence b) holds
 * positions within sequence b, and entry e names token cu_seqlens[b] + e;
 * entries outside [0, t - cu_seqlens[b]] are skipped.  Q, O rows and K, V
 * rows are packed tokens. */
DSA_API dsa_status_t dsa_sparse_gqa_prefill_varlen(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                    const int32_t *idx, const int32_t *cu_seqlens, int nseq,
                                    int row_begin, int n_rows, int Hq, int Hkv, int D, int k, float sm_scale,
                                    uint16_t *O, float *lse, void *stream);

/* ------------------------------------------------------------------------
 * Decode over a paged cache: one new query token per sequence.
 *
 * [REPORT] 5.3 (DSA decode); formulas as above with t = seq_lens[b] - 1: the
 * new token's K, V and indexer key are already in the cache.  Logical token s
 * of sequence b lives in page block_table[b * max_pages + s / 64], slot s % 64.
 *
 *   q             [B, Hq, D] bf16          q8 [B, HI, dI] e4m3
 *   q_scale       [B] float                w  [B, HI] float
 *   k8_cache      [num_pages, 64, dI] e4m3 k_scale_cache [num_pages, 64] float
 *   k_cache,
 *   v_cache       [num_pages, 64, Hkv, D] bf16
 *   block_table   [B, max_pages] int32 (entries past a sequence's end unused)
 *   seq_lens      [B] int32, 1 <= seq_lens[b] <= min(max_seq_len, 64 * max_pages)
 *   max_seq_len   host-side upper bound of seq_lens (sizes grids and workspace)
 *   out           [B, Hq, D] bf16
 *   idx_out       [B, k] int32 selected indices, may be NULL
 *   ws            >= dsa_decode_workspace_size(...) bytes
 * A token on a page id outside [0, num_pages) scores -inf and is skipped by
 * the attention.  q8, k8_cache and k_scale_cache start on 16-byte boundaries
 * (DSA_ERR_INVALID_ARG otherwise): they are copied in 16-byte pieces.
 * dsa_sparse_gqa_decode runs the three stages below on `stream`:
 * scores (dsa_decode_indexer_scores) -> top-k (dsa_topk with row_len =
 * seq_lens) -> attention (dsa_sparse_gqa_decode_attention).
 * ------------------------------------------------------------------------ */
DSA_API size_t dsa_decode_workspace_size(int B, int max_seq_len, int Hq, int Hkv, int D, int k);
DSA_API dsa_status_t dsa_sparse_gqa_decode(const uint16_t *q, const uint8_t *q8, const float *q_scale,
                                   const float *w,
                                   const uint8_t *k8_cache, const float *k_scale_cache,
                                   const uint16_t *k_cache, const uint16_t *v_cache,
                                   const int32_t *block_table, int max_pages, int num_pages,
                                   const int32_t *seq_lens, int max_seq_len,
                                   int B, int Hq, int Hkv, int D, int HI, int dI, int k,
                                   float sm_scale, void *ws, size_t ws_bytes,
                                   uint16_t *out, int32_t *idx_out, void *stream);

/* Decode stage 1: indexer scores of each sequence's query against its cached
 * keys.  scores [B, ld_scores] float, columns 0..seq_lens[b]-1 written;
 * ld_scores >= max_seq_len and ld_scores % 4 == 0.  Same formula and shape
 * support as dsa_indexer_scores. */
DSA_API dsa_status_t dsa_decode_indexer_scores(const uint8_t *q8, const float *q_scale, const float *w,
                                       const uint8_t *k8_cache, const float *k_scale_cache,
                                       const int32_t *block_table, int max_pages, int num_pages,
                                       const int32_t *seq_lens, int max_seq_len,
                                       int B, int HI, int dI,
                                       float *scores, int64_t ld_scores, void *stream);

/* Decode stage 3: attention of each sequence's query over the selected rows
 * idx [B, k] (entries outside [0, seq_lens[b]) skipped), read through the
 * block table.  lse [B, Hq] may be NULL.  ws >=
 * dsa_decode_attention_workspace_size(B, Hq, Hkv, D, k) bytes. */
DSA_API size_t dsa_decode_attention_workspace_size(int B, int Hq, int Hkv, int D, int k);
DSA_API dsa_status_t dsa_sparse_gqa_decode_attention(const uint16_t *q,
                                             const uint16_t *k_cache, const uint16_t *v_cache,
                                             const int32_t *block_table, int max_pages, int num_pages,
                                             const int32_t *seq_lens, const int32_t *idx,
                                             int B, int Hq, int Hkv, int D, int k, float sm_scale,
                                             void *ws, size_t ws_bytes,
                                             uint16_t *out, float *lse, void *stream);

/* ------------------------------------------------------------------------
 * Decode attention that allocates nothing.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory themselves: a plugin or serving hook that is
 * handed only its input and output buffers, or a latency-critical loop in
 * which cudaMalloc (which may synchronise the device, and may fail under
 * memory pressure) is not allowed.  It computes exactly what
 * dsa_sparse_gqa_decode_attention computes, with the same arguments minus the
 * workspace: the split-K partials live in a fixed array inside the library
 * (dsa_decode_attention_fixed_scratch_bytes() bytes, 8 MiB), which every GPU
 * that loads the library holds until the process exits.
 *  - Limit: B * Hkv * 8 * (D + 2) * 4 bytes must fit that array (B <= 504
 *    for Hkv = 4, D = 128); larger batches return DSA_ERR_WORKSPACE without
 *    launching.  Within the limit the split count may be lower than the
 *    workspace variant's, so results can differ from it by rounding only.
 *  - The first call on a device looks up the array's device address with
 *    that device current; make that first call before any stream capture.
 *    The address is kept for the life of the process: after a
 *    cudaDeviceReset of that device it is stale, so do not call this entry
 *    point on a device that has been reset.
 *  - Every call on a device shares the one array: calls whose executions
 *    overlap on the GPU (other streams, other host threads) race.  Nothing
 *    has to be cleared between calls; each call writes every partial it reads.
 *  - No cudaMalloc, cudaFree or allocating library routine is called.
 * ------------------------------------------------------------------------ */
DSA_API size_t dsa_decode_attention_fixed_scratch_bytes(void);
DSA_API dsa_status_t dsa_sparse_gqa_decode_attention_noalloc(const uint16_t *q,
                                             const uint16_t *k_cache, const uint16_t *v_cache,
                                             const int32_t *block_table, int max_pages, int num_pages,
                                             const int32_t *seq_lens, const int32_t *idx,
                                             int B, int Hq, int Hkv, int D, int k, float sm_scale,
                                             uint16_t *out, float *lse, void *stream);

/* ------------------------------------------------------------------------
 * Read-bandwidth probe (diagnostic, not part of the layer; the pages have no
 * counterpart).  Reads `bytes` bytes of `buf` `reps` times with 16-byte loads
 * cached in L2 only (the load form the attention's gathers use), spread over
 * every SM, on `stream`.  A caller times it with events: a buffer that fits
 * in L2 read many times gives the L2 read bandwidth, one pass over a buffer
 * much larger than L2 gives the HBM read bandwidth; both serve as roofline
 * denominators.
 *   buf   device pointer, 16-byte aligned; bytes a multiple of 16, > 0
 *   sink  device pointer to one uint32 the kernel may write (keeps the
 *         loads from being optimised away); its value is meaningless
 *   reps  >= 1
 * ------------------------------------------------------------------------ */
DSA_API dsa_status_t dsa_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
