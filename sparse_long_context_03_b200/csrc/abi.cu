// abi.cu -- the extern "C" entry points declared in include/dsa.h.
//
// Host code here only validates arguments, sizes workspaces and launches the
// kernels on the caller's stream.  It never allocates, frees or synchronises.
// Validation comes before any CUDA call, so an invalid call touches nothing.
#include <nvtx3/nvToolsExt.h>

#include <cstring>

#include "dsa.h"
#include "kernels.h"

namespace {

// One NVTX range per call, named after the entry point, so that a profiler
// attributes every launch to its stage (header-only NVTX: without a tool
// attached a range costs a check of a function pointer).
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
    Range(const Range &) = delete;
    Range &operator=(const Range &) = delete;
};

thread_local char g_last_error[256] = "";

dsa_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return DSA_OK;
    std::strncpy(g_last_error, cudaGetErrorString(e), sizeof(g_last_error) - 1);
    g_last_error[sizeof(g_last_error) - 1] = '\0';
    return DSA_ERR_CUDA;
}

inline cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Layout of the decode workspace: [scores B x ld][idx B x k][top-k]
// [row key ranges 2 x B][attention split-K partials].  The key ranges are
// preset (all-ones) at the start of each call.
struct DecodeWs {
    int64_t ld;
    size_t scores_off, idx_off, topk_off, range_off, attn_off, preset_bytes, total;
};

DecodeWs decode_ws_layout(int B, int max_seq_len, int Hq, int Hkv, int D, int k) {
    DecodeWs w{};
    w.ld = (int64_t)align_up((size_t)(max_seq_len > 0 ? max_seq_len : 1), 4);
    w.scores_off = 0;
    w.idx_off = align_up(w.scores_off + (size_t)B * w.ld * sizeof(float), 256);
    w.topk_off = align_up(w.idx_off + (size_t)B * k * sizeof(int32_t), 256);
    w.range_off = align_up(w.topk_off + dsa::topk_workspace_bytes(B, max_seq_len, k), 256);
    w.attn_off = align_up(w.range_off + (size_t)2 * B * sizeof(uint32_t), 256);
    w.preset_bytes = (size_t)2 * B * sizeof(uint32_t);
    w.total = align_up(w.attn_off + dsa::decode_attention_workspace_bytes(B, Hq, Hkv, D, k), 256);
    return w;
}

}  // namespace

extern "C" {

const char *dsa_status_string(dsa_status_t s) {
    switch (s) {
        case DSA_OK: return "DSA_OK";
        case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
        case DSA_ERR_UNSUPPORTED_SHAPE: return "DSA_ERR_UNSUPPORTED_SHAPE";
        case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
        case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
        case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    }
    return "DSA_ERR_UNKNOWN";
}

int dsa_version(void) { return DSA_VERSION; }

const char *dsa_last_error_string(void) { return g_last_error; }

dsa_status_t dsa_check_device_error(void) {
    unsigned int flag = 0;
    cudaError_t e = dsa::indexer_tc_take_error(&flag);
    if (e != cudaSuccess) return cuda_status(e);
    return flag ? DSA_ERR_TIMEOUT : DSA_OK;
}

dsa_status_t dsa_set_wait_limit_ns(unsigned long long ns) { return cuda_status(dsa::indexer_tc_set_wait_limit(ns)); }

size_t dsa_row_stats_bytes(int n_rows) { return n_rows > 0 ? (size_t)n_rows * 8 * sizeof(float) : 0; }

dsa_status_t dsa_indexer_scores(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                                const float *k_scale, int L, int HI, int dI, int row_begin, int n_rows,
                                float *scores, int64_t ld_scores, void *row_stats, void *stream) {
    const Range range(__func__);
    if (L < 1 || row_begin < 0 || n_rows < 0 || (int64_t)row_begin + n_rows > L) return DSA_ERR_INVALID_ARG;
    if (!dsa::indexer_shape_supported(HI, dI)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (n_rows == 0) return DSA_OK;
    if (!q8 || !q_scale || !w || !k8 || !k_scale || !scores) return DSA_ERR_INVALID_ARG;
    if (ld_scores < (int64_t)row_begin + n_rows || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q8) | reinterpret_cast<uintptr_t>(k8)) % 16 != 0) return DSA_ERR_INVALID_ARG;
    float *stats = static_cast<float *>(row_stats);
    // the tensor-core path addresses q8 rows (L * HI of them) with 32-bit TMA coordinates
    if (dsa::indexer_tc_supported(HI, dI) && (int64_t)L * HI < (1ll << 31))
        return cuda_status(dsa::launch_indexer_prefill_tc(q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows,
                                                          scores, ld_scores, stats, as_stream(stream)));
    cudaError_t e = dsa::launch_indexer_prefill_mma(q8, q_scale, w, k8, k_scale, HI, dI, row_begin, n_rows, scores,
                                                    ld_scores, as_stream(stream));
    if (e == cudaSuccess && stats != nullptr)
        e = dsa::launch_row_stats(scores, ld_scores, row_begin, n_rows, stats, as_stream(stream));
    return cuda_status(e);
}

size_t dsa_topk_workspace_size(int n_rows, int max_len, int k) {
    if (n_rows < 0 || max_len < 0 || k < 1) return 0;
    return dsa::topk_workspace_bytes(n_rows, max_len, k);
}

dsa_status_t dsa_topk(const float *scores, int64_t ld_scores, int row_begin, int n_rows, const int32_t *row_len,
                      int max_len, int k, int32_t *idx, const void *row_stats, void *ws, size_t ws_bytes,
                      void *stream) {
    const Range range(__func__);
    if (n_rows < 0 || row_begin < 0 || k < 1 || max_len < 0) return DSA_ERR_INVALID_ARG;
    if (row_len == nullptr && (int64_t)row_begin + n_rows > max_len) return DSA_ERR_INVALID_ARG;
    if (n_rows == 0) return DSA_OK;
    if (!scores || !idx) return DSA_ERR_INVALID_ARG;
    if (ld_scores < max_len || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(scores) % 16 != 0) return DSA_ERR_INVALID_ARG;
    if (!dsa::topk_k_supported(k)) return DSA_ERR_UNSUPPORTED_SHAPE;
    const size_t need = dsa::topk_workspace_bytes(n_rows, max_len, k);
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return DSA_ERR_WORKSPACE;
    return cuda_status(dsa::launch_topk(scores, ld_scores, row_begin, n_rows, row_len, max_len, k, idx,
                                        static_cast<const float *>(row_stats), ws, ws_bytes, as_stream(stream)));
}

size_t dsa_indexer_topk_workspace_size(int row_begin, int n_rows, int k, int HI, int dI) {
    if (row_begin < 0 || n_rows < 0 || k < 1 || !dsa::fused_topk_supported(k, HI, dI)) return 0;
    return dsa::fused_topk_layout(row_begin, n_rows, k, HI, dI).total;
}

}  // extern "C"

namespace {

dsa_status_t indexer_topk_checked(int stage, const uint8_t *q8, const float *q_scale, const float *w,
                                  const uint8_t *k8, const float *k_scale, int L, int HI, int dI, int row_begin,
                                  int n_rows, int k, int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats,
                                  void *stream, const int32_t *cu = nullptr, int nseq = 0) {
    if (cu != nullptr && nseq < 1) return DSA_ERR_INVALID_ARG;
    if (L < 1 || row_begin < 0 || n_rows < 0 || k < 1 || (int64_t)row_begin + n_rows > L) return DSA_ERR_INVALID_ARG;
    if (!dsa::fused_topk_supported(k, HI, dI) || (int64_t)L * HI >= (1ll << 31)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (n_rows == 0) return DSA_OK;
    if (!q8 || !q_scale || !w || !k8 || !k_scale || !idx) return DSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q8) | reinterpret_cast<uintptr_t>(k8)) % 16 != 0) return DSA_ERR_INVALID_ARG;
    const size_t need = dsa::fused_topk_layout(row_begin, n_rows, k, HI, dI).total;
    if (ws == nullptr || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return DSA_ERR_WORKSPACE;
    for (int st = stage == 0 ? 1 : stage; st <= (stage == 0 ? 3 : stage); ++st) {
        const cudaError_t e = dsa::launch_indexer_topk_stage(st, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin,
                                                             n_rows, k, idx, ws, stats, cu, nseq, as_stream(stream));
        if (e != cudaSuccess) return cuda_status(e);
    }
    return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_indexer_topk(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                              const float *k_scale, int L, int HI, int dI, int row_begin, int n_rows, int k,
                              int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream) {
    const Range range(__func__);
    return indexer_topk_checked(0, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows, k, idx, ws, ws_bytes,
                                stats, stream);
}

dsa_status_t dsa_indexer_topk_varlen(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                                     const float *k_scale, int L, int HI, int dI, const int32_t *cu_seqlens, int nseq,
                                     int row_begin, int n_rows, int k, int32_t *idx, void *ws, size_t ws_bytes,
                                     int64_t *stats, void *stream) {
    const Range range(__func__);
    if (cu_seqlens == nullptr) return DSA_ERR_INVALID_ARG;
    return indexer_topk_checked(0, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows, k, idx, ws, ws_bytes,
                                stats, stream, cu_seqlens, nseq);
}

dsa_status_t dsa_indexer_topk_threshold(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                                        const float *k_scale, int L, int HI, int dI, int row_begin, int n_rows,
                                        int k, int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats,
                                        void *stream) {
    const Range range(__func__);
    return indexer_topk_checked(1, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows, k, idx, ws, ws_bytes,
                                stats, stream);
}

dsa_status_t dsa_indexer_topk_candidates(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                                         const float *k_scale, int L, int HI, int dI, int row_begin, int n_rows,
                                         int k, int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats,
                                         void *stream) {
    const Range range(__func__);
    return indexer_topk_checked(2, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows, k, idx, ws, ws_bytes,
                                stats, stream);
}

dsa_status_t dsa_indexer_topk_select(const uint8_t *q8, const float *q_scale, const float *w, const uint8_t *k8,
                                     const float *k_scale, int L, int HI, int dI, int row_begin, int n_rows, int k,
                                     int32_t *idx, void *ws, size_t ws_bytes, int64_t *stats, void *stream) {
    const Range range(__func__);
    return indexer_topk_checked(3, q8, q_scale, w, k8, k_scale, L, HI, dI, row_begin, n_rows, k, idx, ws, ws_bytes,
                                stats, stream);
}

dsa_status_t dsa_indexer_kl(const float *scores, int64_t ld_scores, int row_begin, int n_rows, const float *p,
                            int G, int64_t ld_p, const int32_t *idx, int k, double *loss_rows, double *loss_total,
                            void *stream) {
    const Range range(__func__);
    if (row_begin < 0 || n_rows < 0 || G < 1 || (idx != nullptr && k < 1)) return DSA_ERR_INVALID_ARG;
    if (n_rows == 0 && loss_total == nullptr) return DSA_OK;
    if ((n_rows > 0 && (!scores || !p || !loss_rows)) || (n_rows == 0 && !loss_rows)) return DSA_ERR_INVALID_ARG;
    if (ld_scores < (int64_t)row_begin + n_rows || ld_p < (int64_t)row_begin + n_rows) return DSA_ERR_INVALID_ARG;
    return cuda_status(dsa::launch_indexer_kl(scores, ld_scores, row_begin, n_rows, p, G, ld_p, idx,
                                              idx ? k : 0, loss_rows, loss_total, as_stream(stream)));
}

dsa_status_t dsa_sparse_gqa_prefill(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const int32_t *idx,
                                    int row_begin, int n_rows, int Hq, int Hkv, int D, int k, float sm_scale,
                                    uint16_t *O, float *lse, void *stream) {
    const Range range(__func__);
    if (row_begin < 0 || n_rows < 0 || k < 1 || Hq < 1 || Hkv < 1) return DSA_ERR_INVALID_ARG;
    if (!dsa::attention_shape_supported(Hq, Hkv, D)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)n_rows * Hkv >= (1ll << 31)) return DSA_ERR_UNSUPPORTED_SHAPE;  // one CTA per (row, group)
    if (n_rows == 0) return DSA_OK;
    if (!Q || !K || !V || !idx || !O) return DSA_ERR_INVALID_ARG;
    return cuda_status(dsa::launch_sparse_prefill(Q, K, V, idx, row_begin, n_rows, Hq, Hkv, D, k, sm_scale, O, lse,
                                                  as_stream(stream)));
}

dsa_status_t dsa_sparse_gqa_prefill_varlen(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                           const int32_t *idx, const int32_t *cu_seqlens, int nseq, int row_begin,
                                           int n_rows, int Hq, int Hkv, int D, int k, float sm_scale, uint16_t *O,
                                           float *lse, void *stream) {
    const Range range(__func__);
    if (cu_seqlens == nullptr || nseq < 1) return DSA_ERR_INVALID_ARG;
    if (row_begin < 0 || n_rows < 0 || k < 1 || Hq < 1 || Hkv < 1) return DSA_ERR_INVALID_ARG;
    if (!dsa::attention_shape_supported(Hq, Hkv, D)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if ((int64_t)n_rows * Hkv >= (1ll << 31)) return DSA_ERR_UNSUPPORTED_SHAPE;  // one CTA per (row, group)
    if (n_rows == 0) return DSA_OK;
    if (!Q || !K || !V || !idx || !O) return DSA_ERR_INVALID_ARG;
    return cuda_status(dsa::launch_sparse_prefill(Q, K, V, idx, row_begin, n_rows, Hq, Hkv, D, k, sm_scale, O, lse,
                                                  as_stream(stream), cu_seqlens, nseq));
}

// The decode indexer copies cache pages and query rows in 16-byte pieces.
static bool paged_keys_aligned(const uint8_t *q8, const uint8_t *k8_cache, const float *k_scale_cache) {
    return (reinterpret_cast<uintptr_t>(q8) | reinterpret_cast<uintptr_t>(k8_cache) |
            reinterpret_cast<uintptr_t>(k_scale_cache)) % 16 == 0;
}

static dsa_status_t check_decode_common(const int32_t *block_table, int max_pages, int num_pages,
                                        const int32_t *seq_lens, int max_seq_len, int B) {
    if (B < 0 || max_pages < 1 || num_pages < 1 || max_seq_len < 0) return DSA_ERR_INVALID_ARG;
    if ((int64_t)max_seq_len > (int64_t)max_pages * DSA_PAGE_SIZE) return DSA_ERR_INVALID_ARG;
    if (B > 0 && (!block_table || !seq_lens)) return DSA_ERR_INVALID_ARG;
    return DSA_OK;
}

dsa_status_t dsa_decode_indexer_scores(const uint8_t *q8, const float *q_scale, const float *w,
                                       const uint8_t *k8_cache, const float *k_scale_cache,
                                       const int32_t *block_table, int max_pages, int num_pages,
                                       const int32_t *seq_lens, int max_seq_len, int B, int HI, int dI,
                                       float *scores, int64_t ld_scores, void *stream) {
    const Range range(__func__);
    dsa_status_t st = check_decode_common(block_table, max_pages, num_pages, seq_lens, max_seq_len, B);
    if (st != DSA_OK) return st;
    if (!dsa::indexer_shape_supported(HI, dI)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (B == 0 || max_seq_len == 0) return DSA_OK;
    if (!q8 || !q_scale || !w || !k8_cache || !k_scale_cache || !scores) return DSA_ERR_INVALID_ARG;
    if (!paged_keys_aligned(q8, k8_cache, k_scale_cache)) return DSA_ERR_INVALID_ARG;
    if (ld_scores < max_seq_len || ld_scores % 4 != 0) return DSA_ERR_INVALID_ARG;
    return cuda_status(dsa::launch_indexer_decode(q8, q_scale, w, k8_cache, k_scale_cache, block_table, max_pages,
                                                  num_pages, seq_lens, max_seq_len, B, HI, dI, scores, ld_scores,
                                                  as_stream(stream)));
}

size_t dsa_decode_attention_workspace_size(int B, int Hq, int Hkv, int D, int k) {
    if (B < 0 || Hkv < 1 || k < 1 || D < 1) return 0;
    return dsa::decode_attention_workspace_bytes(B, Hq, Hkv, D, k);
}

dsa_status_t dsa_sparse_gqa_decode_attention(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                             const int32_t *block_table, int max_pages, int num_pages,
                                             const int32_t *seq_lens, const int32_t *idx, int B, int Hq, int Hkv,
                                             int D, int k, float sm_scale, void *ws, size_t ws_bytes,
                                             uint16_t *out, float *lse, void *stream) {
    const Range range(__func__);
    if (B < 0 || k < 1 || Hq < 1 || Hkv < 1 || max_pages < 1 || num_pages < 1) return DSA_ERR_INVALID_ARG;
    if (!dsa::attention_shape_supported(Hq, Hkv, D)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return DSA_OK;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (ws == nullptr || ws_bytes < dsa::decode_attention_workspace_bytes(B, Hq, Hkv, D, k)) return DSA_ERR_WORKSPACE;
    return cuda_status(dsa::launch_sparse_decode(q, k_cache, v_cache, block_table, max_pages, num_pages, seq_lens,
                                                 idx, B, Hq, Hkv, D, k, sm_scale, ws, ws_bytes, out, lse,
                                                 as_stream(stream)));
}

size_t dsa_decode_attention_fixed_scratch_bytes(void) { return dsa::fixed_scratch_bytes(); }

dsa_status_t dsa_sparse_gqa_decode_attention_noalloc(const uint16_t *q, const uint16_t *k_cache,
                                                     const uint16_t *v_cache, const int32_t *block_table,
                                                     int max_pages, int num_pages, const int32_t *seq_lens,
                                                     const int32_t *idx, int B, int Hq, int Hkv, int D, int k,
                                                     float sm_scale, uint16_t *out, float *lse, void *stream) {
    const Range range(__func__);
    if (B < 0 || k < 1 || Hq < 1 || Hkv < 1 || max_pages < 1 || num_pages < 1) return DSA_ERR_INVALID_ARG;
    if (!dsa::attention_shape_supported(Hq, Hkv, D)) return DSA_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return DSA_OK;
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !idx || !out) return DSA_ERR_INVALID_ARG;
    if (dsa::fixed_scratch_max_split(B, Hkv, D) < 1) {
        std::strncpy(g_last_error,
                     "batch too large for the fixed decode scratch: B * Hkv * 8 * (D + 2) * 4 bytes must not "
                     "exceed dsa_decode_attention_fixed_scratch_bytes()",
                     sizeof(g_last_error) - 1);
        g_last_error[sizeof(g_last_error) - 1] = '\0';
        return DSA_ERR_WORKSPACE;
    }
    return cuda_status(dsa::launch_sparse_decode_fixed_scratch(q, k_cache, v_cache, block_table, max_pages,
                                                               num_pages, seq_lens, idx, B, Hq, Hkv, D, k, sm_scale,
                                                               out, lse, as_stream(stream)));
}

size_t dsa_decode_workspace_size(int B, int max_seq_len, int Hq, int Hkv, int D, int k) {
    if (B < 0 || max_seq_len < 0 || Hkv < 1 || k < 1 || D < 1) return 0;
    return decode_ws_layout(B, max_seq_len, Hq, Hkv, D, k).total;
}

dsa_status_t dsa_sparse_gqa_decode(const uint16_t *q, const uint8_t *q8, const float *q_scale, const float *w,
                                   const uint8_t *k8_cache, const float *k_scale_cache, const uint16_t *k_cache,
                                   const uint16_t *v_cache, const int32_t *block_table, int max_pages,
                                   int num_pages, const int32_t *seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                   int D, int HI, int dI, int k, float sm_scale, void *ws, size_t ws_bytes,
                                   uint16_t *out, int32_t *idx_out, void *stream) {
    const Range range(__func__);
    dsa_status_t st = check_decode_common(block_table, max_pages, num_pages, seq_lens, max_seq_len, B);
    if (st != DSA_OK) return st;
    if (k < 1 || Hq < 1 || Hkv < 1) return DSA_ERR_INVALID_ARG;
    if (!dsa::indexer_shape_supported(HI, dI) || !dsa::attention_shape_supported(Hq, Hkv, D))
        return DSA_ERR_UNSUPPORTED_SHAPE;
    if (B == 0) return DSA_OK;
    if (!q || !q8 || !q_scale || !w || !k8_cache || !k_scale_cache || !k_cache || !v_cache || !out)
        return DSA_ERR_INVALID_ARG;
    if (!paged_keys_aligned(q8, k8_cache, k_scale_cache)) return DSA_ERR_INVALID_ARG;
    const DecodeWs L = decode_ws_layout(B, max_seq_len, Hq, Hkv, D, k);
    if (ws == nullptr || ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    char *base = static_cast<char *>(ws);
    float *scores = reinterpret_cast<float *>(base + L.scores_off);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(base + L.idx_off);
    cudaStream_t s = as_stream(stream);
    uint32_t *keyrange = reinterpret_cast<uint32_t *>(base + L.range_off);
    cudaError_t e = cudaMemsetAsync(keyrange, 0xFF, L.preset_bytes, s);  // row key ranges
    if (e != cudaSuccess) return cuda_status(e);
    bool have_range = false;
    e = dsa::launch_indexer_decode(q8, q_scale, w, k8_cache, k_scale_cache, block_table, max_pages, num_pages,
                                   seq_lens, max_seq_len, B, HI, dI, scores, L.ld, s, keyrange, &have_range);
    if (e != cudaSuccess) return cuda_status(e);
    e = dsa::launch_topk(scores, L.ld, 0, B, seq_lens, max_seq_len, k, idx, nullptr, base + L.topk_off,
                         dsa::topk_workspace_bytes(B, max_seq_len, k), s, have_range ? keyrange : nullptr);
    if (e != cudaSuccess) return cuda_status(e);
    e = dsa::launch_sparse_decode(q, k_cache, v_cache, block_table, max_pages, num_pages, seq_lens, idx, B, Hq, Hkv,
                                  D, k, sm_scale, base + L.attn_off, L.total - L.attn_off, out, nullptr, s);
    return cuda_status(e);
}

dsa_status_t dsa_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink, void *stream) {
    const Range range(__func__);
    if (!buf || !sink || bytes == 0 || bytes % 16 != 0 || reps < 1) return DSA_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(buf) % 16 != 0) return DSA_ERR_INVALID_ARG;
    return cuda_status(dsa::launch_read_probe(buf, bytes, reps, sink, as_stream(stream)));
}

}  // extern "C"
