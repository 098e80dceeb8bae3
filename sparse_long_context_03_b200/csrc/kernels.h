// kernels.h -- internal launchers behind the C ABI (not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace dsa {

// indexer_mma.cu
bool indexer_shape_supported(int HI, int dI);
cudaError_t launch_indexer_prefill_mma(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                       const float *sk, int HI, int dI, int row_begin, int n_rows, float *scores,
                                       int64_t ld, cudaStream_t stream);
cudaError_t launch_row_stats(const float *scores, int64_t ld, int row_begin, int n_rows, float *row_stats,
                             cudaStream_t stream);
// keyrange (optional, [2, B] uint32, every word preset to all-ones): the
// tensor-core path records each row's (min order key, complemented max
// order key) there and sets *range_written.
cudaError_t launch_indexer_decode(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8c,
                                  const float *skc, const int32_t *block_table, int max_pages, int num_pages,
                                  const int32_t *seq_lens, int max_seq_len, int B, int HI, int dI, float *scores,
                                  int64_t ld, cudaStream_t stream, uint32_t *keyrange = nullptr,
                                  bool *range_written = nullptr);

// indexer_tc.cu
bool indexer_tc_supported(int HI, int dI);
cudaError_t launch_indexer_prefill_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                      const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                      float *scores, int64_t ld, float *row_stats, cudaStream_t stream);
cudaError_t indexer_tc_take_error(unsigned int *flag);
// bound of the prefill indexer's pipeline waits on the current device (0: the default)
cudaError_t indexer_tc_set_wait_limit(unsigned long long ns);
// the same kernel scoring every indexer_sample_stride()-th key only:
// sample_scores [n_rows, ld], column j = key j * stride (causal: j * stride <= t);
// with cu (packed sequences, cu [nseq + 1]) the keys of the query's own
// sequence only, column j = the j-th sampled key at or after its start
int indexer_sample_stride();
cudaError_t launch_indexer_sample_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                     const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                     float *sample_scores, int64_t ld, const int32_t *cu, int nseq,
                                     cudaStream_t stream);
// the same kernel keeping only scores >= tau[row]: (index, score) pairs in
// cand [n_rows, 4, seg_cap], counts (uncapped) in cand_count [n_rows, 4]
cudaError_t launch_indexer_cand_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                   const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                   const float *tau, int2 *cand, int *cand_count, int seg_cap, const int32_t *cu,
                                   int nseq, cudaStream_t stream);
bool indexer_decode_tc_supported(int HI, int dI, int B, int max_seq_len);
cudaError_t launch_indexer_decode_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8c,
                                     const float *skc, const int32_t *block_table, int max_pages, int num_pages,
                                     const int32_t *seq_lens, int max_seq_len, int B, int HI, int dI, float *scores,
                                     int64_t ld, uint32_t *keyrange, cudaStream_t stream);

// topk.cu
size_t topk_workspace_bytes(int n_rows, int max_len, int k);
bool topk_k_supported(int k);
// row_keyrange (optional, [2, n_rows] as written by the decode indexer):
// each row's score range, used by the few-long-rows path in place of its
// range pass
cudaError_t launch_topk(const float *scores, int64_t ld, int row_begin, int n_rows, const int32_t *row_len,
                        int max_len, int k, int32_t *idx, const float *row_stats, void *ws, size_t ws_bytes,
                        cudaStream_t stream, const uint32_t *row_keyrange = nullptr);

// topk_fused.cu: the fused indexer + top-k (sampled threshold, candidate
// indexer, exact selection of the candidates, repair of undecided rows)
struct FusedTopkLayout {
    int keep_all;      // rows with at most this many visible keys keep every key as a candidate
    int seg_cap;       // candidates per row segment (four segments per row)
    int64_t lds;       // row stride of the sampled scores
    int repair_ctas;   // CTAs of the repair kernel (one scratch row each)
    int64_t scratch_ld;
    size_t sample_off, tau_off, cand_off, count_off, repair_off, total_off, scratch_off, total;
    size_t select_smem, repair_smem;
};
FusedTopkLayout fused_topk_layout(int row_begin, int n_rows, int k, int HI, int dI);
bool fused_topk_supported(int k, int HI, int dI);
// stage 1: sampled scores and per-row thresholds; 2: candidate indexer;
// 3: exact selection of the candidates and repair of undecided rows
cudaError_t launch_indexer_topk_stage(int stage, const uint8_t *q8, const float *sq, const float *w,
                                      const uint8_t *k8, const float *sk, int L, int HI, int dI, int row_begin,
                                      int n_rows, int k, int32_t *idx, void *ws, int64_t *stats,
                                      const int32_t *cu, int nseq, cudaStream_t stream);

// indexer_kl.cu: the indexer's distillation losses (forward)
cudaError_t launch_indexer_kl(const float *scores, int64_t ld, int row_begin, int n_rows, const float *p, int G,
                              int64_t ld_p, const int32_t *idx, int k, double *loss_rows, double *loss_total,
                              cudaStream_t stream);

// attention.cu
bool attention_shape_supported(int Hq, int Hkv, int D);
// cu [nseq + 1] (optional): packed sequences; index rows hold positions
// within each query's own sequence
cudaError_t launch_sparse_prefill(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const int32_t *idx,
                                  int row_begin, int n_rows, int Hq, int Hkv, int D, int k, float sm_scale,
                                  uint16_t *O, float *lse, cudaStream_t stream, const int32_t *cu = nullptr,
                                  int nseq = 0);
size_t decode_attention_workspace_bytes(int B, int Hq, int Hkv, int D, int k);
cudaError_t launch_sparse_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                 const int32_t *block_table, int max_pages, int num_pages, const int32_t *seq_lens,
                                 const int32_t *idx, int B, int Hq, int Hkv, int D, int k, float sm_scale,
                                 void *ws, size_t ws_bytes, uint16_t *out, float *lse, cudaStream_t stream);

// attention.cu: decode attention with its split-K partials in a fixed device
// array of the library (for callers that cannot allocate)
size_t fixed_scratch_bytes();
int fixed_scratch_max_split(int B, int Hkv, int D);
cudaError_t launch_sparse_decode_fixed_scratch(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                               const int32_t *block_table, int max_pages, int num_pages,
                                               const int32_t *seq_lens, const int32_t *idx, int B, int Hq, int Hkv,
                                               int D, int k, float sm_scale, uint16_t *out, float *lse,
                                               cudaStream_t stream);

// probe.cu: streaming 16-byte reads of a buffer, `reps` passes (bandwidth
// measurement only)
cudaError_t launch_read_probe(const void *buf, size_t bytes, int reps, uint32_t *sink, cudaStream_t stream);

}  // namespace dsa
