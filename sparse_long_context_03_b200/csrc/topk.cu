// topk.cu -- deterministic per-row top-k by radix select.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式:
//     Omega_t = { s | I[t,s] in Top-k(I[t,:]) }
// report translation section 5.1.2 (a row with t+1 <= k keeps all of 0..t)
// and section 5.2.1 (the selection must be deterministic).
//
// Algorithm (no sort).  Scores map to order-preserving 32-bit keys (-0.0 and
// +0.0 equal).  Three histogram passes over 11, 11 and 10 key bits find the
// exact key T of the k-th largest score and how many entries equal to T the
// set still needs ("quota").  A final pass walks the row in index order and
// keeps every entry > T plus the first `quota` entries == T, writing each
// kept index at its rank among the kept ones: the output is ascending and
// ties go to the lower index.  Every step is a count, so the result does not
// depend on scheduling.
//
// One CTA owns one row.  The first pass streams the row from HBM; later passes
// re-read it, normally from L2 (a 128K-token row is 512 KB).  Histogram
// increments are aggregated per warp with match.any so that the heavily
// populated bins of the first pass (scores share sign and exponent) do not
// serialise on one shared-memory address.
#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins = 2048;

// Radix passes over the 32-bit key: bits 31..21, 20..10, 9..0.
__device__ __forceinline__ int pass_shift(int p) { return p == 0 ? 21 : (p == 1 ? 10 : 0); }
__device__ __forceinline__ int pass_bits(int p) { return p == 2 ? 10 : 11; }

__device__ __forceinline__ int row_length(const int32_t *row_len, int r, int row_begin, int max_len) {
    if (row_len == nullptr) return row_begin + r + 1;
    const int n = __ldg(row_len + r);
    return n < 0 ? 0 : (n > max_len ? max_len : n);
}

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(const float *__restrict__ scores, int64_t ld,
                                                                int row_begin, const int32_t *__restrict__ row_len,
                                                                int max_len, int k, int32_t *__restrict__ idx) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_sum[kWarps];
    __shared__ uint32_t sel_bin, sel_remaining;

    const int r = blockIdx.x;
    const int n = row_length(row_len, r, row_begin, max_len);
    const float *row = scores + (size_t)r * ld;
    int32_t *out = idx + (size_t)r * k;
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;

    if (n <= k) {  // short row: everything visible is selected
        for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
        return;
    }

    uint32_t prefix = 0, pmask = 0;
    uint32_t remaining = (uint32_t)k;
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = pass_shift(p);
        const uint32_t dmask = (1u << pass_bits(p)) - 1u;
        for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (int base = warp * 32; base < n; base += kTopkThreads) {
            const int i = base + lane;
            uint32_t bin = 0xFFFFFFFFu;
            if (i < n) {
                const uint32_t key = order_key(row[i]);
                if ((key & pmask) == prefix) bin = (key >> shift) & dmask;
            }
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
            if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
        __syncthreads();

        // Bin b holds the k-th largest iff above(b) < remaining <= above(b) + hist[b],
        // above(b) = sum of bins > b.  Thread j owns bins 4j..4j+3; a block
        // suffix sum over threads gives each thread the count above its bins.
        uint32_t c[4], own = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            c[q] = hist[tid * 4 + q];
            own += c[q];
        }
        // inclusive scan from the top: thread order reversed
        uint32_t v = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, v, o);
            if (lane + o < 32) v += y;
        }
        if (lane == 0) warp_sum[warp] = v;  // total of this warp
        __syncthreads();
        uint32_t above = v - own;  // bins owned by higher lanes of this warp
        for (int w2 = warp + 1; w2 < kWarps; ++w2) above += warp_sum[w2];
#pragma unroll
        for (int q = 3; q >= 0; --q) {
            if (above < remaining && remaining <= above + c[q]) {
                sel_bin = (uint32_t)(tid * 4 + q);
                sel_remaining = remaining - above;
            }
            above += c[q];
        }
        __syncthreads();
        prefix |= sel_bin << shift;
        pmask |= dmask << shift;
        remaining = sel_remaining;
        __syncthreads();
    }

    // Ordered compaction: keep key > T, and key == T while the quota lasts.
    const uint32_t T = prefix;
    const uint32_t quota = remaining;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t run_gt = 0, run_eq = 0;
    for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + tid;
        uint32_t key = 0;
        if (i < n) key = order_key(row[i]);
        const bool gt = i < n && key > T;
        const bool eq = i < n && key == T;
        const uint32_t bg = __ballot_sync(0xFFFFFFFFu, gt), be = __ballot_sync(0xFFFFFFFFu, eq);
        if (lane == 0) warp_sum[warp] = __popc(bg) | (__popc(be) << 16);
        __syncthreads();
        uint32_t before = 0, total = 0;
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2) {
            const uint32_t x = warp_sum[w2];
            before += (w2 < warp) ? x : 0u;
            total += x;
        }
        const uint32_t gt_before = run_gt + (before & 0xFFFFu) + __popc(bg & lt);
        const uint32_t eq_before = run_eq + (before >> 16) + __popc(be & lt);
        if (gt || (eq && eq_before < quota)) out[gt_before + min(eq_before, quota)] = i;
        run_gt += total & 0xFFFFu;
        run_eq += total >> 16;
        __syncthreads();
    }
}

}  // namespace

size_t topk_workspace_bytes(int, int, int) { return 0; }

cudaError_t launch_topk(const float *scores, int64_t ld, int row_begin, int n_rows, const int32_t *row_len,
                        int max_len, int k, int32_t *idx, void *, size_t, cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    topk_rows_kernel<<<n_rows, kTopkThreads, 0, stream>>>(scores, ld, row_begin, row_len, max_len, k, idx);
    return cudaGetLastError();
}

}  // namespace dsa
