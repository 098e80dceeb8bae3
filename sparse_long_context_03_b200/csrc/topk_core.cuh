// topk_core.cuh -- building blocks of the per-row top-k selection, shared by
// the selection over a materialised score row (topk.cu) and the selection
// over the fused indexer's candidate lists (topk_fused.cu).
//
// Scores map to order-preserving 32-bit keys (order_key in common.cuh);
// every step is a count (histograms, block scans), so results do not depend
// on scheduling.
#pragma once

#include "common.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kNB = 2048;          // linear buckets (pass 2) and radix bins
constexpr int kCap = 6144;         // candidates kept in shared memory
constexpr int kSmallCand = 256;    // up to this many candidates are ranked directly
constexpr int kVec = 16;           // consecutive entries per thread per chunk (4 x float4 in flight)
constexpr int kChunk = kThreads * kVec;

struct TopkSmem {
    uint32_t hist[kNB];
    uint32_t ckey[kCap];
    int32_t cidx[kCap];
    uint32_t red[2 * kWarps];
    uint32_t bcast[4];
    // followed by int32_t alist[k]
};

__host__ __device__ constexpr size_t smem_bytes(int k) { return sizeof(TopkSmem) + sizeof(int32_t) * (size_t)k; }

__device__ __forceinline__ int row_length(const int32_t *row_len, int r, int row_begin, int max_len) {
    if (row_len == nullptr) return row_begin + r + 1;
    const int n = __ldg(row_len + r);
    return n < 0 ? 0 : (n > max_len ? max_len : n);
}

// Load entries i0..i0+kVec-1 (fewer at the tail); absent entries get 0.
// A full group is four independent 16-byte loads issued back to back.
__device__ __forceinline__ int load_vals(const float *row, int i0, int n, float (&x)[kVec]) {
    if (i0 + kVec <= n) {
        float4 v[kVec / 4];
#pragma unroll
        for (int q = 0; q < kVec / 4; ++q) v[q] = __ldg(reinterpret_cast<const float4 *>(row + i0) + q);
#pragma unroll
        for (int q = 0; q < kVec / 4; ++q) {
            x[4 * q + 0] = v[q].x;
            x[4 * q + 1] = v[q].y;
            x[4 * q + 2] = v[q].z;
            x[4 * q + 3] = v[q].w;
        }
        return kVec;
    }
    int m = 0;
#pragma unroll
    for (int j = 0; j < kVec; ++j) {
        x[j] = (i0 + j < n) ? __ldg(row + i0 + j) : 0.f;
        m += (i0 + j < n);
    }
    return m;
}

// Bucket of a score in [vmin, vmax]: rounded subtraction and multiplication
// by a positive scale are monotone, and so is truncation, so bucket order is
// score order (-0.0 and +0.0 share a bucket).  The explicit _rn intrinsics
// keep the compiler from contracting the two steps differently in the two
// passes that must agree.
__device__ __forceinline__ uint32_t bucket_of(float x, float vmin, float scale) {
    const uint32_t b = __float2uint_rz(__fmul_rn(__fsub_rn(x, vmin), scale));
    return b < (uint32_t)kNB ? b : (uint32_t)(kNB - 1);
}

// Exclusive block scan of one packed value per thread (two 16-bit counters;
// a chunk has kChunk = 8192 entries, so neither counter overflows).
// Returns the exclusive prefix; *total gets the block total.  Two barriers.
__device__ __forceinline__ uint32_t block_scan_packed(uint32_t v, uint32_t *red, uint32_t *total) {
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) red[warp] = x;
    __syncthreads();
    uint32_t before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const uint32_t s = red[w];
        before += (w < warp) ? s : 0u;
        tot += s;
    }
    __syncthreads();
    *total = tot;
    return before + x - v;
}

// Bin b with above(b) < need <= above(b) + hist[b], above(b) = sum of bins > b;
// thread j owns bins 4j..4j+3.  Writes (b, need - above(b), above(b)) to bcast.
__device__ __forceinline__ void find_threshold_bin(const uint32_t *hist, uint32_t need, uint32_t *red,
                                                   uint32_t *bcast) {
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    uint32_t c[4], own = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        c[q] = hist[tid * 4 + q];
        own += c[q];
    }
    uint32_t v = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, v, o);
        if (lane + o < 32) v += y;
    }
    if (lane == 0) red[warp] = v;
    __syncthreads();
    uint32_t above = v - own;
    for (int w = warp + 1; w < kWarps; ++w) above += red[w];
#pragma unroll
    for (int q = 3; q >= 0; --q) {
        if (above < need && need <= above + c[q]) {
            bcast[0] = (uint32_t)(tid * 4 + q);
            bcast[1] = need - above;
            bcast[2] = above;
        }
        above += c[q];
    }
    __syncthreads();
}

// Radix select of the `need`-th largest key among ckey[0..cnt): returns T and
// how many entries equal to T are to be taken.
template <typename Smem>
__device__ __forceinline__ void select_in_candidates(Smem &sm, int cnt, uint32_t need, uint32_t &T,
                                                     uint32_t &quota) {
    uint32_t prefix = 0, pmask = 0;
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
        const uint32_t dmask = (p == 2 ? 1023u : 2047u);
        for (int i = threadIdx.x; i < kNB; i += kThreads) sm.hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < cnt; i += kThreads) {
            const uint32_t key = sm.ckey[i];
            if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & dmask], 1u);
        }
        __syncthreads();
        find_threshold_bin(sm.hist, need, sm.red, sm.bcast);
        prefix |= sm.bcast[0] << shift;
        pmask |= dmask << shift;
        need = sm.bcast[1];
        __syncthreads();
    }
    T = prefix;
    quota = need;
}

// Loads of a score row: read-only (non-coherent) path for rows written
// before the kernel started, L2 (coherent) for rows written by this kernel.
template <bool kWrittenHere>
__device__ __forceinline__ float row_load(const float *p) {
    if constexpr (kWrittenHere) return __ldcg(p);
    else return __ldg(p);
}

// Slow exact path over the whole row (used when the threshold bucket does
// not fit in shared memory): radix select then ordered compaction.
// kWrittenHere: the row was written earlier in the same kernel.
template <bool kWrittenHere = false>
__device__ void topk_row_radix(const float *row, int n, int k, int32_t *out, TopkSmem &sm) {
    const int tid = threadIdx.x, lane = lane_id();
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)k;
#pragma unroll 1
    for (int p = 0; p < 3; ++p) {
        const int shift = p == 0 ? 21 : (p == 1 ? 10 : 0);
        const uint32_t dmask = (p == 2 ? 1023u : 2047u);
        for (int i = tid; i < kNB; i += kThreads) sm.hist[i] = 0;
        __syncthreads();
        for (int base = (tid >> 5) * 32; base < n; base += kThreads) {
            const int i = base + lane;
            uint32_t bin = 0xFFFFFFFFu;
            if (i < n) {
                const uint32_t key = order_key(row_load<kWrittenHere>(row + i));
                if ((key & pmask) == prefix) bin = (key >> shift) & dmask;
            }
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
            if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&sm.hist[bin], __popc(peers));
        }
        __syncthreads();
        find_threshold_bin(sm.hist, need, sm.red, sm.bcast);
        prefix |= sm.bcast[0] << shift;
        pmask |= dmask << shift;
        need = sm.bcast[1];
        __syncthreads();
    }
    const uint32_t T = prefix, quota = need;
    uint32_t run_gt = 0, run_eq = 0;
    for (int base = 0; base < n; base += kThreads) {
        const int i = base + tid;
        const uint32_t key = i < n ? order_key(row_load<kWrittenHere>(row + i)) : 0u;
        const bool gt = i < n && key > T;
        const bool eq = i < n && key == T;
        uint32_t tot;
        const uint32_t ex = block_scan_packed((gt ? 1u : 0u) | (eq ? 0x10000u : 0u), sm.red, &tot);
        const uint32_t gt_before = run_gt + (ex & 0xFFFFu);
        const uint32_t eq_before = run_eq + (ex >> 16);
        if (gt || (eq && eq_before < quota)) out[gt_before + min(eq_before, quota)] = i;
        run_gt += tot & 0xFFFFu;
        run_eq += tot >> 16;
    }
}

}  // namespace
}  // namespace dsa
