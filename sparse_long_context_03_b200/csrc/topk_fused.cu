// topk_fused.cu -- the top-k of the fused lightning indexer + top-k: the
// score matrix is never written; the indexer keeps only each row's likely
// winners, and this file turns them into Omega_t.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式:
//     Omega_t = { s | I[t,s] in Top-k(I[t,:]) }
// report translation section 5.1.2 (a row with t+1 <= k keeps all of 0..t)
// and section 5.2.1 (deterministic top-k; the chunked indexer is there to
// bound the memory a materialised score matrix takes).
//
// Per chunk of query rows, on one stream:
//   1. the indexer in its sampled mode scores every 32nd key of each row
//      (1/32 of the work);
//   2. sample_threshold_kernel: tau_t = (just below) the r-th largest sampled
//      score of row t, where r is the expected number of sampled keys among
//      the row's k winners plus six standard deviations plus eight -- so
//      that, with overwhelming probability, at least k scores of the row are
//      >= tau_t and at most a few thousand are.  Rows with at most keep_all
//      visible keys get tau = -inf (every key is a candidate);
//   3. the indexer in its candidate mode computes every causal score and
//      keeps (index, score) of those >= tau_t, in four segments per row (one
//      per TMEM lane quarter, each in ascending index order);
//   4. cand_select_kernel: the exact top-k of the candidates (larger score
//      first, lower index on ties; -0.0 == +0.0), written in ascending index
//      order.  The selection is exact whenever the candidates hold at least
//      k entries and no segment overflowed, because then the row's k
//      winners are all >= tau_t and all among the candidates.  Otherwise
//      (the sample was unlucky, or massive exact ties around tau_t) the row
//      is put on a repair list;
//   5. repair_rows_kernel: each listed row is scored again in full (fp32
//      on the CUDA cores) into scratch and selected by the exact whole-row
//      radix path.  With no listed rows it exits at once.
// Only step 2's threshold is sampled; the counts that decide each row are
// exact, so the result does not depend on the sample.
//
// Packed sequences (cu [nseq + 1], optional): row t sees only the keys
// [start(t), t] of its own sequence, and every index is a position within
// that sequence.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "topk_core.cuh"

namespace dsa {

namespace {

constexpr int kSegs = 4;              // candidate segments per row (TMEM lane quarters)
constexpr int kStage = 8192;          // sampled scores staged in shared memory
constexpr int kMaxTies = 512;         // entries equal to the k-th ranked pairwise
constexpr int kRepairThreads = kThreads;

// ---------------------------------------------------------------------------
// 2. per-row threshold from the sampled scores
// ---------------------------------------------------------------------------

struct ThreshSmem {
    uint32_t hist[kNB];
    uint32_t ckey[kStage];
    uint32_t red[2 * kWarps];
    uint32_t bcast[4];
};

__global__ void __launch_bounds__(kThreads) sample_threshold_kernel(const float *__restrict__ sample, int64_t lds,
                                                                   int row_begin, int n_rows, int k, int keep_all,
                                                                   int stride, float *__restrict__ tau,
                                                                   int *__restrict__ repair,
                                                                   unsigned long long *__restrict__ cand_total,
                                                                   const int32_t *__restrict__ cu, int nseq) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    ThreshSmem &sm = *reinterpret_cast<ThreshSmem *>(smem_raw);
    const int r = blockIdx.x, tid = threadIdx.x;
    if (r == 0 && tid == 0) {  // the select step appends to both after this launch
        repair[0] = 0;
        *cand_total = 0ull;
    }
    const int t = row_begin + r;
    const int start = seq_start(cu, nseq, t);
    const int n = t - start + 1;
    if (n <= keep_all) {
        if (tid == 0) tau[r] = -INFINITY;
        return;
    }
    const int m = t / stride - (start + stride - 1) / stride + 1;  // sampled keys visible to row t
    const float mu = (float)k * (float)m / (float)n;
    const int rsel = (int)ceilf(mu + 6.f * sqrtf(mu) + 8.f);
    if (rsel >= m) {
        if (tid == 0) tau[r] = -INFINITY;
        return;
    }
    const float *row = sample + (size_t)r * lds;
    const bool staged = m <= kStage;
    // The threshold only has to lie at or below the rsel-th largest sample:
    // the lower edge of the linear bucket (over the samples' range) that
    // holds it will do, and takes one histogram pass.
    float lo = INFINITY, hi = -INFINITY;
    for (int i = tid; i < m; i += kThreads) {
        const float v = __ldg(row + i);
        if (staged) sm.ckey[i] = __float_as_uint(v);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    {
        const int lane = lane_id(), warp = tid >> 5;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        }
        float *fred = reinterpret_cast<float *>(sm.red);
        if (lane == 0) {
            fred[warp] = lo;
            fred[kWarps + warp] = hi;
        }
        for (int b = tid; b < kNB; b += kThreads) sm.hist[b] = 0u;
        __syncthreads();
        lo = fred[0];
        hi = fred[kWarps];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            lo = fminf(lo, fred[w]);
            hi = fmaxf(hi, fred[kWarps + w]);
        }
        __syncthreads();
    }
    const float range = hi - lo;
    if (!(range > 0.f && range < INFINITY)) {  // all samples equal (or a span beyond fp32): their minimum
        if (tid == 0) tau[r] = lo;
        return;
    }
    const float scale = __fdiv_rn((float)kNB * 0.99999f, range);
    for (int i = tid; i < m; i += kThreads) {
        const float v = staged ? __uint_as_float(sm.ckey[i]) : __ldg(row + i);
        atomicAdd(&sm.hist[bucket_of(v, lo, scale)], 1u);
    }
    __syncthreads();
    find_threshold_bin(sm.hist, (uint32_t)rsel, sm.red, sm.bcast);
    if (tid == 0) {
        // bucket B starts at lo + B / scale up to rounding; a hair below it
        // (only the number of candidates depends on where exactly)
        const uint32_t B = sm.bcast[0];
        tau[r] = lo + (float)B * 0.9999f / scale;
    }
}

// ---------------------------------------------------------------------------
// 4. exact top-k of the candidates
// ---------------------------------------------------------------------------

struct SelectSmem {
    uint32_t hist[kNB];
    uint32_t red[2 * kWarps];
    uint32_t bcast[4];
    int seg_off[kSegs + 1];   // candidate slots of segment q: [seg_off[q], seg_off[q+1])
    int sel_off[kSegs + 1];   // selected entries of segment q: [sel_off[q], sel_off[q+1]) (merge path)
    uint32_t *ckey;           // [4 * seg_cap] scores (as bits), then order keys on the radix path
    int32_t *cidx;            // [4 * seg_cap] key indices
    // then, for rows of up to kBitmapMaxN keys, a bitmap of the row's
    // indices (bit s = key s selected); for longer rows, in the same space,
    uint32_t *bits;           // [kBitmapMaxN / 32]
    uint8_t *flag;            // [4 * seg_cap] 1 = selected (merge path)
    int32_t *sel;             // [k] selected indices, segment by segment, ascending in each (merge path)
};

// Rows up to this many keys emit their selection through a bitmap of the
// row (one popcount scan); longer rows merge the four ascending segment
// lists instead.
constexpr int kBitmapMaxN = 262144;

// The tail holds the bitmap of the chunk's longest row (up to kBitmapMaxN
// keys) or, for longer rows, the merge path's flags and lists.
__host__ __device__ constexpr size_t select_tail_bytes(int seg_cap, int k, int max_n) {
    const size_t bitmap = ((size_t)(max_n < kBitmapMaxN ? max_n : kBitmapMaxN) + 127) / 128 * 16;
    const size_t merge = max_n > kBitmapMaxN ? (size_t)kSegs * seg_cap + (size_t)k * 4 + 16 : 0;
    return bitmap > merge ? bitmap : merge;
}

__host__ __device__ constexpr size_t select_smem_bytes(int seg_cap, int k, int max_n) {
    return (sizeof(SelectSmem) + 15) / 16 * 16 + (size_t)kSegs * seg_cap * 8 + select_tail_bytes(seg_cap, k, max_n);
}

__device__ __forceinline__ void flag_repair(int *repair, int r) {
    const int pos = atomicAdd(&repair[0], 1);
    repair[1 + pos] = r;
}

// Number of entries of the ascending list a[0..n) below v.
__device__ __forceinline__ int lower_bound(const int32_t *a, int n, int32_t v) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < v) lo = mid + 1; else hi = mid;
    }
    return lo;
}

__global__ void __launch_bounds__(kThreads) cand_select_kernel(const int2 *__restrict__ cand,
                                                              const int *__restrict__ cand_count, int seg_cap,
                                                              int row_begin, int k, int32_t *__restrict__ idx,
                                                              int *__restrict__ repair,
                                                              unsigned long long *__restrict__ cand_total,
                                                              const int32_t *__restrict__ cu, int nseq) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    SelectSmem &sm = *reinterpret_cast<SelectSmem *>(smem_raw);
    const int r = blockIdx.x, tid = threadIdx.x;
    const int t = row_begin + r;
    const int n = t - seq_start(cu, nseq, t) + 1;  // keys visible to row t (positions 0..n-1 of its sequence)
    int32_t *out = idx + (size_t)r * k;
    if (n <= k) {  // short row: everything visible is selected
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const bool use_bits = n <= kBitmapMaxN;
    if (tid == 0) {
        sm.ckey = reinterpret_cast<uint32_t *>(smem_raw + (sizeof(SelectSmem) + 15) / 16 * 16);
        sm.cidx = reinterpret_cast<int32_t *>(sm.ckey + kSegs * seg_cap);
        sm.bits = reinterpret_cast<uint32_t *>(sm.cidx + kSegs * seg_cap);
        sm.sel = reinterpret_cast<int32_t *>(sm.bits);
        sm.flag = reinterpret_cast<uint8_t *>(sm.sel + k);
        int total = 0;
        bool bad = false;
        sm.seg_off[0] = 0;
        for (int q = 0; q < kSegs; ++q) {
            const int c = __ldg(cand_count + (size_t)r * kSegs + q);
            bad |= c > seg_cap;
            total += min(c, seg_cap);
            sm.seg_off[q + 1] = total;
        }
        sm.bcast[0] = (bad || total < k) ? 1u : 0u;
        atomicAdd(cand_total, (unsigned long long)total);
    }
    __syncthreads();
    if (sm.bcast[0] != 0u) {  // the candidates cannot decide this row: repair it
        if (tid == 0) flag_repair(repair, r);
        return;
    }
    const int total = sm.seg_off[kSegs];
    const int words = (n + 31) / 32;
    if (use_bits)
        for (int i = tid; i < words; i += kThreads) sm.bits[i] = 0u;
    // load the candidates, segment after segment, and their value range
    // (two candidates per 16-byte load where a segment's start allows it)
    float lo = INFINITY, hi = -INFINITY;
    for (int q = 0; q < kSegs; ++q) {
        const int2 *src = cand + ((size_t)r * kSegs + q) * seg_cap;
        const int o = sm.seg_off[q], c = sm.seg_off[q + 1] - o;
        const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0;
        const int c2 = vec ? c / 2 : 0;
        for (int i = tid; i < c2; i += kThreads) {
            const int4 e = __ldg(reinterpret_cast<const int4 *>(src) + i);
            const float v0 = __int_as_float(e.y), v1 = __int_as_float(e.w);
            lo = fminf(lo, fminf(v0, v1));
            hi = fmaxf(hi, fmaxf(v0, v1));
            sm.ckey[o + 2 * i] = (uint32_t)e.y;
            sm.cidx[o + 2 * i] = e.x;
            sm.ckey[o + 2 * i + 1] = (uint32_t)e.w;
            sm.cidx[o + 2 * i + 1] = e.z;
        }
        for (int i = 2 * c2 + tid; i < c; i += kThreads) {
            const int2 e = __ldg(src + i);
            const float v = __int_as_float(e.y);
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
            sm.ckey[o + i] = (uint32_t)e.y;
            sm.cidx[o + i] = e.x;
        }
    }
    {
        const int lane = lane_id(), warp = tid >> 5;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
        }
        float *fred = reinterpret_cast<float *>(sm.red);
        if (lane == 0) {
            fred[warp] = lo;
            fred[kWarps + warp] = hi;
        }
        for (int b = tid; b < kNB; b += kThreads) sm.hist[b] = 0u;
        __syncthreads();
        lo = fred[0];
        hi = fred[kWarps];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            lo = fminf(lo, fred[w]);
            hi = fmaxf(hi, fred[kWarps + w]);
        }
        __syncthreads();
    }
    // mark(i): candidate in slot i is selected
    auto mark = [&](int i) {
        if (use_bits) {
            const int32_t x = sm.cidx[i];
            atomicOr(&sm.bits[x >> 5], 1u << (x & 31));
        } else {
            sm.flag[i] = 1;
        }
    };
    // Linear buckets over [lo, hi] (a monotone map: bucket order is score
    // order, equal scores share a bucket): the bucket Bt holding the k-th
    // largest, then the few entries of Bt ranked pairwise (larger score
    // first, lower index on ties; -0.0 == +0.0 as floats).
    bool fast = false;
    const float range = hi - lo;
    const float scale = (range > 0.f && range < INFINITY) ? __fdiv_rn((float)kNB * 0.99999f, range) : 0.f;
    if (scale > 0.f) {
        for (int i = tid; i < total; i += kThreads)
            atomicAdd(&sm.hist[bucket_of(__uint_as_float(sm.ckey[i]), lo, scale)], 1u);
        __syncthreads();
        find_threshold_bin(sm.hist, (uint32_t)k, sm.red, sm.bcast);
        const uint32_t Bt = sm.bcast[0], need = sm.bcast[1];
        const uint32_t in_bt = sm.hist[Bt];
        __syncthreads();
        if (in_bt <= (uint32_t)kMaxTies) {
            fast = true;
            uint32_t *tlist = sm.hist;  // [2 * kMaxTies]: (slot, index) of the entries in Bt
            if (tid == 0) sm.bcast[3] = 0u;
            __syncthreads();
            for (int i = tid; i < total; i += kThreads) {
                const uint32_t b = bucket_of(__uint_as_float(sm.ckey[i]), lo, scale);
                if (!use_bits) sm.flag[i] = 0;
                if (b > Bt) {
                    mark(i);
                } else if (b == Bt) {
                    const uint32_t p = atomicAdd(&sm.bcast[3], 1u);
                    tlist[2 * p] = (uint32_t)i;
                    tlist[2 * p + 1] = (uint32_t)sm.cidx[i];
                }
            }
            __syncthreads();
            for (int i = tid; i < (int)in_bt; i += kThreads) {
                const uint32_t si = tlist[2 * i];
                const float vi = __uint_as_float(sm.ckey[si]);
                const int32_t xi = (int32_t)tlist[2 * i + 1];
                uint32_t before = 0;
                for (int j2 = 0; j2 < (int)in_bt; ++j2) {
                    const float vj = __uint_as_float(sm.ckey[tlist[2 * j2]]);
                    before += vj > vi || (vj == vi && (int32_t)tlist[2 * j2 + 1] < xi);
                }
                if (before < need) mark((int)si);
            }
            __syncthreads();
        }
    }
    if (!fast) {
        // exact radix select over the 32-bit order keys (a row whose range
        // is empty or whose threshold bucket is crowded)
        for (int i = tid; i < total; i += kThreads) sm.ckey[i] = order_key(__uint_as_float(sm.ckey[i]));
        __syncthreads();
        // T = the k-th largest key; quota = how many entries equal to T are taken
        uint32_t T, quota;
        select_in_candidates(sm, total, (uint32_t)k, T, quota);
        const uint32_t tied = sm.hist[T & 1023u];  // the last pass's bin of T holds every entry equal to T
        __syncthreads();
        if (tied > (uint32_t)kMaxTies) {
            if (tid == 0) flag_repair(repair, r);
            return;
        }
        // entries equal to T: the quota lowest indices (ranked pairwise in a
        // short list kept in the histogram's space)
        uint32_t *tlist = sm.hist;  // [2 * kMaxTies]: (slot, index)
        if (tid == 0) sm.bcast[3] = 0u;
        __syncthreads();
        for (int i = tid; i < total; i += kThreads) {
            if (!use_bits) sm.flag[i] = 0;
            if (sm.ckey[i] > T) {
                mark(i);
            } else if (sm.ckey[i] == T) {
                const uint32_t p = atomicAdd(&sm.bcast[3], 1u);
                tlist[2 * p] = (uint32_t)i;
                tlist[2 * p + 1] = (uint32_t)sm.cidx[i];
            }
        }
        __syncthreads();
        for (int i = tid; i < (int)tied; i += kThreads) {
            const int32_t xi = (int32_t)tlist[2 * i + 1];
            uint32_t before = 0;
            for (int j2 = 0; j2 < (int)tied; ++j2) before += (int32_t)tlist[2 * j2 + 1] < xi;
            if (before < quota) mark((int)tlist[2 * i]);
        }
        __syncthreads();
    }
    if (use_bits) {
        // the k set bits, in index order: each thread scans a run of words
        const int per = (words + kThreads - 1) / kThreads;
        const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
        uint32_t mine = 0;
        for (int w = w0; w < w1; ++w) mine += __popc(sm.bits[w]);
        uint32_t tot;
        uint32_t pos = block_scan_packed(mine, sm.red, &tot);
        for (int w = w0; w < w1; ++w) {
            uint32_t v = sm.bits[w];
            while (v) {
                const int b = __ffs(v) - 1;
                v &= v - 1u;
                out[pos++] = w * 32 + b;
            }
        }
        return;
    }
    // Longer rows: compact the selected entries in slot order (each thread
    // takes a run of consecutive slots), then merge the four ascending
    // segment lists.
    const int per = (total + kThreads - 1) / kThreads;
    const int i0 = min(total, tid * per), i1 = min(total, i0 + per);
    uint32_t mine = 0;
    for (int i = i0; i < i1; ++i) mine += sm.flag[i];
    uint32_t tot;
    uint32_t pos = block_scan_packed(mine, sm.red, &tot);
    // segment q's selected entries start at the rank of its first slot
    for (int q = 0; q <= kSegs; ++q) {
        const int b = sm.seg_off[q];
        if (b >= i0 && b < i1) {
            uint32_t p = pos;
            for (int i = i0; i < b; ++i) p += sm.flag[i];
            sm.sel_off[q] = (int)p;
        } else if (b == total && tid == 0) {
            sm.sel_off[q] = (int)tot;
        }
    }
    for (int i = i0; i < i1; ++i)
        if (sm.flag[i]) sm.sel[pos++] = sm.cidx[i];
    __syncthreads();
    // an entry's output position is its rank in its own list plus the
    // entries of the other lists with a lower index
    for (int p = tid; p < k; p += kThreads) {
        int q = 0;
        while (q < kSegs - 1 && p >= sm.sel_off[q + 1]) ++q;
        const int32_t v = sm.sel[p];
        int o = p - sm.sel_off[q];
        for (int q2 = 0; q2 < kSegs; ++q2)
            if (q2 != q) o += lower_bound(sm.sel + sm.sel_off[q2], sm.sel_off[q2 + 1] - sm.sel_off[q2], v);
        out[o] = v;
    }
}

// ---------------------------------------------------------------------------
// 5. repair: score a listed row in full on the CUDA cores, then select it
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(h) : "h"(v));
    const __half2 hh = *reinterpret_cast<const __half2 *>(&h);
    return __half22float2(hh);
}

constexpr int kRepairHeads = 8;  // heads accumulated at a time

__global__ void __launch_bounds__(kRepairThreads) repair_rows_kernel(
    const uint8_t *__restrict__ q8, const float *__restrict__ sq, const float *__restrict__ w,
    const uint8_t *__restrict__ k8, const float *__restrict__ sk, int HI, int dI, int row_begin, int k,
    const int *__restrict__ repair, float *__restrict__ scratch, int64_t scratch_ld, int32_t *__restrict__ idx,
    const int32_t *__restrict__ cu, int nseq) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    float *qf = reinterpret_cast<float *>(smem_raw + (sizeof(TopkSmem) + 15) / 16 * 16);  // [HI * dI]
    float *wf = qf + HI * dI;                                                              // [HI]
    const int n_rep = __ldg(repair);
    float *row = scratch + (size_t)blockIdx.x * scratch_ld;
    for (int j = blockIdx.x; j < n_rep; j += gridDim.x) {
        const int r = __ldg(repair + 1 + j);
        const int t = row_begin + r;
        const int start = seq_start(cu, nseq, t);
        const int n = t - start + 1;
        for (int i = threadIdx.x; i < HI * dI / 2; i += kRepairThreads) {
            const uint16_t v = reinterpret_cast<const uint16_t *>(q8 + (size_t)t * HI * dI)[i];
            const float2 f = e4m3x2_to_float2(v);
            qf[2 * i] = f.x;
            qf[2 * i + 1] = f.y;
        }
        for (int i = threadIdx.x; i < HI; i += kRepairThreads) wf[i] = __ldg(w + (size_t)t * HI + i);
        __syncthreads();
        const float sqt = __ldg(sq + t);
        for (int i = threadIdx.x; i < n; i += kRepairThreads) {
            const int s = start + i;
            const uint16_t *kr = reinterpret_cast<const uint16_t *>(k8 + (size_t)s * dI);
            float acc = 0.f;
            for (int h0 = 0; h0 < HI; h0 += kRepairHeads) {
                float d[kRepairHeads];
#pragma unroll
                for (int j2 = 0; j2 < kRepairHeads; ++j2) d[j2] = 0.f;
                for (int c = 0; c < dI; c += 2) {
                    const float2 kf = e4m3x2_to_float2(__ldg(kr + c / 2));
#pragma unroll
                    for (int j2 = 0; j2 < kRepairHeads; ++j2) {
                        const float *qr = qf + (h0 + j2) * dI + c;
                        d[j2] = fmaf(qr[0], kf.x, d[j2]);
                        d[j2] = fmaf(qr[1], kf.y, d[j2]);
                    }
                }
#pragma unroll
                for (int j2 = 0; j2 < kRepairHeads; ++j2) acc = fmaf(wf[h0 + j2], fmaxf(d[j2], 0.f), acc);
            }
            row[i] = acc * sqt * __ldg(sk + s);
        }
        __syncthreads();
        topk_row_radix<true>(row, n, k, idx + (size_t)r * k, sm);
        __syncthreads();
    }
}

__global__ void fused_stats_kernel(const int *__restrict__ repair, const unsigned long long *__restrict__ cand_total,
                                   int64_t *__restrict__ stats) {
    stats[0] = repair[0];
    stats[1] = (int64_t)*cand_total;
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

namespace {

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int sm_count_here() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}


}  // namespace

FusedTopkLayout fused_topk_layout(int row_begin, int n_rows, int k, int HI, int dI) {
    FusedTopkLayout L{};
    const int row_end = row_begin + n_rows;
    const int stride = indexer_sample_stride();
    // candidates per row: room for about twice what the threshold lets through
    // a segment holds about twice its share of what the threshold lets
    // through (about k + 6 sqrt(32 k) + 256 per row); a row with at most
    // keep_all keys keeps them all (each quarter holds at most n/4 + 32)
    L.seg_cap = (3 * k / 4 > 1024 ? 3 * k / 4 : 1024) + 32;
    L.keep_all = kSegs * (L.seg_cap - 32);
    L.lds = ((row_end > 0 ? (row_end - 1) / stride + 1 : 1) + 3) / 4 * 4;
    L.repair_ctas = sm_count_here();
    L.scratch_ld = ((row_end > 0 ? row_end : 1) + 3) / 4 * 4;
    size_t off = 0;
    L.sample_off = off;
    off = align256(off + (size_t)n_rows * L.lds * 4);
    L.tau_off = off;
    off = align256(off + (size_t)n_rows * 4);
    L.cand_off = off;
    off = align256(off + (size_t)n_rows * kSegs * L.seg_cap * 8);
    L.count_off = off;
    off = align256(off + (size_t)n_rows * kSegs * 4);
    L.repair_off = off;
    off = align256(off + ((size_t)n_rows + 1) * 4);
    L.total_off = off;
    off = align256(off + 8);
    L.scratch_off = off;
    off = align256(off + (size_t)L.repair_ctas * L.scratch_ld * 4);
    L.total = off;
    L.select_smem = select_smem_bytes(L.seg_cap, k, row_end > 0 ? row_end : 1);
    L.repair_smem = (sizeof(TopkSmem) + 15) / 16 * 16 + ((size_t)HI * dI + HI) * 4;
    return L;
}

bool fused_topk_supported(int k, int HI, int dI) {
    if (k < 1 || !indexer_tc_supported(HI, dI)) return false;
    // the worst case is a chunk whose rows take the merge path
    const FusedTopkLayout L = fused_topk_layout(0, kBitmapMaxN + 1, k, HI, dI);
    return L.select_smem <= 200 * 1024 && L.repair_smem <= 200 * 1024;
}

namespace {

struct FusedPtrs {
    float *sample, *tau, *scratch;
    int2 *cand;
    int *counts, *repair;
    unsigned long long *cand_total;
};

FusedPtrs fused_ptrs(const FusedTopkLayout &lay, void *ws) {
    char *base = static_cast<char *>(ws);
    FusedPtrs p;
    p.sample = reinterpret_cast<float *>(base + lay.sample_off);
    p.tau = reinterpret_cast<float *>(base + lay.tau_off);
    p.cand = reinterpret_cast<int2 *>(base + lay.cand_off);
    p.counts = reinterpret_cast<int *>(base + lay.count_off);
    p.repair = reinterpret_cast<int *>(base + lay.repair_off);
    p.cand_total = reinterpret_cast<unsigned long long *>(base + lay.total_off);
    p.scratch = reinterpret_cast<float *>(base + lay.scratch_off);
    return p;
}

}  // namespace

cudaError_t launch_indexer_topk_stage(int stage, const uint8_t *q8, const float *sq, const float *w,
                                      const uint8_t *k8, const float *sk, int L, int HI, int dI, int row_begin,
                                      int n_rows, int k, int32_t *idx, void *ws, int64_t *stats,
                                      const int32_t *cu, int nseq, cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    const FusedTopkLayout lay = fused_topk_layout(row_begin, n_rows, k, HI, dI);
    const FusedPtrs P = fused_ptrs(lay, ws);
    const int row_end = row_begin + n_rows;
    cudaError_t e = cudaSuccess;
    if (stage == 1) {
        // sampled scores of the rows that are not kept whole (t + 1 > keep_all)
        const int s0 = row_begin > lay.keep_all ? row_begin : lay.keep_all;
        if (s0 < row_end) {
            e = launch_indexer_sample_tc(q8, sq, w, k8, sk, L, HI, dI, s0, row_end - s0,
                                         P.sample + (size_t)(s0 - row_begin) * lay.lds, lay.lds, cu, nseq, stream);
            if (e != cudaSuccess) return e;
        }
        // thresholds (and the repair list emptied)
        e = set_smem_at_least<sample_threshold_kernel>(sizeof(ThreshSmem));
        if (e != cudaSuccess) return e;
        sample_threshold_kernel<<<n_rows, kThreads, sizeof(ThreshSmem), stream>>>(
            P.sample, lay.lds, row_begin, n_rows, k, lay.keep_all, indexer_sample_stride(), P.tau, P.repair,
            P.cand_total, cu, nseq);
        return cudaGetLastError();
    }
    if (stage == 2) {
        // candidates of the rows with more than k visible keys (t >= k)
        const int c0 = row_begin > k ? row_begin : k;
        if (c0 >= row_end) return cudaSuccess;
        return launch_indexer_cand_tc(q8, sq, w, k8, sk, L, HI, dI, c0, row_end - c0, P.tau + (c0 - row_begin),
                                      P.cand + (size_t)(c0 - row_begin) * kSegs * lay.seg_cap,
                                      P.counts + (size_t)(c0 - row_begin) * kSegs, lay.seg_cap, cu, nseq, stream);
    }
    if (stage == 3) {
        // exact selection, then the repair of the listed rows (which exits at
        // once when there are none)
        e = set_smem_at_least<cand_select_kernel>(lay.select_smem);
        if (e != cudaSuccess) return e;
        cand_select_kernel<<<n_rows, kThreads, lay.select_smem, stream>>>(P.cand, P.counts, lay.seg_cap, row_begin,
                                                                          k, idx, P.repair, P.cand_total, cu, nseq);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = set_smem_at_least<repair_rows_kernel>(lay.repair_smem);
        if (e != cudaSuccess) return e;
        repair_rows_kernel<<<lay.repair_ctas, kRepairThreads, lay.repair_smem, stream>>>(
            q8, sq, w, k8, sk, HI, dI, row_begin, k, P.repair, P.scratch, lay.scratch_ld, idx, cu, nseq);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if (stats != nullptr) {
            fused_stats_kernel<<<1, 1, 0, stream>>>(P.repair, P.cand_total, stats);
            e = cudaGetLastError();
        }
        return e;
    }
    return cudaErrorInvalidValue;
}

}  // namespace dsa
