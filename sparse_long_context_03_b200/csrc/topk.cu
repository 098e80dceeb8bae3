// topk.cu -- deterministic per-row top-k selection.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式:
//     Omega_t = { s | I[t,s] in Top-k(I[t,:]) }
// report translation section 5.1.2 (a row with t+1 <= k keeps all of 0..t)
// and section 5.2.1 (the selection must be deterministic).
//
// Scores map to order-preserving 32-bit keys (-0.0 and +0.0 equal).  The
// selected set is every entry whose key is above the k-th largest key T,
// plus the lowest-indexed entries equal to T; it is emitted in ascending
// index order.  No sort, every step is a count, so the result does not
// depend on scheduling.
//
// Three kernels share the steps below:
//   topk_rows_bitmap_kernel   one CTA per row (prefill chunks; row bounds up
//                             to 557K entries), selection marked in a bitmap;
//   topk_rows_kernel          one CTA per row for longer row bounds, ordered
//                             lists;
//   topk_rows_cluster_kernel  one 8-CTA cluster per row when there are fewer
//                             rows than SMs (decode).
// Per row:
//   1. the row's value range [vmin, vmax] -- skipped when the indexer already
//      produced it (row statistics);
//   2. a histogram over 2048 linear buckets of that range (a monotone map,
//      so bucket order is key order; scores spread over many buckets, which
//      keeps shared-memory atomics free of hot spots) -- of the whole row, or,
//      for long rows with statistics, of a 1/8 sample that brackets the
//      threshold in a band of buckets (the bitmap kernel; see there);
//   3. a collect pass: entries above the threshold bucket (or band) are
//      winners, entries in it are candidates.
// The chosen candidates (by key, then index) are found by direct ranking when
// there are few of them, and otherwise by a small radix select or a second
// histogram; the output is written in ascending index order.  Only
// candidates are turned into keys.  If the threshold bucket holds more
// candidates than fit in shared memory (massive exact ties), the row falls
// back to a radix select over the whole row (11/11/10-bit passes) followed
// by an ordered compaction: slower, same result.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "topk_core.cuh"

namespace dsa {

namespace {


// Final step of one row: the shared lists hold, in index order, the n_above
// winners (alist) and the cnt threshold-bucket candidates (ckey / cidx);
// choose `need` candidates (larger key first, lower index on ties) and merge
// both ascending lists into out[0..n_above+need).
__device__ void finish_row(TopkSmem &sm, const int32_t *alist, uint32_t cnt, uint32_t need, uint32_t n_above,
                           int32_t *out) {
    const int tid = threadIdx.x;
    // choose `need` candidates: larger key first, lower index on ties
    if (cnt <= (uint32_t)kSmallCand) {
        // Direct ranking: candidate i is chosen iff fewer than `need`
        // candidates beat it (larger key, or equal key and lower index).
        // Candidates sit in index order, so "lower index" is "earlier slot".
        const int i = tid;
        const bool act = i < (int)cnt;
        const uint32_t ki = act ? sm.ckey[i] : 0u;
        const int32_t ix = act ? sm.cidx[i] : 0;
        uint32_t rank = 0;
        for (int j = 0; j < (int)cnt; ++j) {
            const uint32_t kj = sm.ckey[j];
            rank += (kj > ki) || (kj == ki && j < i);
        }
        const bool chosen = act && rank < need;
        uint32_t tot;
        const uint32_t ex = block_scan_packed(chosen ? 1u : 0u, sm.red, &tot);
        if (chosen) sm.cidx[ex] = ix;  // ex <= i, and slot i was read above
        __syncthreads();
    } else {
        uint32_t T, quota;
        select_in_candidates(sm, (int)cnt, need, T, quota);
        uint32_t run_g = 0, run_e = 0;
        for (int base = 0; base < (int)cnt; base += kThreads) {
            const int i = base + tid;
            const uint32_t key = i < (int)cnt ? sm.ckey[i] : 0u;
            const int32_t ix = i < (int)cnt ? sm.cidx[i] : 0;
            const bool gt = i < (int)cnt && key > T;
            const bool eq = i < (int)cnt && key == T;
            uint32_t tot;
            const uint32_t ex = block_scan_packed((gt ? 1u : 0u) | (eq ? 0x10000u : 0u), sm.red, &tot);
            const uint32_t gb = run_g + (ex & 0xFFFFu), eb = run_e + (ex >> 16);
            // positions only move left and this chunk was read before the scan's barriers
            if (gt || (eq && eb < quota)) sm.cidx[gb + min(eb, quota)] = ix;
            run_g += tot & 0xFFFFu;
            run_e += tot >> 16;
            __syncthreads();
        }
    }

    // ---- merge the two ascending lists into the output
    const int na = (int)n_above, nd = (int)need;
    const int32_t *dl = sm.cidx;
    for (int a = tid; a < na; a += kThreads) {
        const int32_t v = alist[a];
        int lo = 0, hi = nd;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (dl[mid] < v) lo = mid + 1; else hi = mid;
        }
        out[a + lo] = v;
    }
    for (int d = tid; d < nd; d += kThreads) {
        const int32_t v = dl[d];
        int lo = 0, hi = na;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (alist[mid] < v) lo = mid + 1; else hi = mid;
        }
        out[d + lo] = v;
    }
}

// Value range of one row (n > k), from the indexer's row statistics when
// given, else from a pass over the row; sets the bucket map of the row.
// Returns false when the row was finished here (every entry equal, or a span
// that overflows fp32, which takes the exact whole-row path).
struct RowRange {
    float vmin, scale;
};

__device__ bool row_range(const float *row, int n, int k, int r, const float *row_stats, TopkSmem &sm, int32_t *out,
                          RowRange &rg) {
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    float vmin = INFINITY, vmax = -INFINITY;
    if (row_stats != nullptr) {
        if (tid < 4) {
            vmin = __ldg(row_stats + (size_t)r * 8 + 2 * tid);
            vmax = __ldg(row_stats + (size_t)r * 8 + 2 * tid + 1);
        }
    } else
    for (int i0 = tid * kVec; i0 < n; i0 += kChunk) {
        float x[kVec];
        const int m = load_vals(row, i0, n, x);
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            if (j < m) {
                vmin = fminf(vmin, x[j]);
                vmax = fmaxf(vmax, x[j]);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
    }
    float *fred = reinterpret_cast<float *>(sm.red);
    if (lane == 0) {
        fred[warp] = vmin;
        fred[kWarps + warp] = vmax;
    }
    __syncthreads();
    vmin = fred[0];
    vmax = fred[kWarps];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        vmin = fminf(vmin, fred[w]);
        vmax = fmaxf(vmax, fred[kWarps + w]);
    }
    __syncthreads();
    if (vmin == vmax) {  // every entry ties: the k lowest indices
        for (int i = tid; i < k; i += kThreads) out[i] = i;
        return false;
    }
    const float range = vmax - vmin;
    if (!(range < INFINITY)) {  // span overflows fp32: exact slow path
        topk_row_radix(row, n, k, out, sm);
        return false;
    }
    rg.vmin = vmin;
    // slightly below kNB / range so that vmax itself maps below kNB
    rg.scale = __fdiv_rn((float)kNB * 0.99999f, range);
    return true;
}

// Threshold bucket of one row: a histogram over the kNB buckets of the row's
// range and the bucket Bt holding the k-th largest entry.  Returns false when
// the row was finished here (the threshold bucket does not fit in shared
// memory: exact whole-row path).
struct RowThreshold {
    float vmin, scale;
    uint32_t Bt, need, n_above, cnt;
};

__device__ bool row_hist_threshold(const float *row, int n, int k, const RowRange &rg, TopkSmem &sm, int32_t *out,
                                   RowThreshold &t) {
    const int tid = threadIdx.x;
    for (int i = tid; i < kNB; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i0 = tid * kVec; i0 < n; i0 += kChunk) {
        float x[kVec];
        const int m = load_vals(row, i0, n, x);
#pragma unroll
        for (int j = 0; j < kVec; ++j)
            if (j < m) atomicAdd(&sm.hist[bucket_of(x[j], rg.vmin, rg.scale)], 1u);
    }
    __syncthreads();
    find_threshold_bin(sm.hist, (uint32_t)k, sm.red, sm.bcast);
    t.Bt = sm.bcast[0];
    t.need = sm.bcast[1];       // taken from the threshold bucket
    t.n_above = sm.bcast[2];    // entries in buckets above it
    t.cnt = sm.hist[t.Bt];
    __syncthreads();
    if (t.cnt > (uint32_t)kCap) {
        topk_row_radix(row, n, k, out, sm);
        return false;
    }
    t.vmin = rg.vmin;
    t.scale = rg.scale;
    return true;
}

__device__ bool row_threshold(const float *row, int n, int k, int r, const float *row_stats, TopkSmem &sm,
                              int32_t *out, RowThreshold &t) {
    RowRange rg;
    if (!row_range(row, n, k, r, row_stats, sm, out, rg)) return false;
    return row_hist_threshold(row, n, k, rg, sm, out, t);
}

__global__ void __launch_bounds__(kThreads) topk_rows_kernel(const float *__restrict__ scores, int64_t ld,
                                                            int row_begin, const int32_t *__restrict__ row_len,
                                                            int max_len, int k, int32_t *__restrict__ idx,
                                                            const float *__restrict__ row_stats) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    int32_t *alist = reinterpret_cast<int32_t *>(smem_raw + sizeof(TopkSmem));

    const int r = blockIdx.x;
    const int n = row_length(row_len, r, row_begin, max_len);
    const float *row = scores + (size_t)r * ld;
    int32_t *out = idx + (size_t)r * k;
    const int tid = threadIdx.x;

    if (n <= k) {  // short row: everything visible is selected
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }

    RowThreshold th;
    if (!row_threshold(row, n, k, r, row_stats, sm, out, th)) return;
    const float vmin = th.vmin, scale = th.scale;
    const uint32_t Bt = th.Bt, need = th.need, n_above = th.n_above, cnt = th.cnt;

    // ---- pass 3: ordered collect
    uint32_t run_a = 0, run_c = 0;
    for (int base = 0; base < n; base += kChunk) {
        const int i0 = base + tid * kVec;
        float x[kVec] = {};
        const int m = i0 < n ? load_vals(row, i0, n, x) : 0;
        uint32_t cls[kVec];
        uint32_t na = 0, nc = 0;
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const uint32_t b = bucket_of(x[j], vmin, scale);
            cls[j] = j >= m ? 0u : (b > Bt ? 2u : (b == Bt ? 1u : 0u));
            na += cls[j] == 2u;
            nc += cls[j] == 1u;
        }
        uint32_t tot;
        const uint32_t ex = block_scan_packed(na | (nc << 16), sm.red, &tot);
        uint32_t pa = run_a + (ex & 0xFFFFu), pc = run_c + (ex >> 16);
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            if (cls[j] == 2u) alist[pa++] = i0 + j;
            if (cls[j] == 1u) {
                sm.ckey[pc] = order_key(x[j]);
                sm.cidx[pc] = i0 + j;
                ++pc;
            }
        }
        run_a += tot & 0xFFFFu;
        run_c += tot >> 16;
    }
    __syncthreads();

    finish_row(sm, alist, cnt, need, n_above, out);
}


// ---------------------------------------------------------------------------
// Many rows of moderate length (prefill chunks): the collect pass marks the
// selected entries in a bitmap of the row instead of building ordered lists.
//
// Threshold band.  With the row's range known in advance (the indexer's row
// statistics), a histogram of every eighth 16-entry piece of the row brackets
// the k-th largest entry: the band of buckets [Blo, Bhi] holds the sample's
// (k f +- m)-th largest entries, f the sampled fraction and m four standard
// deviations of the sampled count plus four.  Without statistics, or when the
// band turns out not to contain the k-th entry (or holds too many entries),
// the full histogram gives the exact threshold bucket (Blo = Bhi = Bt).
// Either way the selection is exact: the counts that decide it are taken over
// the whole row in the collect pass, and only the pass that locates the band
// is sampled.
//
// Collect.  Entries above the band are winners: each sets its bit with one
// atomicOr per thread and chunk (a thread's kVec = 16 entries lie in one
// 32-bit word).  Entries in the band go, in any order, to the candidate list
// through one atomicAdd per warp.  No block-wide barrier runs inside the pass.
// The chosen candidates -- larger key first, then lower index -- set their
// bits too (a few by direct ranking; more through a second histogram over
// their own value range), and one scan of the bitmap writes the k indices in
// ascending order.  Rows whose threshold sub-bucket holds too many entries to
// rank pairwise (massive exact ties) take the whole-row radix path.
// ---------------------------------------------------------------------------

constexpr int kMaxTiedRanked = 512;     // tied candidates ranked pairwise
// Rows up to 524288 entries: the bitmap (64 KB) and the lists still fit twice
// per SM up to 262144 entries, once beyond.
constexpr int kBitmapSmemMax = 124 * 1024;
constexpr int kSampleStride = 8;        // one 16-entry piece in eight is sampled
// rows of at least 16 k entries are sampled (below that the band's larger
// candidate list costs about what the skipped histogram saves)
constexpr int kSampleMinRowPerK = 16;

__host__ __device__ constexpr int bitmap_words(int max_len) { return ((max_len + 31) / 32 + 3) / 4 * 4; }
__host__ __device__ constexpr size_t bitmap_smem_bytes(int max_len) {
    return sizeof(TopkSmem) + sizeof(uint32_t) * (size_t)bitmap_words(max_len);
}

// Block-wide sum of one value per thread (two barriers; sm.red reused).
__device__ __forceinline__ uint32_t block_sum(uint32_t v, TopkSmem &sm) {
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    if (lane_id() == 0) sm.red[threadIdx.x >> 5] = v;
    __syncthreads();
    uint32_t tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += sm.red[w];
    __syncthreads();
    return tot;
}

// One pass over the row: entries that classify as winners set their bits,
// candidates join the candidate list (at most kCap are stored; all are
// counted).  Returns the number of winners; the candidate count is left in
// sm.bcast[3].  The trip count is the same for every thread: the warp
// shuffles need all 32 lanes in every iteration.
template <typename Classify>
__device__ uint32_t collect_by(const float *row, int n, Classify classify, TopkSmem &sm, uint32_t *bits) {
    const int tid = threadIdx.x, lane = lane_id();
    const int words = (n + 31) / 32;
    for (int w = tid; w < words; w += kThreads) bits[w] = 0u;
    if (tid == 0) sm.bcast[3] = 0u;
    __syncthreads();
    uint32_t n_win = 0;
    for (int base = 0; base < n; base += kChunk) {
        const int i0 = base + tid * kVec;
        float x[kVec] = {};
        const int m = i0 < n ? load_vals(row, i0, n, x) : 0;
        uint32_t win = 0u, cmask = 0u;
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const uint32_t cls = classify(x[j]);  // 2 winner, 1 candidate, 0 neither
            if (j < m && cls == 2u) win |= 1u << j;
            if (j < m && cls == 1u) cmask |= 1u << j;
        }
        if (win) atomicOr(&bits[i0 >> 5], win << (i0 & 31));
        n_win += __popc(win);
        // warp-aggregated slots for the candidates
        const uint32_t c = __popc(cmask);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t wtot = __shfl_sync(0xFFFFFFFFu, incl, 31);
        uint32_t slot = 0u;
        if (lane == 31 && wtot) slot = atomicAdd(&sm.bcast[3], wtot);
        slot = __shfl_sync(0xFFFFFFFFu, slot, 31) + incl - c;
        while (cmask) {
            const int j = __ffs(cmask) - 1;
            cmask &= cmask - 1u;
            if (slot < (uint32_t)kCap) {
                sm.ckey[slot] = order_key(x[j]);
                sm.cidx[slot] = i0 + j;
            }
            ++slot;
        }
    }
    return block_sum(n_win, sm);  // its barriers also publish the list and the count
}

// Collect by buckets: above Bhi winners, [Blo, Bhi] candidates.
__device__ uint32_t collect_band(const float *row, int n, const RowRange &rg, uint32_t Blo, uint32_t Bhi,
                                 TopkSmem &sm, uint32_t *bits) {
    return collect_by(
        row, n,
        [&](float x) -> uint32_t {
            const uint32_t b = bucket_of(x, rg.vmin, rg.scale);
            return b > Bhi ? 2u : (b >= Blo ? 1u : 0u);
        },
        sm, bits);
}

// Locate the band from a sample of the row and collect it.  Returns true with
// the candidate count and the number still to choose when the band holds the
// k-th largest entry and its candidates fit; false otherwise.
__device__ bool sampled_band(const float *row, int n, int k, const RowRange &rg, TopkSmem &sm, uint32_t *bits,
                             uint32_t &cnt, uint32_t &need) {
    const int tid = threadIdx.x;
    constexpr int kPiece = kVec * kSampleStride;  // entries from one sampled piece to the next
    for (int i = tid; i < kNB; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i0 = tid * kPiece; i0 < n; i0 += kThreads * kPiece) {
        float x[kVec];
        const int m = load_vals(row, i0, n, x);
#pragma unroll
        for (int j = 0; j < kVec; ++j)
            if (j < m) atomicAdd(&sm.hist[bucket_of(x[j], rg.vmin, rg.scale)], 1u);
    }
    const int pieces = (n + kPiece - 1) / kPiece;
    const int n_s = (pieces - 1) * kVec + min(kVec, n - (pieces - 1) * kPiece);
    const float expect = (float)k * (float)n_s / (float)n;
    const float margin = 4.f * sqrtf(expect) + 4.f;
    const int need_hi = max(1, (int)floorf(expect - margin));
    const int need_lo = (int)ceilf(expect + margin);
    __syncthreads();
    find_threshold_bin(sm.hist, (uint32_t)need_hi, sm.red, sm.bcast);
    const uint32_t Bhi = sm.bcast[0];
    __syncthreads();
    uint32_t Blo = 0;
    if (need_lo <= n_s) {
        find_threshold_bin(sm.hist, (uint32_t)need_lo, sm.red, sm.bcast);
        Blo = sm.bcast[0];
        __syncthreads();
    }
    // The pass over the whole row compares values with two thresholds at the
    // band's bucket edges (any monotone split will do: its counts decide).
    const float t_hi = rg.vmin + (float)(Bhi + 1) / rg.scale;
    const float t_lo = Blo == 0 ? -INFINITY : rg.vmin + (float)Blo / rg.scale;
    const uint32_t n_win = collect_by(
        row, n, [&](float x) -> uint32_t { return x >= t_hi ? 2u : (x >= t_lo ? 1u : 0u); }, sm, bits);
    const uint32_t n_cand = sm.bcast[3];
    __syncthreads();
    if (n_win > (uint32_t)k || n_win + n_cand < (uint32_t)k || n_cand > (uint32_t)kCap) return false;
    cnt = n_cand;
    need = (uint32_t)k - n_win;
    return true;
}

// Inverse of order_key (-0.0 comes back as +0.0, which orders the same).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// Choose `need` of the cnt candidates (larger key first, lower index on ties)
// and set their bits: a second histogram over the candidates' own value
// range finds the sub-bucket holding the need-th largest; entries above it
// are chosen and the few inside it are ranked pairwise.  Returns false when
// that sub-bucket holds more than kMaxTiedRanked entries (massive ties): the
// caller then takes the exact whole-row path.
__device__ bool choose_by_fine_histogram(TopkSmem &sm, uint32_t *bits, uint32_t cnt, uint32_t need) {
    if (need == 0) return true;  // the winners alone are the k largest
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    float lo = INFINITY, hi = -INFINITY;
    for (int i = tid; i < (int)cnt; i += kThreads) {
        const float v = key_value(sm.ckey[i]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
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
    for (int i = tid; i < kNB; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    lo = fred[0];
    hi = fred[kWarps];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        lo = fminf(lo, fred[w]);
        hi = fmaxf(hi, fred[kWarps + w]);
    }
    __syncthreads();
    // equal values: one sub-bucket; otherwise the same monotone map as the row's
    const float scale = hi > lo ? __fdiv_rn((float)kNB * 0.99999f, hi - lo) : 0.f;
    for (int i = tid; i < (int)cnt; i += kThreads)
        atomicAdd(&sm.hist[bucket_of(key_value(sm.ckey[i]), lo, scale)], 1u);
    __syncthreads();
    find_threshold_bin(sm.hist, need, sm.red, sm.bcast);
    const uint32_t Bs = sm.bcast[0];
    const uint32_t quota = sm.bcast[1];  // to take from sub-bucket Bs
    const uint32_t in_bs = sm.hist[Bs];
    __syncthreads();
    if (in_bs > (uint32_t)kMaxTiedRanked) return false;
    // entries above Bs are chosen; those in Bs move to a short list (the
    // histogram's space: 2 x kMaxTiedRanked words) and are ranked there
    uint32_t *bs_list = sm.hist;
    if (tid == 0) sm.bcast[3] = 0u;
    __syncthreads();
    for (int i = tid; i < (int)cnt; i += kThreads) {
        const uint32_t ki = sm.ckey[i];
        const uint32_t b = bucket_of(key_value(ki), lo, scale);
        if (b > Bs) {
            const int32_t xi = sm.cidx[i];
            atomicOr(&bits[xi >> 5], 1u << (xi & 31));
        } else if (b == Bs) {
            const uint32_t slot = atomicAdd(&sm.bcast[3], 1u);
            bs_list[2 * slot] = ki;
            bs_list[2 * slot + 1] = (uint32_t)sm.cidx[i];
        }
    }
    __syncthreads();
    for (int i = tid; i < (int)in_bs; i += kThreads) {
        const uint32_t ki = bs_list[2 * i];
        const int32_t xi = (int32_t)bs_list[2 * i + 1];
        uint32_t before = 0;  // entries of the sub-bucket that come first
        for (int j = 0; j < (int)in_bs; ++j) {
            const uint32_t kj = bs_list[2 * j];
            before += (kj > ki) || (kj == ki && (int32_t)bs_list[2 * j + 1] < xi);
        }
        if (before < quota) atomicOr(&bits[xi >> 5], 1u << (xi & 31));
    }
    return true;
}

__global__ void __launch_bounds__(kThreads) topk_rows_bitmap_kernel(const float *__restrict__ scores, int64_t ld,
                                                                   int row_begin,
                                                                   const int32_t *__restrict__ row_len,
                                                                   int max_len, int k, int32_t *__restrict__ idx,
                                                                   const float *__restrict__ row_stats) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    uint32_t *bits = reinterpret_cast<uint32_t *>(smem_raw + sizeof(TopkSmem));

    const int r = blockIdx.x;
    const int n = row_length(row_len, r, row_begin, max_len);
    const float *row = scores + (size_t)r * ld;
    int32_t *out = idx + (size_t)r * k;
    const int tid = threadIdx.x;

    if (n <= k) {  // short row: everything visible is selected
        for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    RowRange rg;
    if (!row_range(row, n, k, r, row_stats, sm, out, rg)) return;
    uint32_t cnt = 0, need = 0;
    bool banded = false;
    if (row_stats != nullptr && n >= kSampleMinRowPerK * k) banded = sampled_band(row, n, k, rg, sm, bits, cnt, need);
    if (!banded) {
        RowThreshold th;
        if (!row_hist_threshold(row, n, k, rg, sm, out, th)) return;
        (void)collect_band(row, n, rg, th.Bt, th.Bt, sm, bits);
        cnt = th.cnt;
        need = th.need;
    }

    // ---- choose `need` of the cnt candidates: larger key first, lower index on ties
    if (cnt <= (uint32_t)kSmallCand) {
        const int i = tid;
        if (i < (int)cnt) {
            const uint32_t ki = sm.ckey[i];
            const int32_t xi = sm.cidx[i];
            uint32_t rank = 0;
            for (int j = 0; j < (int)cnt; ++j) {
                const uint32_t kj = sm.ckey[j];
                rank += (kj > ki) || (kj == ki && sm.cidx[j] < xi);
            }
            if (rank < need) atomicOr(&bits[xi >> 5], 1u << (xi & 31));
        }
    } else if (!choose_by_fine_histogram(sm, bits, cnt, need)) {
        topk_row_radix(row, n, k, out, sm);
        return;
    }
    __syncthreads();

    // ---- the k set bits, in index order
    const int words = (n + 31) / 32;
    const int per = (words + kThreads - 1) / kThreads;
    const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
    uint32_t mine = 0;
    for (int w = w0; w < w1; ++w) mine += __popc(bits[w]);
    uint32_t tot;
    uint32_t pos = block_scan_packed(mine, sm.red, &tot);
    for (int w = w0; w < w1; ++w) {
        uint32_t v = bits[w];
        while (v) {
            const int b = __ffs(v) - 1;
            v &= v - 1u;
            out[pos++] = w * 32 + b;
        }
    }
}

// ---------------------------------------------------------------------------
// Long rows, few of them (decode): one thread-block cluster per row.
//
// The row is cut into kClusterSize contiguous slices, one per CTA.  Each pass
// runs on every slice in parallel; the row's value range (unless the indexer
// recorded it) and the bucket histogram are combined through distributed
// shared memory.  Every exchange is bracketed by hardware cluster barriers
// (no flag polling), and a CTA leaves only after the last barrier that
// follows any remote access to its shared memory.
//
// Usual case (at most kSmallCand entries in the threshold bucket, slices of
// at most 32k entries): every CTA reads each slice's winner and candidate
// counts from the other CTAs' histograms, marks its own winners in a bitmap
// of its slice, and writes its candidates into every CTA's candidate list
// at its slice's offset.  After one barrier every CTA ranks all candidates
// (larger key first, then lower index), marks the chosen ones of its slice
// and writes its slice's set bits in ascending order at its slice's output
// offset -- the output is written by all CTAs at once.  Otherwise rank 0
// gathers the per-slice ordered lists (slices are in index order, so
// concatenation keeps them ascending) and finishes the row as the single-CTA
// kernel does.
// ---------------------------------------------------------------------------

constexpr int kClusterSize = 8;

constexpr int kCoarse = 64;             // super-buckets of the histogram exchange
constexpr int kFine = kNB / kCoarse;     // buckets per super-bucket
static_assert(kNB == 4 * kThreads && kFine == 32 && kCoarse * kClusterSize == kThreads, "exchange layout");

struct ClusterExtra {
    float range[2];        // this slice's min, max
    uint32_t counts[2];    // this slice's winners, candidates
    uint32_t coarse[kCoarse];                 // this slice's super-bucket counts
    uint32_t allc[kClusterSize][kCoarse];     // every slice's super-bucket counts
    uint32_t allf[kClusterSize][kFine];       // every slice's buckets of the threshold super-bucket
    uint32_t sel[8];                          // super-bucket, entries above it; Bt, need, n_above, cnt, Bt - 32 S
    // usual case: per slice, entries above the threshold bucket, entries in
    // it, and chosen candidates; this slice's candidates written so far
    uint32_t slice_above[kClusterSize];
    uint32_t slice_cand[kClusterSize];
    uint32_t slice_chosen[kClusterSize];
    uint32_t ncand;
};

// Dynamic shared memory of the cluster kernel: the single-CTA layout and the
// exchange area, then (cluster_gmax_groups) the largest bucket of each
// 16-entry group of the slice, 2 bytes per group.
__host__ __device__ constexpr size_t cluster_base_bytes(int k) {
    return (smem_bytes(k) + sizeof(ClusterExtra) + 15) / 16 * 16;
}
constexpr size_t kClusterSmemMax = 220 * 1024;

// Groups the group-maxima array holds for rows of at most max_len entries:
// enough for a slice of the usual case (at most 32 k entries) when it fits
// next to the rest; rows whose slices need more take the gathered-list path.
int cluster_gmax_groups(int k, int max_len) {
    const long long chunk_max = ((long long)(max_len + kClusterSize - 1) / kClusterSize + 15) / 16 * 16;
    long long want = chunk_max / kVec;
    if (want > 2ll * k) want = 2ll * k;
    want = (want + 7) / 8 * 8;  // whole 16-byte units
    const long long room = ((long long)kClusterSmemMax - (long long)cluster_base_bytes(k)) / 2;
    if (want > room) want = room / 8 * 8;
    return want > 0 ? (int)want : 0;
}

__global__ void __cluster_dims__(kClusterSize, 1, 1) __launch_bounds__(kThreads, 2)
    topk_rows_cluster_kernel(const float *__restrict__ scores, int64_t ld, int row_begin,
                             const int32_t *__restrict__ row_len, int max_len, int k, int32_t *__restrict__ idx,
                             const float *__restrict__ row_stats, const uint32_t *__restrict__ row_keyrange,
                             int n_rows, int gmax_groups) {
    namespace cgs = cooperative_groups;
    cgs::cluster_group cluster = cgs::this_cluster();
    const int rank = (int)cluster.block_rank();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
    int32_t *alist = reinterpret_cast<int32_t *>(smem_raw + sizeof(TopkSmem));
    ClusterExtra &cx = *reinterpret_cast<ClusterExtra *>(smem_raw + smem_bytes(k));

    const int r = blockIdx.x / kClusterSize;
    const int n = row_length(row_len, r, row_begin, max_len);
    const float *row = scores + (size_t)r * ld;
    int32_t *out = idx + (size_t)r * k;
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;

    if (n <= k) {  // short row (same decision on every CTA of the cluster)
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = i < n ? i : -1;
        return;
    }
    const int chunk = ((n + kClusterSize - 1) / kClusterSize + 15) / 16 * 16;
    const int lo = min(n, rank * chunk), m = min(n, lo + chunk) - lo;
    const float *srow = row + lo;
    // start this slice's trip to L2 now: the range lookup below waits on a
    // global load anyway, and the histogram pass then reads from L2
    for (int i0 = tid * kVec; i0 < m; i0 += kChunk)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(srow + i0));

    // ---- value range of the row
    float vmin = INFINITY, vmax = -INFINITY;
    if (row_stats != nullptr) {
        if (tid < 4) {
            vmin = __ldg(row_stats + (size_t)r * 8 + 2 * tid);
            vmax = __ldg(row_stats + (size_t)r * 8 + 2 * tid + 1);
        }
    } else if (row_keyrange != nullptr) {
        // the decode indexer's record: min order key, complemented max key
        if (tid == 0) {
            vmin = key_value(__ldg(row_keyrange + r));
            vmax = key_value(~__ldg(row_keyrange + n_rows + r));
        }
    } else {
        for (int i0 = tid * kVec; i0 < m; i0 += kChunk) {
            float x[kVec];
            const int c = load_vals(srow, i0, m, x);
#pragma unroll
            for (int j = 0; j < kVec; ++j)
                if (j < c) {
                    vmin = fminf(vmin, x[j]);
                    vmax = fmaxf(vmax, x[j]);
                }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        vmin = fminf(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
        vmax = fmaxf(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
    }
    float *fred = reinterpret_cast<float *>(sm.red);
    if (lane == 0) {
        fred[warp] = vmin;
        fred[kWarps + warp] = vmax;
    }
    for (int i = tid; i < kNB; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    if (tid == 0) {
        float a = fred[0], b = fred[kWarps];
        for (int w = 1; w < kWarps; ++w) {
            a = fminf(a, fred[w]);
            b = fmaxf(b, fred[kWarps + w]);
        }
        cx.range[0] = a;
        cx.range[1] = b;
    }
    if (row_stats != nullptr || row_keyrange != nullptr) {
        // every CTA read the same record: nothing to exchange
        __syncthreads();
        vmin = cx.range[0];
        vmax = cx.range[1];
    } else {
        cluster.sync();
        vmin = INFINITY;
        vmax = -INFINITY;
        for (int q = 0; q < kClusterSize; ++q) {
            const float *rr = cluster.map_shared_rank(cx.range, q);
            vmin = fminf(vmin, rr[0]);
            vmax = fmaxf(vmax, rr[1]);
        }
        cluster.sync();  // every remote read of the ranges is done
    }
    if (vmin == vmax) {  // every entry ties: the k lowest indices
        if (rank == 0)
            for (int i = tid; i < k; i += kThreads) out[i] = i;
        return;
    }
    const float range = vmax - vmin;
    if (!(range < INFINITY)) {
        if (rank == 0) topk_row_radix(row, n, k, out, sm);
        return;
    }
    const float scale = __fdiv_rn((float)kNB * 0.99999f, range);

    // ---- histogram of this slice, and the largest bucket of each 16-entry
    // group (for the collect pass to skip groups below the threshold bucket)
    uint32_t *bm = reinterpret_cast<uint32_t *>(alist);  // usual case: this slice's bitmap
    uint16_t *gmax = reinterpret_cast<uint16_t *>(smem_raw + cluster_base_bytes(k));
    const int bm_words = (chunk + 31) / 32;
    // chunk <= 32 k and chunk / 16 groups fit: bitmap and group maxima fit
    const bool small_slice = bm_words <= k && chunk / kVec <= gmax_groups;
    for (int i0 = tid * kVec; i0 < m; i0 += kChunk) {
        float x[kVec];
        const int c = load_vals(srow, i0, m, x);
        uint32_t gm = 0;
#pragma unroll
        for (int j = 0; j < kVec; ++j)
            if (j < c) {
                const uint32_t b = bucket_of(x[j], vmin, scale);
                atomicAdd(&sm.hist[b], 1u);
                gm = max(gm, b);
            }
        if (small_slice) gmax[i0 >> 4] = (uint16_t)gm;  // i0 is a multiple of kVec = 16
    }
    __syncthreads();
    {
        // super-bucket s = buckets 32 s .. 32 s + 31: eight threads' four buckets
        const uint4 h = reinterpret_cast<const uint4 *>(sm.hist)[tid];
        uint32_t v = h.x + h.y + h.z + h.w;
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
        v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
        if ((tid & 7) == 0) cx.coarse[tid >> 3] = v;
    }
    __syncthreads();
    cluster.sync();

    // ---- the row's threshold bucket, in two small exchanges: every slice's
    // super-bucket counts, then every slice's 32 buckets of the super-bucket
    // that holds the k-th entry
    cx.allc[tid / kCoarse][tid % kCoarse] = cluster.map_shared_rank(cx.coarse, tid / kCoarse)[tid % kCoarse];
    __syncthreads();
    if (warp == 0) {
        // lane l holds super-buckets 2l and 2l + 1
        uint32_t c0 = 0, c1 = 0;
#pragma unroll
        for (int q = 0; q < kClusterSize; ++q) {
            c0 += cx.allc[q][2 * lane];
            c1 += cx.allc[q][2 * lane + 1];
        }
        const uint32_t own = c0 + c1;
        uint32_t v = own;  // becomes the sum over lanes >= this one
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, v, o);
            if (lane + o < 32) v += y;
        }
        const uint32_t above = v - own, kk = (uint32_t)k;
        if (above < kk && kk <= above + c1) {
            cx.sel[0] = 2 * lane + 1;
            cx.sel[1] = above;
        } else if (above + c1 < kk && kk <= above + c1 + c0) {
            cx.sel[0] = 2 * lane;
            cx.sel[1] = above + c1;
        }
    }
    __syncthreads();
    const int S = (int)cx.sel[0];
    if (tid < kClusterSize * kFine)
        cx.allf[tid / kFine][tid % kFine] = cluster.map_shared_rank(sm.hist, tid / kFine)[S * kFine + tid % kFine];
    __syncthreads();
    if (warp == 0) {
        uint32_t f = 0;
#pragma unroll
        for (int q = 0; q < kClusterSize; ++q) f += cx.allf[q][lane];
        uint32_t v = f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, v, o);
            if (lane + o < 32) v += y;
        }
        const uint32_t above = cx.sel[1] + (v - f), kk = (uint32_t)k;
        if (above < kk && kk <= above + f) {
            cx.sel[2] = (uint32_t)(S * kFine + lane);
            cx.sel[3] = kk - above;
            cx.sel[4] = above;
            cx.sel[5] = f;
            cx.sel[6] = (uint32_t)lane;
        }
    }
    __syncthreads();
    const uint32_t Bt = cx.sel[2];
    const uint32_t need = cx.sel[3];
    const uint32_t n_above = cx.sel[4];
    const uint32_t cnt = cx.sel[5];
    const int jt = (int)cx.sel[6];
    const int n_groups = (m + kVec - 1) / kVec;
    // usual case (the same decision on every CTA: it depends on the row, not
    // the slice): up to kSmallCand candidates, then the list of groups to
    // revisit in the rest of the candidate arrays
    const bool usual = cnt <= (uint32_t)kSmallCand && small_slice && chunk / kVec <= kCap - kSmallCand;
    if (usual) {
        // every slice's counts follow from the two exchanges
        if (tid < kClusterSize) {
            uint32_t a = 0;
            for (int sb = S + 1; sb < kCoarse; ++sb) a += cx.allc[tid][sb];
            for (int j = jt + 1; j < kFine; ++j) a += cx.allf[tid][j];
            cx.slice_above[tid] = a;
            cx.slice_cand[tid] = cx.allf[tid][jt];
            cx.slice_chosen[tid] = 0;
        }
        if (tid == 0) cx.ncand = 0;
        for (int w = tid; w < bm_words; w += kThreads) bm[w] = 0;
        __syncthreads();
        // No cluster barrier here: no CTA leaves before the barrier after the
        // collect, the histograms read above are not written again, and the
        // candidate lists written by other CTAs are not read before it.
    } else {
        cluster.sync();  // every remote read of the histograms is done (the paths below may leave early)
    }
    if (usual) {
        uint32_t coff = 0;  // this slice's first slot in the row's candidate list
        for (int q = 0; q < rank; ++q) coff += cx.slice_cand[q];
        // the groups holding an entry at or above the threshold bucket (about
        // one in five), listed so that the loads below are one round for the
        // whole CTA instead of one per group a thread owns
        uint32_t *glist = sm.ckey + kSmallCand;
        if (tid == 0) cx.counts[0] = 0;
        __syncthreads();
        for (int g0 = 0; g0 < n_groups; g0 += kThreads) {
            const int g = g0 + tid;
            const bool hit = g < n_groups && gmax[g] >= Bt;
            const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
            uint32_t base = 0;
            if (lane == 0 && bal) base = atomicAdd(&cx.counts[0], (uint32_t)__popc(bal));
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
            if (hit) glist[base + __popc(bal & ((1u << lane) - 1u))] = (uint32_t)g;
        }
        __syncthreads();
        const int n_hit = (int)cx.counts[0];
        for (int gi = tid; gi < n_hit; gi += kThreads) {
            const int i0 = (int)glist[gi] * kVec;
            float x[kVec];
            const int c = load_vals(srow, i0, m, x);
            uint32_t win = 0;
#pragma unroll
            for (int j = 0; j < kVec; ++j) {
                if (j >= c) continue;
                const uint32_t b = bucket_of(x[j], vmin, scale);
                if (b > Bt) {
                    win |= 1u << j;
                } else if (b == Bt) {
                    const uint32_t pos = coff + atomicAdd(&cx.ncand, 1u);
                    const uint32_t key = order_key(x[j]);
                    for (int q = 0; q < kClusterSize; ++q) {
                        cluster.map_shared_rank(sm.ckey, q)[pos] = key;
                        cluster.map_shared_rank(sm.cidx, q)[pos] = lo + i0 + j;
                    }
                }
            }
            // i0 is a multiple of kVec = 16: the group is one half of a word
            if (win) atomicOr(&bm[i0 >> 5], win << (i0 & 31));
        }
        __syncthreads();
        cluster.sync();  // every CTA holds the row's cnt candidates; no remote access follows

        if (tid < (int)cnt) {
            const uint32_t ki = sm.ckey[tid];
            const int32_t xi = sm.cidx[tid];
            uint32_t rk = 0;
            for (int j = 0; j < (int)cnt; ++j) {
                const uint32_t kj = sm.ckey[j];
                rk += (kj > ki) || (kj == ki && sm.cidx[j] < xi);
            }
            if (rk < need) {
                const int q = xi / chunk;
                atomicAdd(&cx.slice_chosen[q], 1u);
                if (q == rank) atomicOr(&bm[(xi - lo) >> 5], 1u << ((xi - lo) & 31));
            }
        }
        __syncthreads();
        uint32_t off = 0;  // this slice's first output position
        for (int q = 0; q < rank; ++q) off += cx.slice_above[q] + cx.slice_chosen[q];
        const int words = (m + 31) / 32;
        const int per = (words + kThreads - 1) / kThreads;
        const int w0 = min(words, tid * per), w1 = min(words, w0 + per);
        uint32_t mine = 0;
        for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
        uint32_t tot;
        uint32_t pos = off + block_scan_packed(mine, sm.red, &tot);
        for (int w = w0; w < w1; ++w) {
            uint32_t v = bm[w];
            while (v) {
                const int b = __ffs(v) - 1;
                v &= v - 1u;
                out[pos++] = lo + w * 32 + b;
            }
        }
        return;
    }
    if (cnt > (uint32_t)kCap) {
        if (rank == 0) topk_row_radix(row, n, k, out, sm);
        return;
    }

    // ---- ordered collect of this slice
    uint32_t run_a = 0, run_c = 0;
    for (int base = 0; base < m; base += kChunk) {
        const int i0 = base + tid * kVec;
        float x[kVec] = {};
        const int c = i0 < m ? load_vals(srow, i0, m, x) : 0;
        uint32_t cls[kVec];
        uint32_t na = 0, nc = 0;
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const uint32_t b = bucket_of(x[j], vmin, scale);
            cls[j] = j >= c ? 0u : (b > Bt ? 2u : (b == Bt ? 1u : 0u));
            na += cls[j] == 2u;
            nc += cls[j] == 1u;
        }
        uint32_t tot;
        const uint32_t ex = block_scan_packed(na | (nc << 16), sm.red, &tot);
        uint32_t pa = run_a + (ex & 0xFFFFu), pc = run_c + (ex >> 16);
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            if (cls[j] == 2u) alist[pa++] = lo + i0 + j;
            if (cls[j] == 1u) {
                sm.ckey[pc] = order_key(x[j]);
                sm.cidx[pc] = lo + i0 + j;
                ++pc;
            }
        }
        run_a += tot & 0xFFFFu;
        run_c += tot >> 16;
    }
    if (tid == 0) {
        cx.counts[0] = run_a;
        cx.counts[1] = run_c;
    }
    __syncthreads();
    cluster.sync();

    // ---- rank 0 appends the other slices' lists (in rank = index order)
    if (rank == 0) {
        uint32_t off_a = run_a, off_c = run_c;
        for (int q = 1; q < kClusterSize; ++q) {
            const uint32_t *qc = cluster.map_shared_rank(cx.counts, q);
            const uint32_t qa = qc[0], qn = qc[1];
            const int32_t *qal = reinterpret_cast<const int32_t *>(
                reinterpret_cast<const uint8_t *>(cluster.map_shared_rank(&sm, q)) + sizeof(TopkSmem));
            const TopkSmem *qs = cluster.map_shared_rank(&sm, q);
            for (uint32_t i = tid; i < qa; i += kThreads) alist[off_a + i] = qal[i];
            for (uint32_t i = tid; i < qn; i += kThreads) {
                sm.ckey[off_c + i] = qs->ckey[i];
                sm.cidx[off_c + i] = qs->cidx[i];
            }
            off_a += qa;
            off_c += qn;
        }
        __syncthreads();
    }
    cluster.sync();  // rank 0 has read every remote list
    if (rank != 0) return;
    finish_row(sm, alist, cnt, need, n_above, out);
}

}  // namespace

size_t topk_workspace_bytes(int, int, int) { return 0; }

cudaError_t launch_topk(const float *scores, int64_t ld, int row_begin, int n_rows, const int32_t *row_len,
                        int max_len, int k, int32_t *idx, const float *row_stats, void *, size_t,
                        cudaStream_t stream, const uint32_t *row_keyrange) {
    if (n_rows == 0) return cudaSuccess;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (max_len >= 16384 && n_rows < (sms > 0 ? sms : 148)) {
        // few long rows: a cluster of CTAs per row keeps every SM busy
        const int gmax_groups = cluster_gmax_groups(k, max_len);
        const size_t csmem = cluster_base_bytes(k) + (size_t)gmax_groups * 2;
        if (csmem > kClusterSmemMax) return cudaErrorInvalidValue;
        cudaError_t e = set_smem_at_least<topk_rows_cluster_kernel>(csmem);
        if (e != cudaSuccess) return e;
        topk_rows_cluster_kernel<<<n_rows * kClusterSize, kThreads, csmem, stream>>>(
            scores, ld, row_begin, row_len, max_len, k, idx, row_stats, row_keyrange, n_rows, gmax_groups);
        return cudaGetLastError();
    }
    if (bitmap_smem_bytes(max_len) <= (size_t)kBitmapSmemMax) {
        const size_t bsmem = bitmap_smem_bytes(max_len);
        cudaError_t e = set_smem_at_least<topk_rows_bitmap_kernel>(bsmem);
        if (e != cudaSuccess) return e;
        topk_rows_bitmap_kernel<<<n_rows, kThreads, bsmem, stream>>>(scores, ld, row_begin, row_len, max_len, k, idx,
                                                                     row_stats);
        return cudaGetLastError();
    }
    const size_t smem = smem_bytes(k);
    if (smem > 220 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = set_smem_at_least<topk_rows_kernel>(smem);
    if (e != cudaSuccess) return e;
    topk_rows_kernel<<<n_rows, kThreads, smem, stream>>>(scores, ld, row_begin, row_len, max_len, k, idx,
                                                         row_stats);
    return cudaGetLastError();
}

bool topk_k_supported(int k) { return cluster_base_bytes(k) <= kClusterSmemMax; }

}  // namespace dsa
