// indexer_tc.cu -- prefill lightning indexer on the 5th-generation tensor
// cores (tcgen05, FP8 e4m3 x e4m3 -> fp32 in TMEM), fed by TMA.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式, indexer:
//     I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s]),  s <= t
// one key head shared by every indexer head, FP8 (report translation,
// section 2.3.1).  With positive per-token scales,
//     I[t,s] = sq[t] * sk[s] * sum_j w[t,j] * ReLU(q8[t,j] . k8[s]).
//
// GEMM view: A = 128 keys x dI (K-major, TMA tile), B = NQ queries x HI heads
// = 128 rows x dI (K-major, one query block), D = 128 x 128 fp32 in TMEM
// (lane = key, column = (query, head)).  Keys on M means one epilogue thread
// owns one key and reduces over heads inside its own registers.
//
// Warp roles (one CTA per SM, persistent over query blocks):
//   producer    TMA: the query block (double-buffered) and a ring of key
//               tiles (kStages deep);
//   MMA         allocates 512 TMEM columns (four 128-column accumulators)
//               and issues the UMMAs (dI/32 per tile), committing to
//               mbarriers;
//   epilogue    4 x (128 / CW) warps: warp w reads TMEM lanes 32*(w%4).. and
//               the CW = max(32, HI) columns of one query (or 32/HI whole
//               queries) with 32x32b loads, so each thread holds one key and
//               its query's head weights live in registers for the whole
//               query block: ReLU, weighted head sum (packed f32x2 FMA), the
//               two scales and the causal mask, then a coalesced store.
// An accumulator is handed back as soon as its last tcgen05.ld completes; with
// four of them the UMMAs run up to three tiles ahead of the epilogue.
//
// Every mbarrier wait is bounded (globaltimer); on timeout the kernel sets
// an error flag, every role unwinds, and TMEM is freed before exit.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_util.cuh"

namespace dsa {

__device__ unsigned int g_indexer_tc_error;
// Bound of the prefill indexer's pipeline waits (between its TMA, MMA and
// epilogue roles), in ns.  The default is far above any legitimate wait; a
// test lowers it to make the waits give up and exercise the unwinding.  The
// waits that drain copies in flight and the final MMA completion keep their
// own fixed bounds.
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

namespace {

// Pipeline waits with the bound above.  The bound is read only once a wait
// has to spin (the barrier was not already complete), so it occupies no
// register in the common case.
__device__ __forceinline__ uint64_t pipe_wait_limit() {
    return *const_cast<const volatile unsigned long long *>(&g_wait_limit_ns);
}

__device__ __forceinline__ bool pipe_wait(uint32_t bar, uint32_t parity) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    return tc::mbar_wait(bar, parity, pipe_wait_limit());
}

__device__ __forceinline__ bool pipe_wait_sleep(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    return tc::mbar_wait_sleep(bar, parity, pipe_wait_limit(), sleep_ns);
}

}  // namespace

namespace {

constexpr int kTileM = 128;     // keys per MMA (UMMA M)
constexpr int kTileN = 128;     // (query, head) columns per tile
constexpr int kStepKeys = 256;  // keys per pipeline step: two MMA tiles
constexpr int kAccBufs = 4;     // TMEM accumulators (4 x 128 = 512 columns) ...
constexpr int kPairs = kAccBufs / 2;  // ... used in pairs, one pair per step
constexpr uint32_t kTmemCols = 512;

// With dI = 64 a tile needs only two MMAs, so the single MMA thread's fixed
// cost per step (barrier waits, fences, commits) sets the pace; a step of two
// tiles (one 256-row TMA box, 2 x dI/32 MMAs into an accumulator pair, one
// commit) halves that cost per MMA.

// Columns per epilogue warp and the warp counts for HI heads per query.  Two
// MMA warps take alternate steps, each into its own accumulator pair: the
// fixed cost of one issuing thread per step (two mbarrier waits, fences, two
// commits: about 900 cycles) is what paced a single MMA warp, and two of them
// overlap it.  With 19 warps, three of the four schedulers hold five warps,
// whose 16K-register files cap a thread at 96 registers (HI <= 32); HI = 64
// has 11 warps.
template <int HI>
struct EpiShape {
    static constexpr int CW = HI > 32 ? HI : 32;
    static constexpr int kEpiWarps = 4 * (kTileN / CW);
    static constexpr int kThreads = (kEpiWarps + 3) * 32;
    static constexpr int kProducerWarp = kEpiWarps;
    static constexpr int kMmaWarp = kEpiWarps + 1;  // and kMmaWarp + 1
    static constexpr int kMaxRegs = kThreads > 512 ? 96 : 168;
};
// The sampled mode scores every 32nd key (the threshold pre-pass of the
// fused indexer + top-k).
constexpr int kSampleStride = 32;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr uint32_t kIssuerSleepNs = 32;            // back-off of the TMA and MMA warps


template <int DI>
struct Layout {
    static constexpr int kTileBytes = kStepKeys * DI;  // one step of keys
    // even: stage s then serves steps of one parity only, i.e. of one MMA
    // warp, which waits for its phases in order
    static constexpr int kStages = ((200 * 1024 - 2 * kTileN * DI) / kTileBytes > 8
                                        ? 8
                                        : (200 * 1024 - 2 * kTileN * DI) / kTileBytes) & ~1;
    static constexpr int kQBytes = kTileN * DI;
    static constexpr int kKeys = 0;
    static constexpr int kQ = kKeys + kStages * kTileBytes;
    static constexpr int kBars = kQ + 2 * kQBytes;              // uint64 barriers
    static constexpr int kNumBars = 2 * kStages + 4 + 2 * kPairs + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kBytes = kTmemSlot + 16;
    static constexpr int kAlloc = kBytes + 1024;                // slack for 1024-byte alignment
};

__device__ __forceinline__ void record_timeout() { atomicOr(&g_indexer_tc_error, 1u); }

// What the epilogue does with a score.
enum IndexerMode : int {
    kModeScores = 0,   // store every causal score (and optionally each row's range)
    kModeSample = 1,   // the same over every kSampleStride-th key only (sampled scores)
    kModeCand = 2,     // keep only scores >= the row's threshold, as (index, score) pairs
};

// Outputs of one launch.  Scores modes: scores [n_rows, ld] (row r = query
// row_begin + r; in the sampled mode column j is key j * kSampleStride) and
// optional row_stats [n_rows, 8].  Candidate mode: tau [n_rows] (the row's
// threshold), cand [n_rows, 4, seg_cap] (index, score) pairs, one segment per
// TMEM lane quarter, in ascending key order within a segment, and
// cand_count [n_rows, 4] (the number of entries each segment would hold;
// entries past seg_cap are dropped).  With packed sequences every key index
// and output column is relative to the start of the query's sequence.
struct EpiArgs {
    float *scores;
    int64_t ld;
    float *row_stats;
    const float *tau;
    int2 *cand;
    int *cand_count;
    int seg_cap;
    // packed sequences (VARLEN): query t sees the keys [start(t), t] of its
    // own sequence, start(t) from cu [nseq + 1]; output columns and
    // candidate indices are positions relative to start(t)
    const int32_t *cu;
    int nseq;
};

template <int HI, int DI, int MODE, bool VARLEN>
__global__ void __maxnreg__(EpiShape<HI>::kMaxRegs) indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                                 const __grid_constant__ CUtensorMap tmap_q,
                                                                 const float *__restrict__ sq,
                                                                 const float *__restrict__ w,
                                                                 const float *__restrict__ sk, int row_begin,
                                                                 int n_rows, const EpiArgs args) {
    using Lay = Layout<DI>;
    using ES = EpiShape<HI>;
    constexpr int kEpiWarps = ES::kEpiWarps, kProducerWarp = ES::kProducerWarp, kMmaWarp = ES::kMmaWarp;
    constexpr int CW = ES::CW;          // columns per epilogue warp
    constexpr int NQ = kTileN / HI;     // queries per block
    constexpr int QPW = CW / HI;        // whole queries per epilogue warp (1 when HI >= 32)
    constexpr int KSTEPS = DI / 32;
    constexpr int kStages = Lay::kStages;
    constexpr uint32_t IDESC = tc::idesc_e4m3_f32(kTileM, kTileN);
    // key j of the key tensor map is token j * KS; query t sees keys j <= t / KS
    constexpr int KS = MODE == kModeSample ? kSampleStride : 1;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bars = sbase + Lay::kBars;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kStages + s); };
    auto qfull_bar = [&](int b) { return bars + 8u * (2 * kStages + b); };
    auto qempty_bar = [&](int b) { return bars + 8u * (2 * kStages + 2 + b); };
    auto tfull_bar = [&](int b) { return bars + 8u * (2 * kStages + 4 + b); };
    auto tempty_bar = [&](int b) { return bars + 8u * (2 * kStages + 4 + kPairs + b); };
    const uint32_t mma_done_bar = bars + 8u * (2 * kStages + 4 + 2 * kPairs);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + Lay::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int row_end = row_begin + n_rows;
    const int nb = (n_rows + NQ - 1) / NQ;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(full_bar(s), 1);
            tc::mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(qfull_bar(b), 1);
            tc::mbar_init(qempty_bar(b), 2);  // one commit per MMA warp
        }
        for (int b = 0; b < kPairs; ++b) {
            tc::mbar_init(tfull_bar(b), 1);
            tc::mbar_init(tempty_bar(b), kEpiWarps);
        }
        tc::mbar_init(mma_done_bar, 2);
        tc::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tc::tmem_alloc(sbase + Lay::kTmemSlot, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tc::tma_prefetch_desc(&tmap_k);
        tc::tma_prefetch_desc(&tmap_q);
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int bi = 0, n_issued = 0, q_issued = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < nb && ok; i += gridDim.x, ++bi) {
                const int qb = nb - 1 - i;
                const int t0 = row_begin + qb * NQ;
                const int t_hi = min(t0 + NQ, row_end) - 1;
                const int nstep = (t_hi / KS) / kStepKeys + 1;
                const int st_lo = VARLEN ? ((seq_start(args.cu, args.nseq, t0) + KS - 1) / KS) / kStepKeys : 0;
                const int qs = bi & 1;
                if (!pipe_wait_sleep(qempty_bar(qs), ((bi >> 1) & 1) ^ 1, kIssuerSleepNs)) {
                    ok = false;
                    break;
                }
                tc::mbar_arrive_expect_tx(qfull_bar(qs), Lay::kQBytes);
                tc::tma_load_2d(sbase + Lay::kQ + qs * Lay::kQBytes, &tmap_q, 0, t0 * HI, qfull_bar(qs));
                ++q_issued;
                for (int st = st_lo; st < nstep; ++st) {
                    if (!pipe_wait_sleep(empty_bar(stage), phase ^ 1, kIssuerSleepNs)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(full_bar(stage), Lay::kTileBytes);
                    tc::tma_load_2d(sbase + Lay::kKeys + stage * Lay::kTileBytes, &tmap_k, 0, st * kStepKeys,
                                    full_bar(stage));
                    ++n_issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) record_timeout();
            // Drain: every issued copy has landed before the CTA may exit
            // (load j used stage j % kStages in its (j / kStages)-th phase).
            const uint64_t lim = ok ? kWaitLimitNs : 100000000ull;
            for (int j = max(0, n_issued - kStages); j < n_issued; ++j)
                (void)tc::mbar_wait(full_bar(j % kStages), (uint32_t)((j / kStages) & 1), lim);
            for (int j = max(0, q_issued - 2); j < q_issued; ++j)
                (void)tc::mbar_wait(qfull_bar(j & 1), (uint32_t)((j >> 1) & 1), lim);
        }
    } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
        // ------------------------------------------------------------ UMMA
        // MMA warp mw issues the steps it with it % 2 == mw, into pair mw.
        // Both warps walk every query block and wait for its query tile, so
        // each waits for every barrier phase it uses in order.
        static_assert(kPairs == 2, "one accumulator pair per MMA warp");
        const int mw = warp - kMmaWarp;
        if (lane == 0) {
            int it = 0, bi = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < nb && ok; i += gridDim.x, ++bi) {
                const int qb = nb - 1 - i;
                const int t0 = row_begin + qb * NQ;
                const int t_hi = min(t0 + NQ, row_end) - 1;
                const int nstep = (t_hi / KS) / kStepKeys + 1;
                const int st_lo = VARLEN ? ((seq_start(args.cu, args.nseq, t0) + KS - 1) / KS) / kStepKeys : 0;
                const int qs = bi & 1;
                if (!pipe_wait_sleep(qfull_bar(qs), (bi >> 1) & 1, kIssuerSleepNs)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t qaddr = sbase + Lay::kQ + qs * Lay::kQBytes;
                for (int st = st_lo; st < nstep; ++st, ++it) {
                    if ((it & 1) != mw) continue;
                    const int pr = mw;
                    const int stage = it % kStages;
                    if (!pipe_wait_sleep(tempty_bar(pr), ((it / kPairs) & 1) ^ 1, kIssuerSleepNs) ||
                        !pipe_wait_sleep(full_bar(stage), (it / kStages) & 1, kIssuerSleepNs)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t kaddr = sbase + Lay::kKeys + stage * Lay::kTileBytes;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {  // keys 0..127 and 128..255 of the step
                        const uint32_t d = tmem_base + (uint32_t)((2 * pr + h) * kTileN);
                        const uint32_t ka = kaddr + (uint32_t)(h * kTileM * DI);
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks) {
                            tc::umma_f8(d, tc::smem_desc_kmajor(ka + ks * 32, DI),
                                        tc::smem_desc_kmajor(qaddr + ks * 32, DI), IDESC, ks > 0 ? 1u : 0u);
                        }
                    }
                    tc::umma_commit(empty_bar(stage));
                    tc::umma_commit(tfull_bar(pr));
                }
                tc::umma_commit(qempty_bar(qs));
            }
            if (!ok) record_timeout();
            // every UMMA issued above has completed before TMEM is freed
            tc::umma_commit(mma_done_bar);
            (void)tc::mbar_wait(mma_done_bar, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        // Thread = one key of the tile (lane quarter qw), CW columns = QPW
        // whole queries.  The TMEM reads, the ReLU + head sum and the score
        // stores (or the candidate ballot) each cost about as much at 128K;
        // the MMA/TMA pipeline alone runs about 2.4x faster than the whole.
        const int qw = warp & 3;          // TMEM lane quarter: keys 32*qw ..
        const int cg = warp >> 2;         // column group: columns cg*CW ..
        const uint32_t lane_base = tmem_base + ((uint32_t)(qw * 32) << 16);
        int it = 0;
        bool ok = true;
        for (int i = blockIdx.x; i < nb && ok; i += gridDim.x) {
            const int qb = nb - 1 - i;
            const int t0 = row_begin + qb * NQ;
            const int t_hi = min(t0 + NQ, row_end) - 1;
            const int nstep = (t_hi / KS) / kStepKeys + 1;
            const int st_lo = VARLEN ? ((seq_start(args.cu, args.nseq, t0) + KS - 1) / KS) / kStepKeys : 0;
            // this warp's query head weights, in registers for the whole block
            float2 wv[CW / 2];
#pragma unroll
            for (int c = 0; c < CW; c += 2) {
                const int t = t0 + (cg * CW + c) / HI;
                wv[c / 2] = t <= t_hi ? __ldg(reinterpret_cast<const float2 *>(w + (size_t)t0 * HI + cg * CW + c))
                                      : make_float2(0.f, 0.f);
            }
            float sqv[QPW], vlo[QPW], vhi[QPW], tau[QPW];
            int cnt[QPW], jlo[QPW];  // jlo: first visible key (key-map units) of each query
#pragma unroll
            for (int q = 0; q < QPW; ++q) {
                const int t = t0 + (cg * CW) / HI + q;
                jlo[q] = VARLEN && t <= t_hi ? (seq_start(args.cu, args.nseq, t) + KS - 1) / KS : 0;
                sqv[q] = t <= t_hi ? __ldg(sq + t) : 0.f;
                vlo[q] = INFINITY;
                vhi[q] = -INFINITY;
                cnt[q] = 0;
                if constexpr (MODE == kModeCand) tau[q] = t <= t_hi ? __ldg(args.tau + (t - row_begin)) : INFINITY;
                else tau[q] = 0.f;
            }
            for (int st = st_lo; st < nstep; ++st, ++it) {
                const int pr = it % kPairs;
                if (!pipe_wait(tfull_bar(pr), (it / kPairs) & 1)) { ok = false; break; }
                tc::tc_fence_after();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int buf = 2 * pr + h;
                    const int s = st * kStepKeys + h * kTileM + qw * 32 + lane;  // key index (token s * KS)
                    const float sks = s * KS <= t_hi ? __ldg(sk + (size_t)s * KS) : 0.f;
                    float2 part[QPW][2];
#pragma unroll
                    for (int q = 0; q < QPW; ++q) part[q][0] = part[q][1] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int c = 0; c < CW / 32; ++c) {
                        float acc[32];
                        tc::tmem_ld32(lane_base + (uint32_t)(buf * kTileN + cg * CW + c * 32), acc);
                        tc::tmem_wait_ld();
                        if (h == 1 && c == CW / 32 - 1) {  // the pair is read: hand it back before the math
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(tempty_bar(pr));
                        }
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const int col = c * 32 + j;              // within this warp's CW columns
                            const int q = col / HI;                  // compile-time after unrolling
                            const int chain = (j >> 2) & 1;
                            part[q][chain] = tc::ffma2(wv[col / 2],
                                                       make_float2(fmaxf(acc[j], 0.f), fmaxf(acc[j + 1], 0.f)),
                                                       part[q][chain]);
                            part[q][chain] = tc::ffma2(wv[col / 2 + 1],
                                                       make_float2(fmaxf(acc[j + 2], 0.f), fmaxf(acc[j + 3], 0.f)),
                                                       part[q][chain]);
                        }
                    }
#pragma unroll
                    for (int q = 0; q < QPW; ++q) {
                        const int t = t0 + (cg * CW) / HI + q;
                        const bool vis = t <= t_hi && s * KS <= t && (!VARLEN || s >= jlo[q]);
                        if constexpr (MODE == kModeCand) {
                            // keep the scores at or above the row's threshold: warp-aggregated
                            // slots in this warp's own segment of the row (keys in ascending order)
                            const float v = (part[q][0].x + part[q][1].x) + (part[q][0].y + part[q][1].y);
                            const float score = v * sqv[q] * sks;
                            const bool keep = vis && score >= tau[q];
                            const uint32_t b = __ballot_sync(0xFFFFFFFFu, keep);
                            if (b != 0u) {
                                const int pos = cnt[q] + __popc(b & ((1u << lane) - 1u));
                                if (keep && pos < args.seg_cap)
                                    args.cand[((size_t)(t - row_begin) * 4 + qw) * args.seg_cap + pos] =
                                        make_int2(s - jlo[q], __float_as_int(score));
                                cnt[q] += __popc(b);
                            }
                        } else if (vis) {
                            const float v = (part[q][0].x + part[q][1].x) + (part[q][0].y + part[q][1].y);
                            const float score = v * sqv[q] * sks;
                            args.scores[(size_t)(t - row_begin) * args.ld + (s - jlo[q])] = score;
                            if constexpr (MODE == kModeScores) {
                                vlo[q] = fminf(vlo[q], score);
                                vhi[q] = fmaxf(vhi[q], score);
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            if constexpr (MODE == kModeCand) {
#pragma unroll
                for (int q = 0; q < QPW; ++q) {
                    const int t = t0 + (cg * CW) / HI + q;
                    if (lane == 0 && t <= t_hi) args.cand_count[(size_t)(t - row_begin) * 4 + qw] = cnt[q];
                }
            } else if (MODE == kModeScores && args.row_stats != nullptr) {
                // per-(row, lane quarter) range of the scores just written
#pragma unroll
                for (int q = 0; q < QPW; ++q) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        vlo[q] = fminf(vlo[q], __shfl_xor_sync(0xFFFFFFFFu, vlo[q], o));
                        vhi[q] = fmaxf(vhi[q], __shfl_xor_sync(0xFFFFFFFFu, vhi[q], o));
                    }
                    const int t = t0 + (cg * CW) / HI + q;
                    if (lane == 0 && t <= t_hi) {
                        float *st8 = args.row_stats + (size_t)(t - row_begin) * 8;
                        st8[2 * qw] = vlo[q];
                        st8[2 * qw + 1] = vhi[q];
                    }
                }
            }
        }
        if (!ok) record_timeout();
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ===========================================================================
// Decode: one query token per sequence against its paged cache ("Kwai
// Keye-VL-2.0 Technical Report" review, DSA decode, section 5.3).
//
// GEMM view: A = 128 cached keys, i.e. two 64-token pages (K-major rows of
// dI bytes, one TMA box per page), B = the sequence's HI indexer heads padded
// to N = max(16, HI) rows, D = 128 x N fp32 in TMEM (lane = key, column =
// head).  A step is up to SP pages of one sequence (SP = 8 for dI <= 64, 4 for
// dI = 128): SP/2 such tiles into SP/2 accumulators.  A sequence of n tokens
// has ceil(n / (64 SP)) steps; the steps of the whole batch are numbered
// through a prefix sum over the sequences and split into equal contiguous
// ranges, one per CTA, so long and short sequences share the SMs evenly.
//
// Warp roles (one CTA per SM):
//   producers  four warps share every step: warp p issues the TMA boxes of
//              pages 2p and 2p+1 (SP = 8) plus bulk copies of their 64 key
//              scales.  One thread issuing bulk copies moves about a third of
//              what the SM's HBM share needs; four of them reach it.  Each
//              warp looks up the page ids of 32 consecutive steps at a time.
//              The first producer also writes the step's 16-byte record
//              (sequence, step, length, page validity) and copies each
//              sequence's query rows, in sequence order, into one of two
//              swizzled query slots;
//   MMA        two warps take alternate steps, (SP/2) x (dI/32) UMMAs per
//              step into an (SP/2) x N column accumulator.  One thread's
//              cost per step (barrier waits, fences, eight UMMAs and two
//              commits: about 0.7 us) was most of the step period with one
//              MMA warp; two overlap it;
//   epilogue   kDecGroups groups of four warps take alternate steps: per tile
//              each thread owns one key, reads its N columns, ReLU and the
//              head-weighted sum, the two scales, and stores one score.
// A stage is refilled once its UMMAs completed and the epilogue group read
// its scales and record (five arrivals).
// ===========================================================================

constexpr int kDecMaxB = 4096;     // sequences whose step prefix fits in shared memory
constexpr int kDecPage = 64;       // tokens per cache page
constexpr int kDecGroups = 2;
constexpr int kDecProducers = 4;
constexpr int kDecProducer0 = 4 * kDecGroups;         // warps 0 .. 4G-1: epilogue
constexpr int kDecMmaWarp = kDecProducer0 + kDecProducers;  // two MMA warps: kDecMmaWarp, kDecMmaWarp + 1
constexpr int kDecThreads = (kDecMmaWarp + 2) * 32;
// 14 warps leave four on one scheduler, whose 16K registers cap a thread at 128.
constexpr int kDecMaxRegs = 128;

template <int N, int DI>
struct DecLayout {
    static constexpr int SP = DI > 64 ? 4 : 8;                   // pages per step
    static constexpr int kTiles = SP / 2;                        // 128-key MMA tiles per step
    static constexpr int kKeyBytes = SP * kDecPage * DI;
    static constexpr int kScales = kKeyBytes;                    // SP * 64 floats
    static constexpr int kMeta = kScales + SP * kDecPage * 4;    // int4 record
    static constexpr int kStageBytes = (kMeta + 16 + 1023) / 1024 * 1024;
    static constexpr int kQBytes = (N * DI + 1023) / 1024 * 1024;
    static constexpr int kPrefixBytes = ((kDecMaxB + 1) * 4 + 15) / 16 * 16;
    static constexpr int kFixed = 2 * kQBytes + kPrefixBytes + 1024;
    static constexpr int kStages = (212 * 1024 - kFixed) / kStageBytes;
    static constexpr int kAccCols = kTiles * N;                  // TMEM columns per step
    static constexpr int kAccBufs = 512 / kAccCols > 8 ? 8 : 512 / kAccCols;
    static constexpr int kQ = kStages * kStageBytes;
    static constexpr int kPrefix = kQ + 2 * kQBytes;
    static constexpr int kBars = kPrefix + kPrefixBytes;
    static constexpr int kNumBars = 2 * kStages + 4 + 2 * kAccBufs + 1;
    static constexpr int kTmemSlot = kBars + kNumBars * 8;
    static constexpr int kBytes = kTmemSlot + 16;
    static constexpr int kAlloc = kBytes + 1024;
    static_assert(SP == 2 * kDecProducers || SP == kDecProducers, "pages per producer");
    static_assert(kStages >= 4, "decode indexer ring too shallow");
    static_assert(kAccBufs % kDecGroups == 0, "an accumulator serves one epilogue group");
    static_assert(kAlloc <= 227 * 1024, "decode indexer shared memory");
};

// In-place inclusive prefix sum of a[0..n) by the whole block; `scratch`
// holds blockDim.x ints.
__device__ void block_inclusive_scan(int *a, int n, int *scratch) {
    const int T = blockDim.x, t = threadIdx.x;
    const int chunk = (n + T - 1) / T;
    const int lo = min(n, t * chunk), hi = min(n, lo + chunk);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += a[i];
    scratch[t] = sum;
    __syncthreads();
    if (t < 32) {
        int carry = 0;
        for (int base = 0; base < T; base += 32) {
            const int v = base + t < T ? scratch[base + t] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (t >= o) incl += u;
            }
            if (base + t < T) scratch[base + t] = carry + incl - v;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
    }
    __syncthreads();
    int run = scratch[t];
    for (int i = lo; i < hi; ++i) {
        run += a[i];
        a[i] = run;
    }
    __syncthreads();
}

template <int N, int DI>
__global__ void __maxnreg__(kDecMaxRegs) indexer_decode_tc_kernel(
    const __grid_constant__ CUtensorMap tmap_k, const uint8_t *__restrict__ q8, const float *__restrict__ sq,
    const float *__restrict__ w, const float *__restrict__ skc, const int32_t *__restrict__ block_table,
    int max_pages, int num_pages, const int32_t *__restrict__ seq_lens, int max_seq_len, int B, int HI,
    float *__restrict__ scores, int64_t ld, uint32_t *__restrict__ keyrange) {
    using Lay = DecLayout<N, DI>;
    constexpr int S = Lay::kStages, A = Lay::kAccBufs, G = kDecGroups;
    constexpr int SP = Lay::SP, T = Lay::kTiles, PPW = SP / kDecProducers;  // pages per producer warp
    constexpr int KSTEPS = DI / 32;
    constexpr int CPR = DI / 16;  // 16-byte chunks per key or query row
    constexpr uint32_t IDESC = tc::idesc_e4m3_f32(2 * kDecPage, N);
    constexpr uint32_t kPageTx = kDecPage * DI + kDecPage * 4;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    int *prefix = reinterpret_cast<int *>(smem + Lay::kPrefix);
    const uint32_t bars = sbase + Lay::kBars;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
    auto qfull_bar = [&](int q) { return bars + 8u * (2 * S + q); };
    auto qempty_bar = [&](int q) { return bars + 8u * (2 * S + 2 + q); };
    auto tfull_bar = [&](int a) { return bars + 8u * (2 * S + 4 + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (2 * S + 4 + A + a); };
    const uint32_t mma_done_bar = bars + 8u * (2 * S + 4 + 2 * A);
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + Lay::kTmemSlot);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int cap = min(max_seq_len, max_pages * kDecPage);
    auto seq_len_of = [&](int b) { return min(max(__ldg(seq_lens + b), 0), cap); };

    // steps per sequence, then their prefix: prefix[b] = first step of b
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int pages = (seq_len_of(b) + kDecPage - 1) / kDecPage;
        prefix[b + 1] = (pages + SP - 1) / SP;
    }
    if (threadIdx.x == 0) {
        prefix[0] = 0;
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(full_bar(s), kDecProducers);
            tc::mbar_init(empty_bar(s), 1 + 4);
        }
        for (int q = 0; q < 2; ++q) {
            tc::mbar_init(qfull_bar(q), 1);
            tc::mbar_init(qempty_bar(q), 2);  // one release per MMA warp
        }
        for (int a = 0; a < A; ++a) {
            tc::mbar_init(tfull_bar(a), 1);
            tc::mbar_init(tempty_bar(a), 4);
        }
        tc::mbar_init(mma_done_bar, 2);
        tc::fence_mbar_init();
    }
    if (warp == kDecMmaWarp) {
        tc::tmem_alloc(sbase + Lay::kTmemSlot, kTmemCols);
        tc::tmem_relinquish();
    }
    if (warp >= kDecProducer0 && warp < kDecMmaWarp && lane == 0) tc::tma_prefetch_desc(&tmap_k);
    __syncthreads();
    block_inclusive_scan(prefix + 1, B, reinterpret_cast<int *>(smem));  // scratch: stage 0, not yet in use
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = prefix[B];
    const int i0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
    const int i1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
    const int nsteps = i1 - i0;

    if (warp >= kDecProducer0 && warp < kDecMmaWarp) {
        // ------------------------------------------------------------ producers
        const int pw = warp - kDecProducer0;
        bool ok = true;
        int carry = 0;     // sequence starts in earlier batches
        int n_issued = 0;  // steps this warp has arrived on
        for (int base = 0; base < nsteps && ok; base += 32) {
            int my_b = 0, my_st = 0, my_n = 0, my_np = 0;
            int my_pg[SP];  // every page of the step: the first warp records their validity
#pragma unroll
            for (int k = 0; k < SP; ++k) my_pg[k] = 0;
            const bool valid = base + lane < nsteps;
            if (valid) {
                const int gi = i0 + base + lane;
                int lo = 0, hi = B;  // prefix[lo] <= gi < prefix[hi]
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (prefix[mid] <= gi) lo = mid;
                    else hi = mid;
                }
                my_b = lo;
                my_st = gi - prefix[lo];
                my_n = seq_len_of(lo);
                const int pages = (my_n + kDecPage - 1) / kDecPage;
                my_np = min(SP, pages - SP * my_st);
                const int32_t *bt = block_table + (size_t)lo * max_pages + SP * my_st;
#pragma unroll
                for (int k = 0; k < SP; ++k)
                    if (k < my_np) my_pg[k] = __ldg(bt + k);
            }
            // steps that begin a sequence (or the range) take the next query slot
            const unsigned starts = __ballot_sync(0xFFFFFFFFu, valid && (my_st == 0 || base + lane == 0));
            const int cnt = min(32, nsteps - base);
            for (int j = 0; j < cnt; ++j) {
                const int b = __shfl_sync(0xFFFFFFFFu, my_b, j);
                const int st = __shfl_sync(0xFFFFFFFFu, my_st, j);
                const int n = __shfl_sync(0xFFFFFFFFu, my_n, j);
                const int np = __shfl_sync(0xFFFFFFFFu, my_np, j);
                int flags = 0;  // bit i: page i of the step maps a cache page
                int pg[PPW];
#pragma unroll
                for (int k = 0; k < SP; ++k) {
                    const int p = __shfl_sync(0xFFFFFFFFu, my_pg[k], j);
                    if (k < np && p >= 0 && p < num_pages) flags |= 1 << k;
                    if (k / PPW == pw) pg[k % PPW] = p;
                }
                if (pw == 0 && ((starts >> j) & 1u)) {
                    // the sequence's query rows, zero-padded to N, swizzled like a TMA box;
                    // one warp copies them all, in order, so that a slot's empty
                    // barrier is never two phases behind the wait for it
                    const int qc = carry + __popc(starts & (0xFFFFFFFFu >> (31 - j))) - 1;
                    const int qs = qc & 1;
                    int got = 1;
                    if (lane == 0)
                        got = tc::mbar_wait_sleep(qempty_bar(qs), ((qc >> 1) & 1) ^ 1, kWaitLimitNs, kIssuerSleepNs);
                    if (!__shfl_sync(0xFFFFFFFFu, got, 0)) {
                        ok = false;
                        break;
                    }
                    const uint32_t qaddr = sbase + Lay::kQ + qs * Lay::kQBytes;
                    for (int c = lane; c < N * CPR; c += 32) {
                        const int row = c / CPR, ch = c % CPR;
                        uint4 v = make_uint4(0u, 0u, 0u, 0u);
                        if (row < HI) v = __ldg(reinterpret_cast<const uint4 *>(q8 + ((size_t)b * HI + row) * DI) + ch);
                        const int sw = ch ^ ((row * DI >> 7) & (CPR - 1));
                        st_shared_v4(qaddr + row * DI + sw * 16, v);
                    }
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(qfull_bar(qs));
                }
                const int li = base + j, s = li % S;
                int got = 1;
                if (lane == 0) {
                    // every producer waits for every step in order, so no wait
                    // here runs two phases ahead of its barrier
                    got = tc::mbar_wait_sleep(empty_bar(s), ((li / S) & 1) ^ 1, kWaitLimitNs, kIssuerSleepNs);
                    if (got) {
                        const uint32_t st_addr = sbase + s * Lay::kStageBytes;
                        const int mine = max(0, min(PPW, np - PPW * pw));
                        if (pw == 0)
                            *reinterpret_cast<int4 *>(smem + s * Lay::kStageBytes + Lay::kMeta) =
                                make_int4(b, st, n, flags);
                        if (mine > 0) tc::mbar_arrive_expect_tx(full_bar(s), (uint32_t)mine * kPageTx);
                        else tc::mbar_arrive(full_bar(s));
#pragma unroll
                        for (int k = 0; k < PPW; ++k) {
                            const int pi = PPW * pw + k;
                            if (pi < np) {
                                const int p = (flags >> pi) & 1 ? pg[k] : 0;
                                tc::tma_load_2d(st_addr + pi * kDecPage * DI, &tmap_k, 0, p * kDecPage, full_bar(s));
                                tc::bulk_load(st_addr + Lay::kScales + pi * kDecPage * 4, skc + (size_t)p * kDecPage,
                                              kDecPage * 4, full_bar(s));
                            }
                        }
                    }
                }
                if (!__shfl_sync(0xFFFFFFFFu, got, 0)) {
                    ok = false;
                    break;
                }
                ++n_issued;
            }
            carry += __popc(starts);
        }
        if (lane == 0) {
            if (!ok) record_timeout();
            // this warp's copies have landed before the CTA may exit: only the
            // last S steps can still be in flight, each the latest use of its stage
            const uint64_t lim = ok ? kWaitLimitNs : 100000000ull;
            for (int li = max(0, n_issued - S); li < n_issued; ++li)
                (void)tc::mbar_wait(full_bar(li % S), (uint32_t)((li / S) & 1), lim);
        }
        __syncwarp();
    } else if (warp >= kDecMmaWarp) {
        // ------------------------------------------------------------ UMMA
        // Two MMA warps take alternate steps: one thread's issue cost per
        // step (eight small UMMAs, two commits, the waits) is most of a step
        // period, and two threads overlap it.  Accumulator a = li % A serves
        // one warp only (A even).  Both warps walk every step of the range,
        // find its sequence from the step prefix, and release each query
        // slot when they pass its sequence (the release counts two arrivals),
        // so a warp that had no step of a short sequence still releases its
        // slot; a warp waits for a slot's query only when it uses it.  No
        // barrier runs two phases ahead of a wait: refilling a stage, an
        // accumulator or a slot needs this warp's own earlier release.
        static_assert(Lay::kAccBufs % 2 == 0, "an accumulator serves one MMA warp");
        const int mw = warp - kDecMmaWarp;
        if (lane == 0) {
            bool ok = true;
            int cur_b = -1, qc = -1, b = 0;
            bool have_q = false;
            for (int li = 0; li < nsteps; ++li) {
                const int gi = i0 + li;
                while (prefix[b + 1] <= gi) ++b;  // prefix[B] = total > gi
                if (b != cur_b) {
                    if (qc >= 0) tc::umma_commit(qempty_bar(qc & 1));
                    cur_b = b;
                    ++qc;
                    have_q = false;
                }
                if ((li & 1) != mw) continue;
                const int s = li % S, a = li % A;
                if (!have_q) {
                    if (!tc::mbar_wait_sleep(qfull_bar(qc & 1), (qc >> 1) & 1, kWaitLimitNs, kIssuerSleepNs)) {
                        ok = false;
                        break;
                    }
                    have_q = true;
                }
                if (!tc::mbar_wait_sleep(full_bar(s), (li / S) & 1, kWaitLimitNs, kIssuerSleepNs) ||
                    !tc::mbar_wait_sleep(tempty_bar(a), ((li / A) & 1) ^ 1, kWaitLimitNs, kIssuerSleepNs)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t kaddr = sbase + s * Lay::kStageBytes;
                const uint32_t qaddr = sbase + Lay::kQ + (qc & 1) * Lay::kQBytes;
                const int st = gi - prefix[b];
                const int pages = min(SP, (seq_len_of(b) + kDecPage - 1) / kDecPage - SP * st);
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    if (2 * t >= pages) break;
                    const uint32_t d = tmem_base + (uint32_t)(a * Lay::kAccCols + t * N);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        tc::umma_f8(d, tc::smem_desc_kmajor(kaddr + t * 2 * kDecPage * DI + ks * 32, DI),
                                    tc::smem_desc_kmajor(qaddr + ks * 32, DI), IDESC, ks > 0 ? 1u : 0u);
                }
                tc::umma_commit(empty_bar(s));
                tc::umma_commit(tfull_bar(a));
            }
            if (!ok) record_timeout();
            // every UMMA either warp issued has completed before TMEM is freed
            tc::umma_commit(mma_done_bar);
            (void)tc::mbar_wait(mma_done_bar, 0, kWaitLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int grp = warp / 4;
        const int qw = warp & 3;  // TMEM lane quarter
        const uint32_t lane_base = tmem_base + ((uint32_t)(qw * 32) << 16);
        int cur_b = -1;
        float wv[N];
        float sqb = 0.f;
        // Each row's score range for the top-k, as order keys:
        // keyrange[b] = min key, keyrange[B + b] = complement of the max key
        // (both preset to all-ones, so atomicMin keeps each).  A warp keeps a
        // running range over its consecutive steps of one sequence and adds
        // it in when the sequence changes and at the end.
        int rng_b = -1;
        float rng_lo = INFINITY, rng_hi = -INFINITY;
        auto flush_range = [&]() {
            if (keyrange == nullptr || rng_b < 0) return;
            const uint32_t klo =
                __reduce_min_sync(0xFFFFFFFFu, rng_lo == INFINITY ? 0xFFFFFFFFu : order_key(rng_lo));
            const uint32_t khi =
                __reduce_min_sync(0xFFFFFFFFu, rng_hi == -INFINITY ? 0xFFFFFFFFu : ~order_key(rng_hi));
            if (lane == 0 && rng_b < B) {
                atomicMin(keyrange + rng_b, klo);
                atomicMin(keyrange + B + rng_b, khi);
            }
            rng_lo = INFINITY;
            rng_hi = -INFINITY;
        };
#pragma unroll
        for (int h = 0; h < N; ++h) wv[h] = 0.f;
        bool ok = true;
        for (int li = grp; li < nsteps; li += G) {
            const int s = li % S, a = li % A;
            if (!tc::mbar_wait(tfull_bar(a), (li / A) & 1, kWaitLimitNs) ||
                !tc::mbar_wait(full_bar(s), (li / S) & 1, kWaitLimitNs)) {
                ok = false;
                break;
            }
            tc::tc_fence_after();
            const uint8_t *stp = smem + s * Lay::kStageBytes;
            const int4 meta = *reinterpret_cast<const int4 *>(stp + Lay::kMeta);
            float sk[T];
#pragma unroll
            for (int t = 0; t < T; ++t) sk[t] = reinterpret_cast<const float *>(stp + Lay::kScales)[t * 128 + qw * 32 + lane];
            const int step_pages = min(SP, (meta.z + kDecPage - 1) / kDecPage - SP * meta.y);
            float v[T];
#pragma unroll
            for (int t = 0; t < T; ++t) {
                float part[4] = {0.f, 0.f, 0.f, 0.f};
                if (2 * t < step_pages) {
#pragma unroll
                    for (int c0 = 0; c0 < N; c0 += 16) {
                        float acc[16];
                        tc::tmem_ld16(lane_base + (uint32_t)(a * Lay::kAccCols + t * N + c0), acc);
                        tc::tmem_wait_ld();
                        if (meta.x != cur_b) {
                            cur_b = meta.x;
#pragma unroll
                            for (int h = 0; h < N; ++h) wv[h] = h < HI ? __ldg(w + (size_t)cur_b * HI + h) : 0.f;
                            sqb = __ldg(sq + cur_b);
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) part[j & 3] = fmaf(wv[c0 + j], fmaxf(acc[j], 0.f), part[j & 3]);
                    }
                }
                v[t] = (part[0] + part[1]) + (part[2] + part[3]);
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(tempty_bar(a));
                tc::mbar_arrive(empty_bar(s));
            }
            if (keyrange != nullptr && meta.x != rng_b) {
                flush_range();
                rng_b = meta.x;
            }
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const int pi = 2 * t + (qw >> 1);  // page of the step
                const int tok = (SP * meta.y + pi) * kDecPage + (qw & 1) * 32 + lane;
                if (tok < meta.z) {
                    const float sc = ((meta.w >> pi) & 1) ? v[t] * sqb * sk[t] : -INFINITY;
                    scores[(size_t)cur_b * ld + tok] = sc;
                    rng_lo = fminf(rng_lo, sc);
                    rng_hi = fmaxf(rng_hi, sc);
                }
            }
        }
        if (ok) flush_range();
        if (!ok) record_timeout();
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == kDecMmaWarp) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D uint8 tensor map: rows of `row_bytes` bytes every `row_stride` bytes
// (row_bytes when 0), boxes of box_rows rows, swizzled by the row width
// (32/64/128 bytes).
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, int row_bytes, int box_rows, uint64_t row_stride = 0) {
    auto enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(row_stride ? row_stride : (uint64_t)row_bytes)};
    const cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle swz = row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                   : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_32B;
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int HI, int DI, int MODE, bool VARLEN>
cudaError_t launch_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8, const float *sk, int L,
                      int row_begin, int n_rows, const EpiArgs &a, cudaStream_t stream) {
    constexpr int KS = MODE == kModeSample ? kSampleStride : 1;
    CUtensorMap mk, mq;
    if (!make_map(&mk, k8, (uint64_t)((L + KS - 1) / KS), DI, kStepKeys, (uint64_t)KS * DI))
        return cudaErrorInvalidValue;
    if (!make_map(&mq, q8, (uint64_t)L * HI, DI, kTileN)) return cudaErrorInvalidValue;
    constexpr int NQ = kTileN / HI;
    const int nb = (n_rows + NQ - 1) / NQ;
    const int grid = nb < sm_count() ? nb : sm_count();
    // at least 116 KB so that one CTA (and its 512 TMEM columns) owns each SM
    constexpr int smem = Layout<DI>::kAlloc > 116 * 1024 ? Layout<DI>::kAlloc : 116 * 1024;
    cudaError_t e = set_smem_at_least<indexer_tc_kernel<HI, DI, MODE, VARLEN>>(smem);
    if (e != cudaSuccess) return e;
    indexer_tc_kernel<HI, DI, MODE, VARLEN><<<grid, EpiShape<HI>::kThreads, smem, stream>>>(mk, mq, sq, w, sk,
                                                                                           row_begin, n_rows, a);
    return cudaGetLastError();
}

template <int N, int DI>
cudaError_t launch_decode_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8c, const float *skc,
                             const int32_t *block_table, int max_pages, int num_pages, const int32_t *seq_lens,
                             int max_seq_len, int B, int HI, float *scores, int64_t ld, uint32_t *keyrange,
                             cudaStream_t stream) {
    CUtensorMap mk;
    if (!make_map(&mk, k8c, (uint64_t)num_pages * kDecPage, DI, kDecPage)) return cudaErrorInvalidValue;
    constexpr int smem = DecLayout<N, DI>::kAlloc > 116 * 1024 ? DecLayout<N, DI>::kAlloc : 116 * 1024;
    cudaError_t e = set_smem_at_least<indexer_decode_tc_kernel<N, DI>>(smem);
    if (e != cudaSuccess) return e;
    indexer_decode_tc_kernel<N, DI><<<sm_count(), kDecThreads, smem, stream>>>(
        mk, q8, sq, w, skc, block_table, max_pages, num_pages, seq_lens, max_seq_len, B, HI, scores, ld, keyrange);
    return cudaGetLastError();
}

}  // namespace

bool indexer_tc_supported(int HI, int dI) {
    return (HI == 8 || HI == 16 || HI == 32 || HI == 64) && (dI == 32 || dI == 64 || dI == 128);
}

namespace {

template <int MODE>
cudaError_t launch_prefill_mode(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                const float *sk, int L, int HI, int dI, int row_begin, int n_rows, const EpiArgs &a,
                                cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    // packed sequences only on the fused path's modes (the scores mode keeps one sequence per call)
    constexpr bool kVarlenModes = MODE != kModeScores;
    auto by_di = [&](auto hi) -> cudaError_t {
        constexpr int H = decltype(hi)::value;
        if (kVarlenModes && a.cu != nullptr) {
            switch (dI) {
                case 32: return launch_tc<H, 32, MODE, kVarlenModes>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
                case 64: return launch_tc<H, 64, MODE, kVarlenModes>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
                case 128: return launch_tc<H, 128, MODE, kVarlenModes>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
                default: return cudaErrorInvalidValue;
            }
        }
        switch (dI) {
            case 32: return launch_tc<H, 32, MODE, false>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
            case 64: return launch_tc<H, 64, MODE, false>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
            case 128: return launch_tc<H, 128, MODE, false>(q8, sq, w, k8, sk, L, row_begin, n_rows, a, stream);
            default: return cudaErrorInvalidValue;
        }
    };
    switch (HI) {
        case 8: return by_di(std::integral_constant<int, 8>{});
        case 16: return by_di(std::integral_constant<int, 16>{});
        case 32: return by_di(std::integral_constant<int, 32>{});
        case 64: return by_di(std::integral_constant<int, 64>{});
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_indexer_prefill_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                      const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                      float *scores, int64_t ld, float *row_stats, cudaStream_t stream) {
    EpiArgs a{};
    a.scores = scores;
    a.ld = ld;
    a.row_stats = row_stats;
    return launch_prefill_mode<kModeScores>(q8, sq, w, k8, sk, L, HI, dI, row_begin, n_rows, a, stream);
}

cudaError_t launch_indexer_sample_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                     const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                     float *sample_scores, int64_t ld, const int32_t *cu, int nseq,
                                     cudaStream_t stream) {
    EpiArgs a{};
    a.scores = sample_scores;
    a.ld = ld;
    a.cu = cu;
    a.nseq = nseq;
    return launch_prefill_mode<kModeSample>(q8, sq, w, k8, sk, L, HI, dI, row_begin, n_rows, a, stream);
}

cudaError_t launch_indexer_cand_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                   const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                   const float *tau, int2 *cand, int *cand_count, int seg_cap, const int32_t *cu,
                                   int nseq, cudaStream_t stream) {
    EpiArgs a{};
    a.cu = cu;
    a.nseq = nseq;
    a.tau = tau;
    a.cand = cand;
    a.cand_count = cand_count;
    a.seg_cap = seg_cap;
    return launch_prefill_mode<kModeCand>(q8, sq, w, k8, sk, L, HI, dI, row_begin, n_rows, a, stream);
}

int indexer_sample_stride() { return kSampleStride; }

cudaError_t indexer_tc_set_wait_limit(unsigned long long ns) {
    const unsigned long long v = ns ? ns : kWaitLimitNs;
    return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof v);
}

cudaError_t indexer_tc_take_error(unsigned int *flag) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_indexer_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_indexer_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace dsa

namespace dsa {

bool indexer_decode_tc_supported(int HI, int dI, int B, int max_seq_len) {
    const bool shape = (HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64) && (dI == 32 || dI == 64 || dI == 128);
    // the step prefix lives in shared memory and is counted in int
    return shape && B <= kDecMaxB && (int64_t)B * ((max_seq_len + kDecPage - 1) / kDecPage) < (1ll << 31);
}

cudaError_t launch_indexer_decode_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8c,
                                     const float *skc, const int32_t *block_table, int max_pages, int num_pages,
                                     const int32_t *seq_lens, int max_seq_len, int B, int HI, int dI, float *scores,
                                     int64_t ld, uint32_t *keyrange, cudaStream_t stream) {
    if (B == 0 || max_seq_len == 0) return cudaSuccess;
    auto by_di = [&](auto n) -> cudaError_t {
        constexpr int NN = decltype(n)::value;
        switch (dI) {
            case 32: return launch_decode_tc<NN, 32>(q8, sq, w, k8c, skc, block_table, max_pages, num_pages, seq_lens,
                                                     max_seq_len, B, HI, scores, ld, keyrange, stream);
            case 64: return launch_decode_tc<NN, 64>(q8, sq, w, k8c, skc, block_table, max_pages, num_pages, seq_lens,
                                                     max_seq_len, B, HI, scores, ld, keyrange, stream);
            case 128: return launch_decode_tc<NN, 128>(q8, sq, w, k8c, skc, block_table, max_pages, num_pages,
                                                       seq_lens, max_seq_len, B, HI, scores, ld, keyrange, stream);
            default: return cudaErrorInvalidValue;
        }
    };
    if (HI <= 16) return by_di(std::integral_constant<int, 16>{});
    if (HI == 32) return by_di(std::integral_constant<int, 32>{});
    return by_di(std::integral_constant<int, 64>{});
}

}  // namespace dsa
