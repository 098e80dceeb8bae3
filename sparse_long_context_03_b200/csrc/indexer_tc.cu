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

// Columns per epilogue warp and the warp counts for HI heads per query.  With
// 18 warps, two of the four schedulers hold five warps, whose 16K-register
// files cap a thread at 96 registers (HI <= 32); HI = 64 has 10 warps.
template <int HI>
struct EpiShape {
    static constexpr int CW = HI > 32 ? HI : 32;
    static constexpr int kEpiWarps = 4 * (kTileN / CW);
    static constexpr int kThreads = (kEpiWarps + 2) * 32;
    static constexpr int kProducerWarp = kEpiWarps;
    static constexpr int kMmaWarp = kEpiWarps + 1;
};
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr uint32_t kIssuerSleepNs = 32;            // back-off of the TMA and MMA warps


template <int DI>
struct Layout {
    static constexpr int kTileBytes = kStepKeys * DI;  // one step of keys
    static constexpr int kStages = (200 * 1024 - 2 * kTileN * DI) / kTileBytes > 8
                                       ? 8
                                       : (200 * 1024 - 2 * kTileN * DI) / kTileBytes;
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

template <int HI, int DI>
__global__ void __launch_bounds__(EpiShape<HI>::kThreads, 1) indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                                 const __grid_constant__ CUtensorMap tmap_q,
                                                                 const float *__restrict__ sq,
                                                                 const float *__restrict__ w,
                                                                 const float *__restrict__ sk, int row_begin,
                                                                 int n_rows, float *__restrict__ scores,
                                                                 int64_t ld, float *__restrict__ row_stats) {
    using Lay = Layout<DI>;
    using ES = EpiShape<HI>;
    constexpr int kEpiWarps = ES::kEpiWarps, kProducerWarp = ES::kProducerWarp, kMmaWarp = ES::kMmaWarp;
    constexpr int CW = ES::CW;          // columns per epilogue warp
    constexpr int NQ = kTileN / HI;     // queries per block
    constexpr int QPW = CW / HI;        // whole queries per epilogue warp (1 when HI >= 32)
    constexpr int KSTEPS = DI / 32;
    constexpr int kStages = Lay::kStages;
    constexpr uint32_t IDESC = tc::idesc_e4m3_f32(kTileM, kTileN);

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
            tc::mbar_init(qempty_bar(b), 1);
        }
        for (int b = 0; b < kPairs; ++b) {
            tc::mbar_init(tfull_bar(b), 1);
            tc::mbar_init(tempty_bar(b), kEpiWarps);
        }
        tc::mbar_init(mma_done_bar, 1);
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
                const int nstep = t_hi / kStepKeys + 1;
                const int qs = bi & 1;
                if (!tc::mbar_wait_sleep(qempty_bar(qs), ((bi >> 1) & 1) ^ 1, kWaitLimitNs, kIssuerSleepNs)) {
                    ok = false;
                    break;
                }
                tc::mbar_arrive_expect_tx(qfull_bar(qs), Lay::kQBytes);
                tc::tma_load_2d(sbase + Lay::kQ + qs * Lay::kQBytes, &tmap_q, 0, t0 * HI, qfull_bar(qs));
                ++q_issued;
                for (int st = 0; st < nstep; ++st) {
                    if (!tc::mbar_wait_sleep(empty_bar(stage), phase ^ 1, kWaitLimitNs, kIssuerSleepNs)) {
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
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ UMMA
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0, bi = 0;
            bool ok = true;
            for (int i = blockIdx.x; i < nb && ok; i += gridDim.x, ++bi) {
                const int qb = nb - 1 - i;
                const int t0 = row_begin + qb * NQ;
                const int t_hi = min(t0 + NQ, row_end) - 1;
                const int nstep = t_hi / kStepKeys + 1;
                const int qs = bi & 1;
                if (!tc::mbar_wait_sleep(qfull_bar(qs), (bi >> 1) & 1, kWaitLimitNs, kIssuerSleepNs)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const uint32_t qaddr = sbase + Lay::kQ + qs * Lay::kQBytes;
                for (int st = 0; st < nstep; ++st, ++it) {
                    const int pr = it % kPairs;
                    if (!tc::mbar_wait_sleep(tempty_bar(pr), ((it / kPairs) & 1) ^ 1, kWaitLimitNs,
                                             kIssuerSleepNs) ||
                        !tc::mbar_wait_sleep(full_bar(stage), phase, kWaitLimitNs, kIssuerSleepNs)) {
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
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
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
        const int qw = warp & 3;          // TMEM lane quarter: keys 32*qw ..
        const int cg = warp >> 2;         // column group: columns cg*CW ..
        const uint32_t lane_base = tmem_base + ((uint32_t)(qw * 32) << 16);
        int it = 0;
        bool ok = true;
        for (int i = blockIdx.x; i < nb && ok; i += gridDim.x) {
            const int qb = nb - 1 - i;
            const int t0 = row_begin + qb * NQ;
            const int t_hi = min(t0 + NQ, row_end) - 1;
            const int nstep = t_hi / kStepKeys + 1;
            // this warp's query head weights, in registers for the whole block
            float2 wv[CW / 2];
#pragma unroll
            for (int c = 0; c < CW; c += 2) {
                const int t = t0 + (cg * CW + c) / HI;
                wv[c / 2] = t <= t_hi ? __ldg(reinterpret_cast<const float2 *>(w + (size_t)t0 * HI + cg * CW + c))
                                      : make_float2(0.f, 0.f);
            }
            float sqv[QPW], vlo[QPW], vhi[QPW];
#pragma unroll
            for (int q = 0; q < QPW; ++q) {
                const int t = t0 + (cg * CW) / HI + q;
                sqv[q] = t <= t_hi ? __ldg(sq + t) : 0.f;
                vlo[q] = INFINITY;
                vhi[q] = -INFINITY;
            }
            for (int st = 0; st < nstep; ++st, ++it) {
                const int pr = it % kPairs;
                if (!tc::mbar_wait(tfull_bar(pr), (it / kPairs) & 1, kWaitLimitNs)) { ok = false; break; }
                tc::tc_fence_after();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int buf = 2 * pr + h;
                    const int s = st * kStepKeys + h * kTileM + qw * 32 + lane;
                    const float sks = s <= t_hi ? __ldg(sk + s) : 0.f;
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
                        if (t <= t_hi && s <= t) {
                            const float v = (part[q][0].x + part[q][1].x) + (part[q][0].y + part[q][1].y);
                            const float score = v * sqv[q] * sks;
                            scores[(size_t)(t - row_begin) * ld + s] = score;
                            vlo[q] = fminf(vlo[q], score);
                            vhi[q] = fmaxf(vhi[q], score);
                        }
                    }
                }
            }
            if (row_stats != nullptr && ok) {
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
                        float *st8 = row_stats + (size_t)(t - row_begin) * 8;
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

// 2D uint8 tensor map: rows of `row_bytes` bytes, boxes of box_rows rows,
// swizzled by the row width (32/64/128 bytes).
bool make_map(CUtensorMap *m, const void *base, uint64_t rows, int row_bytes, int box_rows) {
    auto enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
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

template <int HI, int DI>
cudaError_t launch_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8, const float *sk, int L,
                      int row_begin, int n_rows, float *scores, int64_t ld, float *row_stats, cudaStream_t stream) {
    CUtensorMap mk, mq;
    if (!make_map(&mk, k8, (uint64_t)L, DI, kStepKeys)) return cudaErrorInvalidValue;
    if (!make_map(&mq, q8, (uint64_t)L * HI, DI, kTileN)) return cudaErrorInvalidValue;
    constexpr int NQ = kTileN / HI;
    const int nb = (n_rows + NQ - 1) / NQ;
    const int grid = nb < sm_count() ? nb : sm_count();
    // at least 116 KB so that one CTA (and its 512 TMEM columns) owns each SM
    constexpr int smem = Layout<DI>::kAlloc > 116 * 1024 ? Layout<DI>::kAlloc : 116 * 1024;
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<HI, DI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    indexer_tc_kernel<HI, DI><<<grid, EpiShape<HI>::kThreads, smem, stream>>>(mk, mq, sq, w, sk, row_begin, n_rows,
                                                                             scores, ld, row_stats);
    return cudaGetLastError();
}

}  // namespace

bool indexer_tc_supported(int HI, int dI) {
    return (HI == 8 || HI == 16 || HI == 32 || HI == 64) && (dI == 32 || dI == 64 || dI == 128);
}

cudaError_t launch_indexer_prefill_tc(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                      const float *sk, int L, int HI, int dI, int row_begin, int n_rows,
                                      float *scores, int64_t ld, float *row_stats, cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    auto by_di = [&](auto hi) -> cudaError_t {
        constexpr int H = decltype(hi)::value;
        switch (dI) {
            case 32: return launch_tc<H, 32>(q8, sq, w, k8, sk, L, row_begin, n_rows, scores, ld, row_stats, stream);
            case 64: return launch_tc<H, 64>(q8, sq, w, k8, sk, L, row_begin, n_rows, scores, ld, row_stats, stream);
            case 128: return launch_tc<H, 128>(q8, sq, w, k8, sk, L, row_begin, n_rows, scores, ld, row_stats, stream);
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

cudaError_t indexer_tc_take_error(unsigned int *flag) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_indexer_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_indexer_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace dsa
