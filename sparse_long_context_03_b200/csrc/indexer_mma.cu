// indexer_mma.cu -- lightning-indexer scores on warp-level FP8 tensor-core MMA.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式, indexer:
//     I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s])
// with one key head shared by every indexer head and FP8 inputs (report
// translation, section 2.3.1).  The per-token scales are positive, so
//     I[t,s] = sq[t] * sk[s] * sum_j w[t,j] * ReLU(q8[t,j] . k8[s])
// where the byte dot products run on the tensor cores (e4m3 x e4m3 -> fp32).
//
// GEMM orientation: M = keys (16 per warp), N = indexer heads (8 per MMA
// tile), K = dI.  Each thread's accumulators cover two keys and two heads per
// tile, so the ReLU, the weighted head sum and the causal mask are applied in
// registers; the head sum finishes with two xor-shuffles across the 4 lanes
// that share a key.
//
// Two kernels share this, both for cases the tcgen05 kernels of
// indexer_tc.cu do not take: a prefill indexer for HI = 4, and a paged decode
// indexer (one query per sequence, keys read through the block table) for
// batches above 4096 sequences or caches of 2^31 rows and more.
// launch_indexer_decode picks the tcgen05 decode kernel whenever it applies.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

// Score contribution of one query against the warp's 16 keys.  a: key
// fragments [KS][4]; b(nt, ks, half) yields the query fragment; wv(nt, i) the
// head weights.  Returns the two per-key sums (keys gid and gid+8), complete
// on every lane after the shuffles.
template <int KS, int NT, typename BF, typename WF>
__device__ __forceinline__ void score_16keys(const uint32_t (&a)[KS][4], BF bfrag, WF wv, float &p0, float &p1) {
    p0 = 0.f;
    p1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) mma_e4m3_16832(acc, a[ks], bfrag(nt, ks, 0), bfrag(nt, ks, 1));
        const float wa = wv(nt, 0), wb = wv(nt, 1);
        p0 = fmaf(wa, fmaxf(acc[0], 0.f), p0);
        p0 = fmaf(wb, fmaxf(acc[1], 0.f), p0);
        p1 = fmaf(wa, fmaxf(acc[2], 0.f), p1);
        p1 = fmaf(wb, fmaxf(acc[3], 0.f), p1);
    }
    p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
    p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
    p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
}

// Key fragments of 16 consecutive key rows (row stride DI bytes) for the
// m16n8k32 A operand: a[ks][0] row gid, bytes ks*32 + tig*4; [1] row gid+8;
// [2] row gid, bytes +16; [3] row gid+8, bytes +16.
template <int DI>
__device__ __forceinline__ void load_key_frags(uint32_t (&a)[DI / 32][4], const uint8_t *row0, const uint8_t *row8,
                                               bool ok0, bool ok8, int tig) {
#pragma unroll
    for (int ks = 0; ks < DI / 32; ++ks) {
        const int off = ks * 32 + tig * 4;
        a[ks][0] = ok0 ? __ldg(reinterpret_cast<const uint32_t *>(row0 + off)) : 0u;
        a[ks][1] = ok8 ? __ldg(reinterpret_cast<const uint32_t *>(row8 + off)) : 0u;
        a[ks][2] = ok0 ? __ldg(reinterpret_cast<const uint32_t *>(row0 + off + 16)) : 0u;
        a[ks][3] = ok8 ? __ldg(reinterpret_cast<const uint32_t *>(row8 + off + 16)) : 0u;
    }
}

constexpr int kKeysPerCta = 128;  // 8 warps x 16 keys

// Queries per prefill CTA: as many as fit 40 KB of static shared memory.
template <int DI, int NT>
constexpr int prefill_qb() {
    constexpr int per_query = NT * 8 * (DI + 16);
    return per_query * 16 <= 40960 ? 16 : (per_query * 8 <= 40960 ? 8 : 4);
}

template <int DI, int NT>
__global__ void __launch_bounds__(256) indexer_prefill_mma_kernel(
    const uint8_t *__restrict__ q8, const float *__restrict__ sq, const float *__restrict__ w,
    const uint8_t *__restrict__ k8, const float *__restrict__ sk, int HI, int row_begin, int n_rows,
    float *__restrict__ scores, int64_t ld) {
    constexpr int KS = DI / 32;
    constexpr int HP = NT * 8;      // heads padded to the MMA tile
    constexpr int QROW = DI + 16;   // padded smem row: conflict-free fragment loads
    constexpr int kPrefillQB = prefill_qb<DI, NT>();
    __shared__ __align__(16) uint8_t q_s[kPrefillQB * HP * QROW];
    __shared__ float w_s[kPrefillQB][HP];
    __shared__ float sq_s[kPrefillQB];

    const int t0 = row_begin + blockIdx.y * kPrefillQB;
    const int t_last = min(t0 + kPrefillQB, row_begin + n_rows) - 1;
    const int s0 = blockIdx.x * kKeysPerCta;
    if (s0 > t_last) return;  // tile entirely above the causal diagonal

    for (int i = threadIdx.x; i < kPrefillQB * HP * (DI / 16); i += blockDim.x) {
        const int row = i / (DI / 16), c16 = i % (DI / 16);
        const int qi = row / HP, h = row % HP, t = t0 + qi;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (t <= t_last && h < HI) v = __ldg(reinterpret_cast<const uint4 *>(q8 + ((size_t)t * HI + h) * DI) + c16);
        *reinterpret_cast<uint4 *>(q_s + row * QROW + c16 * 16) = v;
    }
    for (int i = threadIdx.x; i < kPrefillQB * HP; i += blockDim.x) {
        const int qi = i / HP, h = i % HP, t = t0 + qi;
        w_s[qi][h] = (t <= t_last && h < HI) ? __ldg(w + (size_t)t * HI + h) : 0.f;
    }
    if (threadIdx.x < kPrefillQB) {
        const int t = t0 + threadIdx.x;
        sq_s[threadIdx.x] = t <= t_last ? __ldg(sq + t) : 0.f;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = lane_id(), gid = lane >> 2, tig = lane & 3;
    const int sb = s0 + warp * 16;
    if (sb > t_last) return;
    const int key0 = sb + gid, key8 = key0 + 8;
    uint32_t a[KS][4];
    load_key_frags<DI>(a, k8 + (size_t)key0 * DI, k8 + (size_t)key8 * DI, key0 <= t_last, key8 <= t_last, tig);
    const float sk0 = key0 <= t_last ? __ldg(sk + key0) : 0.f;
    const float sk8 = key8 <= t_last ? __ldg(sk + key8) : 0.f;

    for (int qi = 0; qi < kPrefillQB; ++qi) {
        const int t = t0 + qi;
        if (t > t_last) break;
        if (sb > t) continue;
        const uint8_t *qrow = q_s + (qi * HP) * QROW;
        float p0, p1;
        score_16keys<KS, NT>(
            a,
            [&](int nt, int ks, int half) {
                return *reinterpret_cast<const uint32_t *>(qrow + (nt * 8 + gid) * QROW + ks * 32 + tig * 4 + half * 16);
            },
            [&](int nt, int i) { return w_s[qi][nt * 8 + tig * 2 + i]; }, p0, p1);
        const float f = sq_s[qi];
        float *srow = scores + (size_t)(t - row_begin) * ld;
        if (tig == 0 && key0 <= t) srow[key0] = p0 * f * sk0;
        if (tig == 1 && key8 <= t) srow[key8] = p1 * f * sk8;
    }
}

constexpr int kDecodeWarps = 8;
constexpr int kDecodePagesPerWarp = 4;
constexpr int kDecodePagesPerCta = kDecodeWarps * kDecodePagesPerWarp;

// Shared staging of one cached page: 64 key rows at a pitch of dI + 16 bytes
// (8 rows read by one ldmatrix then start in 8 different bank groups), then
// the 64 key scales.
template <int DI>
constexpr int page_stage_bytes() {
    return kPage * (DI + 16) + kPage * 4;
}

template <int DI, int NT>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2) indexer_decode_mma_kernel(
    const uint8_t *__restrict__ q8, const float *__restrict__ sq, const float *__restrict__ w,
    const uint8_t *__restrict__ k8c, const float *__restrict__ skc, const int32_t *__restrict__ block_table,
    int max_pages, int num_pages, const int32_t *__restrict__ seq_lens, int max_seq_len, int HI,
    float *__restrict__ scores, int64_t ld) {
    constexpr int KS = DI / 32;
    constexpr int PITCH = DI + 16;
    constexpr int STAGE = page_stage_bytes<DI>();
    constexpr int CPR = DI / 16;  // 16-byte chunks per key row
    extern __shared__ __align__(16) uint8_t smem[];
    const int b = blockIdx.y;
    const int n = min(min(__ldg(seq_lens + b), max_seq_len), max_pages * kPage);
    const int warp = threadIdx.x >> 5, lane = lane_id(), gid = lane >> 2, tig = lane & 3;
    const int lp0 = blockIdx.x * kDecodePagesPerCta + warp;   // this warp's pages: lp0 + kDecodeWarps * i
    if (lp0 * kPage >= n) return;
    uint8_t *ws = smem + warp * 2 * STAGE;
    const uint32_t ws_u32 = smem_u32(ws);

    // Query fragments (m16n8k32 B operand, column n = head): b0 bytes
    // ks*32 + tig*4 of head nt*8+gid, b1 the same +16.
    uint32_t qf[NT][KS][2];
    float wf[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + gid;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const uint8_t *qp = q8 + ((size_t)b * HI + h) * DI + ks * 32 + tig * 4;
            qf[nt][ks][0] = h < HI ? __ldg(reinterpret_cast<const uint32_t *>(qp)) : 0u;
            qf[nt][ks][1] = h < HI ? __ldg(reinterpret_cast<const uint32_t *>(qp + 16)) : 0u;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int hw = nt * 8 + tig * 2 + i;
            wf[nt][i] = hw < HI ? __ldg(w + (size_t)b * HI + hw) : 0.f;
        }
    }
    const float f = __ldg(sq + b);
    float *srow = scores + (size_t)b * ld;

    auto page_of = [&](int i) -> int { return lp0 + kDecodeWarps * i; };
    auto page_id = [&](int lp) -> int {
        const int pg = __ldg(block_table + (size_t)b * max_pages + lp);
        return (pg >= 0 && pg < num_pages) ? pg : -1;
    };
    auto issue = [&](int i) {
        const int lp = page_of(i);
        const int pg = page_id(lp);
        const uint32_t st = ws_u32 + (uint32_t)((i & 1) * STAGE);
        const uint8_t *src = k8c + (size_t)(pg < 0 ? 0 : pg) * kPage * DI;
#pragma unroll
        for (int c = lane; c < kPage * CPR; c += 32) {
            const int row = c / CPR, ch = c % CPR;
            cp_async_16(st + row * PITCH + ch * 16, src + row * DI + ch * 16);
        }
        if (lane < kPage * 4 / 16) cp_async_16(st + kPage * PITCH + lane * 16,
                                                skc + (size_t)(pg < 0 ? 0 : pg) * kPage + lane * 4);
    };
    int np = 0;
    while (np < kDecodePagesPerWarp && page_of(np) * kPage < n) ++np;
    issue(0);
    cp_async_commit();
    for (int i = 0; i < np; ++i) {
        if (i + 1 < np) issue(i + 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const int lp = page_of(i);
        const bool page_ok = page_id(lp) >= 0;
        const int sb = lp * kPage;
        const uint32_t st = ws_u32 + (uint32_t)((i & 1) * STAGE);
        const float *sks = reinterpret_cast<const float *>(ws + (i & 1) * STAGE + kPage * PITCH);
#pragma unroll 1
        for (int m = 0; m < 4; ++m) {
            uint32_t a[KS][4];
            const int row = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) ldmatrix_x4(a[ks], st + row * PITCH + ks * 32 + (lane >> 4) * 16);
            float p0, p1;
            score_16keys<KS, NT>(
                a, [&](int nt, int ks, int half) { return qf[nt][ks][half]; },
                [&](int nt, int j) { return wf[nt][j]; }, p0, p1);
            const int k0 = m * 16 + gid, k8 = k0 + 8;
            const int key0 = sb + k0, key8 = sb + k8;
            if (tig == 0 && key0 < n) srow[key0] = page_ok ? p0 * f * sks[k0] : -INFINITY;
            if (tig == 1 && key8 < n) srow[key8] = page_ok ? p1 * f * sks[k8] : -INFINITY;
        }
        __syncwarp();
    }
    cp_async_wait<0>();
}

// Calls launch(integral_constant<DI>, integral_constant<NT>) for a supported
// (HI, dI); HI = 4 uses one 8-wide head tile with the upper half zeroed.
template <typename F>
bool dispatch_shape(int HI, int dI, F &&launch) {
    auto by_nt = [&](auto di) -> bool {
        switch (HI) {
            case 4:
            case 8: return launch(di, std::integral_constant<int, 1>{});
            case 16: return launch(di, std::integral_constant<int, 2>{});
            case 32: return launch(di, std::integral_constant<int, 4>{});
            case 64: return launch(di, std::integral_constant<int, 8>{});
            default: return false;
        }
    };
    switch (dI) {
        case 32: return by_nt(std::integral_constant<int, 32>{});
        case 64: return by_nt(std::integral_constant<int, 64>{});
        case 128: return by_nt(std::integral_constant<int, 128>{});
        default: return false;
    }
}

// Row value range of already written prefill score rows (one warp per row),
// in the row-statistics layout the top-k reads: four (min, max) partials per
// row; here the first carries the whole row and the others are empty.
__global__ void __launch_bounds__(256) row_stats_kernel(const float *__restrict__ scores, int64_t ld, int row_begin,
                                                        int n_rows, float *__restrict__ row_stats) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int lane = lane_id(), n = row_begin + r + 1;
    const float *row = scores + (size_t)r * ld;
    float lo = INFINITY, hi = -INFINITY;
    for (int i = lane; i < n; i += 32) {
        const float v = __ldg(row + i);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    if (lane < 8) row_stats[(size_t)r * 8 + lane] = lane == 0 ? lo : (lane == 1 ? hi : ((lane & 1) ? -INFINITY : INFINITY));
}

}  // namespace

cudaError_t launch_row_stats(const float *scores, int64_t ld, int row_begin, int n_rows, float *row_stats,
                             cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    row_stats_kernel<<<(n_rows + 7) / 8, 256, 0, stream>>>(scores, ld, row_begin, n_rows, row_stats);
    return cudaGetLastError();
}

bool indexer_shape_supported(int HI, int dI) {
    return (HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64) && (dI == 32 || dI == 64 || dI == 128);
}

cudaError_t launch_indexer_prefill_mma(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8,
                                       const float *sk, int HI, int dI, int row_begin, int n_rows, float *scores,
                                       int64_t ld, cudaStream_t stream) {
    if (n_rows == 0) return cudaSuccess;
    const int key_tiles = (row_begin + n_rows + kKeysPerCta - 1) / kKeysPerCta;
    const bool ok = dispatch_shape(HI, dI, [&](auto di, auto nt) {
        constexpr int DI = decltype(di)::value, NT = decltype(nt)::value;
        constexpr int QB = prefill_qb<DI, NT>();
        const dim3 grid(key_tiles, (n_rows + QB - 1) / QB);
        indexer_prefill_mma_kernel<DI, NT><<<grid, 256, 0, stream>>>(q8, sq, w, k8, sk, HI, row_begin, n_rows,
                                                                    scores, ld);
        return true;
    });
    return ok ? cudaGetLastError() : cudaErrorInvalidValue;
}

cudaError_t launch_indexer_decode(const uint8_t *q8, const float *sq, const float *w, const uint8_t *k8c,
                                  const float *skc, const int32_t *block_table, int max_pages, int num_pages,
                                  const int32_t *seq_lens, int max_seq_len, int B, int HI, int dI, float *scores,
                                  int64_t ld, cudaStream_t stream, uint32_t *keyrange, bool *range_written) {
    if (range_written != nullptr) *range_written = false;
    if (B == 0 || max_seq_len == 0) return cudaSuccess;
    // the tensor-core path, unless the batch outgrows its shared-memory prefix
    // or the cache its 32-bit TMA row coordinates
    if ((int64_t)num_pages * kPage < (1ll << 31) && indexer_decode_tc_supported(HI, dI, B, max_seq_len)) {
        if (range_written != nullptr) *range_written = keyrange != nullptr;
        return launch_indexer_decode_tc(q8, sq, w, k8c, skc, block_table, max_pages, num_pages, seq_lens, max_seq_len,
                                        B, HI, dI, scores, ld, keyrange, stream);
    }
    const int pages = (max_seq_len + kPage - 1) / kPage;
    const dim3 grid((pages + kDecodePagesPerCta - 1) / kDecodePagesPerCta, B);
    cudaError_t err = cudaSuccess;
    const bool ok = dispatch_shape(HI, dI, [&](auto di, auto nt) {
        constexpr int DI = decltype(di)::value, NT = decltype(nt)::value;
        constexpr int smem = kDecodeWarps * 2 * page_stage_bytes<DI>();
        err = set_smem_at_least<indexer_decode_mma_kernel<DI, NT>>(smem);
        if (err != cudaSuccess) return true;
        indexer_decode_mma_kernel<DI, NT><<<grid, kDecodeWarps * 32, smem, stream>>>(
            q8, sq, w, k8c, skc, block_table, max_pages, num_pages, seq_lens, max_seq_len, HI, scores, ld);
        err = cudaGetLastError();
        return true;
    });
    return ok ? err : cudaErrorInvalidValue;
}

}  // namespace dsa
