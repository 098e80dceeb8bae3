// attention.cu -- sparse GQA attention over the selected key rows.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式:
//     u[t,g] = Attn(h[t,g], { c[s,g] | s in Omega_t })
// report translation section 2.3.2: one index set Omega_t for every KV group,
// group outputs concatenated; section 5.1.2: a row below k visits only its
// t+1 causally visible entries.  Attn is read as scaled dot-product softmax
// attention; head h uses group g = h / (Hq / Hkv).
//
// Work unit: one warp owns one (query, KV group) pair and all G <= 8 query
// heads of that group.  Each selected key row of the group (D bf16 values of
// K, the same of V) is gathered ONCE per pair with 16-byte cp.async copies
// into a swizzled shared-memory stage and serves every head of the group.
// Per 16-key block:
//   S^T[16 keys x 8 heads] = K_blk[16 x D] . Q^T[D x 8]      (mma m16n8k16, M = keys)
//   online softmax per head (exp2 domain, running max / sum)
//   O^T[D x 8 heads]     += V_blk^T[D x 16] . P^T[16 x 8]    (mma m16n8k16)
// P^T moves from accumulator layout to the B-operand layout with one
// movmatrix.trans per 8x8 half, so no shared-memory round trip is needed.
// Keys sit on the MMA M dimension, so the 8-wide N dimension is exactly the
// 8 heads of a group: no padded rows are multiplied.
//
// Prefill: a CTA is one warp, one (query, group) pair.
// Decode: the k selected rows of a (sequence, group) are split across warps
// (split-K); each split writes (max, sum, unnormalised O) to the workspace and
// a combine kernel merges them.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

// Two stages of 16 keys per warp (16 KB) and one warp per CTA: 13 warps
// share an SM's shared memory, and a warp's slot is handed to the next
// (query, group) the moment it finishes, not when its CTA's slowest warp
// does.  The kernel is bound by the latency of its L2 gathers, so more
// resident warps beat deeper per-warp pipelines: three stages and 8 warps per
// SM ran 40 % slower, two warps per CTA 17 % slower.
constexpr int kWarpsPerCta = 1;
constexpr int kStages = 2;
constexpr int kBlk = 16;  // keys per pipeline stage

template <int D>
constexpr int stage_bytes() {
    return kBlk * D * 2 * 2;  // K and V, bf16
}
template <int D>
constexpr int warp_smem_bytes() {
    return kStages * stage_bytes<D>();
}

// Running state of one warp's online softmax; lane (gid, tig) holds heads
// 2*tig and 2*tig+1 and, for each 16-row m-tile md of O^T, dims md*16+gid
// and md*16+gid+8.
template <int D>
struct WarpAttn {
    static constexpr int KT = D / 16;
    uint32_t qf[KT][2];
    float o[KT][4];
    float m[2], l[2];
};

// Byte offset of 16-byte chunk `c` of key row `row` inside a stage buffer:
// chunks are XOR-swizzled by the row's low 3 bits so that ldmatrix reads of
// 8 rows at one logical chunk hit 8 different bank groups.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)(row * (D * 2) + ((c ^ (row & 7)) << 4));
}

// Gather the K and V rows of one 16-key block into a stage.  rowaddr holds,
// in lanes 0..15, the element offset of key (lane)'s row for this group.
template <int D>
__device__ __forceinline__ void gather_block(uint32_t ks, uint32_t vs, const uint16_t *K, const uint16_t *V,
                                             int64_t rowaddr, int lane) {
    constexpr int CPR = D / 8;          // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;       // rows per warp-wide pass
    const int c = lane % CPR, rsub = lane / CPR;
#pragma unroll
    for (int it = 0; it < kBlk / RPI; ++it) {
        const int key = rsub + it * RPI;
        const int64_t off = __shfl_sync(0xFFFFFFFFu, rowaddr, key);
        cp_async_16(ks + swz<D>(key, c), K + off + c * 8);
        cp_async_16(vs + swz<D>(key, c), V + off + c * 8);
    }
}

template <int D>
__device__ __forceinline__ void attend_block(WarpAttn<D> &st, uint32_t ks, uint32_t vs, bool valid0, bool valid8,
                                             float scale_log2, int lane) {
    constexpr int KT = D / 16;
    // S^T = K . Q^T
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    {
        const int krow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
            uint32_t a[4];
            ldmatrix_x4(a, ks + swz<D>(krow, kk * 2 + (lane >> 4)));
            mma_bf16_16816(s, a, st.qf[kk][0], st.qf[kk][1]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) s[i] *= scale_log2;
    if (!valid0) s[0] = s[1] = -INFINITY;
    if (!valid8) s[2] = s[3] = -INFINITY;

    float mx[2] = {fmaxf(s[0], s[2]), fmaxf(s[1], s[3])};
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xFFFFFFFFu, mx[0], o));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xFFFFFFFFu, mx[1], o));
    }
    float alpha[2], mref[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float mn = fmaxf(st.m[i], mx[i]);
        mref[i] = mn == -INFINITY ? 0.f : mn;
        alpha[i] = fast_exp2(st.m[i] - mref[i]);  // exp2(-inf) = 0 on the first valid block
        st.m[i] = mn;
    }
    const float p0 = fast_exp2(s[0] - mref[0]), p1 = fast_exp2(s[1] - mref[1]);
    const float p2 = fast_exp2(s[2] - mref[0]), p3 = fast_exp2(s[3] - mref[1]);
    st.l[0] = st.l[0] * alpha[0] + p0 + p2;
    st.l[1] = st.l[1] * alpha[1] + p1 + p3;
    // the running max moves on few blocks: skip the rescale when no head's did
    if (__any_sync(0xFFFFFFFFu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int md = 0; md < KT; ++md) {
            st.o[md][0] *= alpha[0];
            st.o[md][1] *= alpha[1];
            st.o[md][2] *= alpha[0];
            st.o[md][3] *= alpha[1];
        }
    }
    // P^T (keys x heads) -> B operand (k = keys, n = heads)
    const uint32_t b0 = movmatrix_trans(pack_bf16x2(p0, p1));
    const uint32_t b1 = movmatrix_trans(pack_bf16x2(p2, p3));
    // O^T += V^T . P^T
    const int vrow = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
    for (int md = 0; md < KT; ++md) {
        uint32_t a[4];
        ldmatrix_x4_trans(a, vs + swz<D>(vrow, md * 2 + ((lane >> 3) & 1)));
        mma_bf16_16816(st.o[md], a, b0, b1);
    }
}

// Query fragments of the group's heads (B operand of S^T = K . Q^T):
// qf[kk][0] = Q[head gid][kk*16 + 2*tig .. +1], qf[kk][1] = same dims + 8.
template <int D>
__device__ __forceinline__ void load_q(WarpAttn<D> &st, const uint16_t *Qg, int G, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint16_t *p = Qg + (size_t)gid * D + kk * 16 + tig * 2;
        st.qf[kk][0] = gid < G ? __ldg(reinterpret_cast<const uint32_t *>(p)) : 0u;
        st.qf[kk][1] = gid < G ? __ldg(reinterpret_cast<const uint32_t *>(p + 8)) : 0u;
    }
#pragma unroll
    for (int md = 0; md < D / 16; ++md)
#pragma unroll
        for (int i = 0; i < 4; ++i) st.o[md][i] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
}

// Run the pipelined gather + attend loop over the entries [e_begin, e_end)
// of one index row.  resolve(s) maps a selected token index to the element
// offset of its K/V row for this group, or -1 when the entry is to be
// skipped (outside the visible range, or on an unmapped page).
template <int D, typename Resolve>
__device__ __forceinline__ void attend_range(WarpAttn<D> &st, uint8_t *wsmem, const int32_t *idx_row, int e_begin,
                                             int e_end, const uint16_t *K, const uint16_t *V, float scale_log2,
                                             Resolve resolve, int lane) {
    const uint32_t base = smem_u32(wsmem);
    const int nblk = (e_end - e_begin + kBlk - 1) / kBlk;
    uint64_t vmasks = 0;  // 16-bit validity mask per stage
    auto issue = [&](int blk) {
        const int st_i = blk % kStages;
        int64_t rowaddr = 0;
        bool valid = false;
        if (lane < kBlk) {
            const int e = e_begin + blk * kBlk + lane;
            if (e < e_end) {
                const int64_t a = resolve(__ldg(idx_row + e));
                valid = a >= 0;
                rowaddr = valid ? a : 0;
            }
        }
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, valid) & 0xFFFFu;
        vmasks = (vmasks & ~(0xFFFFull << (16 * st_i))) | ((uint64_t)m << (16 * st_i));
        const uint32_t ks = base + st_i * stage_bytes<D>();
        gather_block<D>(ks, ks + kBlk * D * 2, K, V, rowaddr, lane);
    };
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) {
        if (i < nblk) issue(i);
        cp_async_commit();
    }
    const int gid = lane >> 2;
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk + kStages - 1 < nblk) issue(blk + kStages - 1);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const int st_i = blk % kStages;
        const uint32_t m = (uint32_t)(vmasks >> (16 * st_i)) & 0xFFFFu;
        const uint32_t ks = base + st_i * stage_bytes<D>();
        attend_block<D>(st, ks, ks + kBlk * D * 2, (m >> gid) & 1u, (m >> (gid + 8)) & 1u, scale_log2, lane);
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();
}

template <int D>
__device__ __forceinline__ void reduce_sums(WarpAttn<D> &st) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        st.l[0] += __shfl_xor_sync(0xFFFFFFFFu, st.l[0], o);
        st.l[1] += __shfl_xor_sync(0xFFFFFFFFu, st.l[1], o);
    }
}

template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32) sparse_prefill_kernel(
    const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K, const uint16_t *__restrict__ V,
    const int32_t *__restrict__ idx, int row_begin, int n_rows, int Hq, int Hkv, int k, float scale_log2,
    uint16_t *__restrict__ O, float *__restrict__ lse, int group_major, const int32_t *__restrict__ cu, int nseq) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int pair = blockIdx.x * kWarpsPerCta + warp;
    if (pair >= n_rows * Hkv) return;
    // group-major: the warps resident at one time share one KV group, whose
    // K and V rows then fit in L2 even when the whole K and V do not
    const int r = group_major ? pair % n_rows : pair / Hkv;
    const int g = group_major ? pair / n_rows : pair % Hkv;
    const int t = row_begin + r;
    const int G = Hq / Hkv;
    uint8_t *wsmem = smem + warp * warp_smem_bytes<D>();

    WarpAttn<D> st;
    load_q<D>(st, Q + ((size_t)r * Hq + (size_t)g * G) * D, G, lane);
    // packed sequences: row t attends to positions 0..t-start of its own
    // sequence, i.e. tokens start..t (start = 0 for a single sequence)
    const int start = seq_start(cu, nseq, t);
    const int n_vis = min(k, t - start + 1);
    attend_range<D>(
        st, wsmem, idx + (size_t)r * k, 0, n_vis, K, V, scale_log2,
        [&](int32_t s) -> int64_t {
            return (s >= 0 && s <= t - start) ? ((int64_t)(start + s) * Hkv + g) * D : -1;
        },
        lane);
    reduce_sums<D>(st);

    // Normalise, stage the group's [G, D] output tile in shared memory, then
    // write it with 16-byte stores (the G heads of a group are contiguous).
    const int gid = lane >> 2, tig = lane & 3;
    const float inv0 = st.l[0] > 0.f ? 1.f / st.l[0] : 0.f;
    const float inv1 = st.l[1] > 0.f ? 1.f / st.l[1] : 0.f;
    uint16_t *os = reinterpret_cast<uint16_t *>(wsmem);
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
        const int d0 = md * 16 + gid;
        os[(2 * tig) * D + d0] = float_to_bf16_bits(st.o[md][0] * inv0);
        os[(2 * tig + 1) * D + d0] = float_to_bf16_bits(st.o[md][1] * inv1);
        os[(2 * tig) * D + d0 + 8] = float_to_bf16_bits(st.o[md][2] * inv0);
        os[(2 * tig + 1) * D + d0 + 8] = float_to_bf16_bits(st.o[md][3] * inv1);
    }
    __syncwarp();
    uint4 *dst = reinterpret_cast<uint4 *>(O + ((size_t)r * Hq + (size_t)g * G) * D);
    const uint4 *src = reinterpret_cast<const uint4 *>(os);
    for (int i = lane; i < G * D / 8; i += 32) dst[i] = src[i];
    if (lse != nullptr && gid == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int h = 2 * tig + i;
            if (h < G) {
                const float v = st.l[i] > 0.f ? (st.m[i] + __log2f(st.l[i])) * kLn2 : -INFINITY;
                lse[(size_t)r * Hq + (size_t)g * G + h] = v;
            }
        }
    }
}

// Decode split-K partial: rows [sp*chunk, min(k, (sp+1)*chunk)) of the index
// row of sequence b, group g.  Writes, per head h < 8, D unnormalised output
// values followed by the running max (log2 domain) and the sum of weights.
template <int D>
__global__ void __launch_bounds__(kWarpsPerCta * 32) sparse_decode_split_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ k_cache, const uint16_t *__restrict__ v_cache,
    const int32_t *__restrict__ block_table, int max_pages, int num_pages, const int32_t *__restrict__ seq_lens,
    const int32_t *__restrict__ idx, int B, int Hq, int Hkv, int k, int chunk, int nsplit, float scale_log2,
    float *__restrict__ part) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int item = blockIdx.x * kWarpsPerCta + warp;
    if (item >= B * Hkv * nsplit) return;
    const int sp = item % nsplit, bg = item / nsplit;
    const int b = bg / Hkv, g = bg % Hkv;
    const int G = Hq / Hkv;
    uint8_t *wsmem = smem + warp * warp_smem_bytes<D>();
    const int n = min(__ldg(seq_lens + b), max_pages * kPage);
    const int n_vis = min(k, n);
    const int e0 = min(sp * chunk, n_vis), e1 = min(e0 + chunk, n_vis);

    WarpAttn<D> st;
    load_q<D>(st, q + ((size_t)b * Hq + (size_t)g * G) * D, G, lane);
    const int32_t *bt = block_table + (size_t)b * max_pages;
    attend_range<D>(
        st, wsmem, idx + (size_t)b * k, e0, e1, k_cache, v_cache, scale_log2,
        [&](int32_t s) -> int64_t {
            if (s < 0 || s >= n) return -1;
            const int page = __ldg(bt + s / kPage);
            if (page < 0 || page >= num_pages) return -1;
            return (((int64_t)page * kPage + s % kPage) * Hkv + g) * D;
        },
        lane);
    reduce_sums<D>(st);

    const int gid = lane >> 2, tig = lane & 3;
    float *pb = part + (size_t)item * 8 * (D + 2);
#pragma unroll
    for (int md = 0; md < D / 16; ++md) {
        const int d0 = md * 16 + gid;
        pb[(2 * tig) * (D + 2) + d0] = st.o[md][0];
        pb[(2 * tig + 1) * (D + 2) + d0] = st.o[md][1];
        pb[(2 * tig) * (D + 2) + d0 + 8] = st.o[md][2];
        pb[(2 * tig + 1) * (D + 2) + d0 + 8] = st.o[md][3];
    }
    if (gid == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            pb[(2 * tig + i) * (D + 2) + D] = st.m[i];
            pb[(2 * tig + i) * (D + 2) + D + 1] = st.l[i];
        }
    }
}

// Merge the split-K partials of one (sequence, head): one CTA of D threads.
// The splits' running maxima are loaded in parallel and reduced; then each
// thread folds the splits in order, eight at a time with their loads issued
// together (the partials sit in L2, so a load-per-step chain would pay the
// L2 latency once per split).
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const float *__restrict__ part, int Hq, int Hkv,
                                                           int nsplit, uint16_t *__restrict__ out,
                                                           float *__restrict__ lse) {
    constexpr int kBatch = 8;
    __shared__ float red[D / 32];
    const int bh = blockIdx.x;
    const int b = bh / Hq, h = bh % Hq;
    const int G = Hq / Hkv, g = h / G, hh = h % G;
    const float *p0 = part + ((size_t)(b * Hkv + g) * nsplit) * 8 * (D + 2) + (size_t)hh * (D + 2);
    const size_t stride = (size_t)8 * (D + 2);
    const int d = threadIdx.x;
    float M = -INFINITY;
    for (int sp = d; sp < nsplit; sp += D) M = fmaxf(M, p0[sp * stride + D]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
    if ((d & 31) == 0) red[d >> 5] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < D / 32; ++w) M = fmaxf(M, red[w]);
    const float Mref = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc = 0.f;
    for (int sp0 = 0; sp0 < nsplit; sp0 += kBatch) {
        float pv[kBatch], mv[kBatch], lv[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const float *p = p0 + (size_t)min(sp0 + j, nsplit - 1) * stride;
            pv[j] = p[d];
            mv[j] = p[D];
            lv[j] = p[D + 1];
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            if (sp0 + j < nsplit) {
                const float f = fast_exp2(mv[j] - Mref);
                L = fmaf(lv[j], f, L);
                acc = fmaf(pv[j], f, acc);
            }
        }
    }
    out[(size_t)bh * D + d] = float_to_bf16_bits(L > 0.f ? acc / L : 0.f);
    if (lse != nullptr && d == 0) lse[bh] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
}

struct DecodeSplit {
    int chunk, nsplit;
};

// Upper bound on resident split warps that workspaces are sized for (148
// SMs x 16 warps); a launch never uses more splits than this allows.
constexpr int kSplitSlotsBound = 148 * 16;

// Split the k index rows of each (sequence, group) pair so that all pairs'
// warps are resident at once (`slots` = warps the device holds): one wave,
// no tail of a few warps running alone.  Chunks are 16-key aligned.
DecodeSplit decode_split(int B, int Hkv, int k, int slots) {
    const int pairs = B * Hkv > 0 ? B * Hkv : 1;
    int want = slots / pairs;
    const int max_split = (k + kBlk - 1) / kBlk;
    want = want < 1 ? 1 : (want > max_split ? max_split : want);
    int chunk = (k + want - 1) / want;
    chunk = (chunk + kBlk - 1) / kBlk * kBlk;
    const int nsplit = (k + chunk - 1) / chunk;
    return {chunk, nsplit};
}

template <typename F>
bool dispatch_d(int D, F &&f) {
    switch (D) {
        case 64: return f(std::integral_constant<int, 64>{});
        case 128: return f(std::integral_constant<int, 128>{});
        default: return false;
    }
}

// Split warps the current device holds at once (SMs x resident one-warp
// CTAs of the split kernel), looked up once per device, at most
// kSplitSlotsBound.
template <int D>
int decode_split_slots() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return kSplitSlotsBound;
    int v = cached[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        constexpr int smem = kWarpsPerCta * warp_smem_bytes<D>();
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            set_smem_at_least<sparse_decode_split_kernel<D>>(smem) == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sparse_decode_split_kernel<D>,
                                                          kWarpsPerCta * 32, smem) == cudaSuccess &&
            sms > 0 && per_sm > 0)
            v = sms * per_sm * kWarpsPerCta;
        else
            v = kSplitSlotsBound;
        cached[dev].store(v, std::memory_order_relaxed);
    }
    return v < kSplitSlotsBound ? v : kSplitSlotsBound;
}

int decode_split_slots_for(int D) { return D == 64 ? decode_split_slots<64>() : decode_split_slots<128>(); }

}  // namespace

bool attention_shape_supported(int Hq, int Hkv, int D) {
    return Hkv >= 1 && Hq >= Hkv && Hq % Hkv == 0 && Hq / Hkv <= 8 && (D == 64 || D == 128);
}

cudaError_t launch_sparse_prefill(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const int32_t *idx,
                                  int row_begin, int n_rows, int Hq, int Hkv, int D, int k, float sm_scale,
                                  uint16_t *O, float *lse, cudaStream_t stream, const int32_t *cu, int nseq) {
    if (n_rows == 0) return cudaSuccess;
    const int64_t pairs = (int64_t)n_rows * Hkv;
    const int grid = (int)((pairs + kWarpsPerCta - 1) / kWarpsPerCta);
    // Walk the pairs group by group once the visible K and V rows outgrow
    // half of L2 (at 128K tokens they are 268 MB; one group's share fits).
    const int64_t kv_bytes = 2ll * (row_begin + n_rows) * Hkv * D * 2;
    const bool group_major = Hkv > 1 && kv_bytes > (64ll << 20);
    cudaError_t err = cudaSuccess;
    const bool ok = dispatch_d(D, [&](auto dc) {
        constexpr int DD = decltype(dc)::value;
        constexpr int smem = kWarpsPerCta * warp_smem_bytes<DD>();
        err = set_smem_at_least<sparse_prefill_kernel<DD>>(smem);
        if (err != cudaSuccess) return true;
        sparse_prefill_kernel<DD><<<grid, kWarpsPerCta * 32, smem, stream>>>(Q, K, V, idx, row_begin, n_rows, Hq,
                                                                             Hkv, k, sm_scale * kLog2e, O, lse,
                                                                             group_major ? 1 : 0, cu, nseq);
        err = cudaGetLastError();
        return true;
    });
    return ok ? err : cudaErrorInvalidValue;
}

size_t decode_attention_workspace_bytes(int B, int Hq, int Hkv, int D, int k) {
    (void)Hq;
    const DecodeSplit s = decode_split(B, Hkv, k, kSplitSlotsBound);
    return (size_t)B * Hkv * s.nsplit * 8 * (D + 2) * sizeof(float);
}

cudaError_t launch_sparse_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                 const int32_t *block_table, int max_pages, int num_pages, const int32_t *seq_lens,
                                 const int32_t *idx, int B, int Hq, int Hkv, int D, int k, float sm_scale, void *ws,
                                 size_t ws_bytes, uint16_t *out, float *lse, cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    if (ws_bytes < decode_attention_workspace_bytes(B, Hq, Hkv, D, k)) return cudaErrorInvalidValue;
    if (D != 64 && D != 128) return cudaErrorInvalidValue;
    const DecodeSplit s = decode_split(B, Hkv, k, decode_split_slots_for(D));
    const int items = B * Hkv * s.nsplit;
    const int grid = (items + kWarpsPerCta - 1) / kWarpsPerCta;
    float *part = static_cast<float *>(ws);
    cudaError_t err = cudaSuccess;
    const bool ok = dispatch_d(D, [&](auto dc) {
        constexpr int DD = decltype(dc)::value;
        constexpr int smem = kWarpsPerCta * warp_smem_bytes<DD>();
        err = set_smem_at_least<sparse_decode_split_kernel<DD>>(smem);
        if (err != cudaSuccess) return true;
        sparse_decode_split_kernel<DD><<<grid, kWarpsPerCta * 32, smem, stream>>>(
            q, k_cache, v_cache, block_table, max_pages, num_pages, seq_lens, idx, B, Hq, Hkv, k, s.chunk, s.nsplit,
            sm_scale * kLog2e, part);
        err = cudaGetLastError();
        if (err != cudaSuccess) return true;
        decode_combine_kernel<DD><<<B * Hq, DD, 0, stream>>>(part, Hq, Hkv, s.nsplit, out, lse);
        err = cudaGetLastError();
        return true;
    });
    return ok ? err : cudaErrorInvalidValue;
}

}  // namespace dsa

// ---------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// The split-K partials of the decode attention normally live in a workspace
// the caller allocates.  This variant keeps them in a fixed array that is part
// of the library image instead: every GPU that loads the library holds
// kFixedScratchBytes of it until the process exits.  All calls on a device
// share the array, so calls whose executions overlap on that device race.
// Every partial the combine pass reads is written by the split pass of the
// same call, so nothing has to be cleared between calls.
// ---------------------------------------------------------------------------

namespace dsa {
constexpr size_t kFixedScratchBytes = size_t(8) << 20;  // 8 MiB
}  // namespace dsa

static __device__ __align__(256) float g_decode_fixed_scratch[dsa::kFixedScratchBytes / sizeof(float)];

namespace dsa {

namespace {

// Device address of g_decode_fixed_scratch on the current device.  In host
// code the array's name is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
float *fixed_scratch_on_current_device(cudaError_t *err) {
    constexpr int kMaxDevices = 64;
    static std::atomic<float *> cached[kMaxDevices];
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= kMaxDevices) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    float *p = cached[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        void *addr = nullptr;
        *err = cudaGetSymbolAddress(&addr, g_decode_fixed_scratch);
        if (*err != cudaSuccess) return nullptr;
        p = static_cast<float *>(addr);
        cached[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

size_t fixed_scratch_bytes() { return kFixedScratchBytes; }

// Largest split count whose partials fit the fixed array (0 if even one split
// does not fit).
int fixed_scratch_max_split(int B, int Hkv, int D) {
    const size_t per_split = (size_t)B * Hkv * 8 * (D + 2) * sizeof(float);
    if (per_split == 0) return 1 << 30;
    const size_t n = kFixedScratchBytes / per_split;
    return n > (size_t)(1 << 30) ? (1 << 30) : (int)n;
}

cudaError_t launch_sparse_decode_fixed_scratch(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                                               const int32_t *block_table, int max_pages, int num_pages,
                                               const int32_t *seq_lens, const int32_t *idx, int B, int Hq, int Hkv,
                                               int D, int k, float sm_scale, uint16_t *out, float *lse,
                                               cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    const int cap = fixed_scratch_max_split(B, Hkv, D);
    if (cap < 1) return cudaErrorInvalidValue;
    cudaError_t err = cudaSuccess;
    float *part = fixed_scratch_on_current_device(&err);
    if (part == nullptr) return err;
    // Same split rule as the workspace variant, capped so the partials fit.
    if (D != 64 && D != 128) return cudaErrorInvalidValue;
    DecodeSplit s = decode_split(B, Hkv, k, decode_split_slots_for(D));
    if (s.nsplit > cap) {
        int chunk = (k + cap - 1) / cap;
        chunk = (chunk + kBlk - 1) / kBlk * kBlk;
        s = {chunk, (k + chunk - 1) / chunk};
    }
    const int items = B * Hkv * s.nsplit;
    const int grid = (items + kWarpsPerCta - 1) / kWarpsPerCta;
    const bool ok = dispatch_d(D, [&](auto dc) {
        constexpr int DD = decltype(dc)::value;
        constexpr int smem = kWarpsPerCta * warp_smem_bytes<DD>();
        err = cudaFuncSetAttribute(sparse_decode_split_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   smem);
        if (err != cudaSuccess) return true;
        sparse_decode_split_kernel<DD><<<grid, kWarpsPerCta * 32, smem, stream>>>(
            q, k_cache, v_cache, block_table, max_pages, num_pages, seq_lens, idx, B, Hq, Hkv, k, s.chunk, s.nsplit,
            sm_scale * kLog2e, part);
        err = cudaGetLastError();
        if (err != cudaSuccess) return true;
        decode_combine_kernel<DD><<<B * Hq, DD, 0, stream>>>(part, Hq, Hkv, s.nsplit, out, lse);
        err = cudaGetLastError();
        return true;
    });
    return ok ? err : cudaErrorInvalidValue;
}

}  // namespace dsa
