// indexer_kl.cu -- the indexer's distillation losses, forward only.
//
// "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式:
//     dense warm-up     L = sum_t sum_g KL( p[t,:,g]   || Softmax(I[t,:])   )
//     sparse adaptation L = sum_t sum_g KL( p[t,S_t,g] || Softmax(I[t,S_t]) )
// report translation section 2.3.3: p[t,:,g] is group g's aggregated dense
// attention, normalised; in the sparse stage it is truncated to the selected
// set S_t and renormalised, and the softmax runs over S_t.
//
// One CTA per query row.  With S = sum_s p_s, A = sum_s p_s ln p_s and
// B = sum_s p_s I_s over the set, m = max I and Z = sum exp(I_s - m):
//     KL_g = A / S - ln S - (B / S - m - ln Z)
// (the normalised target p/S against log Softmax = I - m - ln Z).  Every sum
// is accumulated in fp64 from the fp32 inputs, in a fixed order per thread
// and a fixed tree across threads, so the result does not depend on
// scheduling.  A group without target mass on the set contributes 0.
#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kKlThreads = 256;
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlGroupsPerPass = 4;

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Sum of one value per thread over the block (fixed order); every thread
// gets the result.  red holds kKlWarps doubles.
__device__ __forceinline__ double block_sum_d(double v, double *red) {
    v = warp_sum(v);
    if (lane_id() == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < kKlWarps; ++w) s += red[w];
    __syncthreads();
    return s;
}

__global__ void __launch_bounds__(kKlThreads) indexer_kl_kernel(const float *__restrict__ scores, int64_t ld,
                                                               int row_begin, const float *__restrict__ p, int G,
                                                               int64_t ld_p, const int32_t *__restrict__ idx, int k,
                                                               double *__restrict__ loss) {
    __shared__ double red[kKlWarps];
    __shared__ float fred[kKlWarps];
    const int r = blockIdx.x, tid = threadIdx.x;
    const int t = row_begin + r;
    const int n = idx ? k : t + 1;  // entries to visit
    const float *Ir = scores + (size_t)r * ld;
    auto key = [&](int i) -> int { return idx ? __ldg(idx + (size_t)r * k + i) : i; };

    // the largest score over the set
    float mx = -INFINITY;
    for (int i = tid; i < n; i += kKlThreads) {
        const int s = key(i);
        if (s >= 0 && s <= t) mx = fmaxf(mx, __ldg(Ir + s));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane_id() == 0) fred[tid >> 5] = mx;
    __syncthreads();
    mx = fred[0];
#pragma unroll
    for (int w = 1; w < kKlWarps; ++w) mx = fmaxf(mx, fred[w]);
    if (mx == -INFINITY) {  // no key in the set
        if (tid == 0) loss[r] = 0.0;
        return;
    }
    const double m = (double)mx;

    double row_loss = 0.0, logz = 0.0;
    for (int g0 = 0; g0 < G; g0 += kKlGroupsPerPass) {
        double z = 0.0, S[kKlGroupsPerPass], A[kKlGroupsPerPass], B[kKlGroupsPerPass];
#pragma unroll
        for (int j = 0; j < kKlGroupsPerPass; ++j) S[j] = A[j] = B[j] = 0.0;
        for (int i = tid; i < n; i += kKlThreads) {
            const int s = key(i);
            if (s < 0 || s > t) continue;
            const double x = (double)__ldg(Ir + s);
            if (g0 == 0) z += exp(x - m);
#pragma unroll
            for (int j = 0; j < kKlGroupsPerPass; ++j) {
                if (g0 + j < G) {
                    const double pv = (double)__ldg(p + ((size_t)r * G + g0 + j) * ld_p + s);
                    S[j] += pv;
                    if (pv > 0.0) A[j] += pv * log(pv);
                    B[j] += pv * x;
                }
            }
        }
        if (g0 == 0) logz = log(block_sum_d(z, red));
#pragma unroll
        for (int j = 0; j < kKlGroupsPerPass; ++j) {
            if (g0 + j >= G) break;
            const double Sg = block_sum_d(S[j], red);
            const double Ag = block_sum_d(A[j], red);
            const double Bg = block_sum_d(B[j], red);
            if (Sg > 0.0) row_loss += (Ag / Sg - log(Sg)) - (Bg / Sg - m - logz);
        }
    }
    if (tid == 0) loss[r] = row_loss;
}

// The total over rows in a fixed order: thread i sums rows i, i + 512, ...,
// then a fixed tree.
__global__ void __launch_bounds__(512) kl_total_kernel(const double *__restrict__ loss, int n_rows,
                                                       double *__restrict__ total) {
    __shared__ double part[512];
    double s = 0.0;
    for (int i = threadIdx.x; i < n_rows; i += 512) s += loss[i];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 256; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *total = part[0];
}

}  // namespace

cudaError_t launch_indexer_kl(const float *scores, int64_t ld, int row_begin, int n_rows, const float *p, int G,
                              int64_t ld_p, const int32_t *idx, int k, double *loss_rows, double *loss_total,
                              cudaStream_t stream) {
    if (n_rows > 0) {
        indexer_kl_kernel<<<n_rows, kKlThreads, 0, stream>>>(scores, ld, row_begin, p, G, ld_p, idx, k, loss_rows);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (loss_total != nullptr) {
        kl_total_kernel<<<1, 512, 0, stream>>>(loss_rows, n_rows, loss_total);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace dsa
