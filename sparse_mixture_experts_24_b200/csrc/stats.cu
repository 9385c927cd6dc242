// stats.cu -- the router's load-balancing statistics, as the Switch
// Transformers load-balancing loss uses them ("Mixture of Experts: Why Mixtral
// Only Wakes Up Two Specialists", Part 5, "Tool 2: a fine for favouritism"):
//   f_i = share of the routed (token, slot) pairs sent to expert i,
//   P_i = average over the tokens of the router probability of expert i
//         (softmax over all n logits),
//   aux = alpha * n * sum_i f_i * P_i.
// Deterministic: every float sum runs in a fixed order (lanes own experts,
// warps own fixed token subsets, blocks are summed in block order); the
// expert counts are integer atomics.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kStatsTokens = 256;  // tokens per block

// Block b: P partial sums over its tokens -> partial[b][n]; expert counts of
// its (token, slot) pairs -> atomics into counts[n].
__global__ void __launch_bounds__(256) stats_partial_kernel(const float* __restrict__ logits, int splits,
                                                            int64_t T, int n, int K,
                                                            const int32_t* __restrict__ idx,
                                                            float* __restrict__ partial,
                                                            int32_t* __restrict__ counts) {
    griddep_wait();
    __shared__ float red[8][256];
    __shared__ int32_t hist[256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < n; e += 256) hist[e] = 0;
    __syncthreads();
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kStatsTokens;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = warp; j < kStatsTokens; j += 8) {
        const int64_t t = t0 + j;
        if (t >= T) break;
        float v[8];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            float a = 0.f;
            if (e < n)
                for (int sp = 0; sp < splits; ++sp) a += logits[(static_cast<int64_t>(sp) * T + t) * n + e];
            v[i] = (e < n) ? a : -INFINITY;
            m = fmaxf(m, v[i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] = (lane + 32 * i < n) ? expf(v[i] - m) : 0.f;
            z += v[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const float inv = 1.f / z;
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i] * inv;
        if (lane < K) {
            const int e = idx[t * K + lane];
            if (e >= 0 && e < n) atomicAdd(&hist[e], 1);
        }
        if (K > 32)
            for (int k = 32 + lane; k < K; k += 32) {
                const int e = idx[t * K + k];
                if (e >= 0 && e < n) atomicAdd(&hist[e], 1);
            }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < n) red[warp][lane + 32 * i] = acc[i];
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += 256) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w][e];
        partial[static_cast<int64_t>(blockIdx.x) * n + e] = s;
        if (hist[e]) atomicAdd(&counts[e], hist[e]);
    }
    griddep_launch_dependents();
}

__global__ void __launch_bounds__(256) stats_final_kernel(const float* __restrict__ partial, int nblk,
                                                          int64_t T, int n, int K, float alpha,
                                                          const int32_t* __restrict__ counts,
                                                          float* __restrict__ f, float* __restrict__ P,
                                                          float* __restrict__ aux) {
    griddep_wait();
    __shared__ float fp[256];
    const int e = threadIdx.x;
    float prod = 0.f;
    if (e < n) {
        float s = 0.f;
        for (int b = 0; b < nblk; ++b) s += partial[static_cast<int64_t>(b) * n + e];
        const float pe = s / static_cast<float>(T);
        const float fe = static_cast<float>(counts[e]) / static_cast<float>(T * K);
        P[e] = pe;
        f[e] = fe;
        prod = fe * pe;
    }
    fp[e] = prod;
    __syncthreads();
    if (e == 0) {
        float s = 0.f;
        for (int i = 0; i < n; ++i) s += fp[i];
        aux[0] = alpha * static_cast<float>(n) * s;
    }
    griddep_launch_dependents();
}

cudaError_t launch_router_stats(const float* logits, int splits, int64_t T, int n, int K,
                                const int32_t* topk_idx, float alpha, float* partial,
                                int32_t* counts, float* f, float* P, float* aux, cudaStream_t st) {
    const int nblk = static_cast<int>((T + kStatsTokens - 1) / kStatsTokens);
    cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * n, st);
    if (e != cudaSuccess) return e;
    launch_k(stats_partial_kernel, dim3(nblk), dim3(256), 0, st, logits, splits, T, n, K, topk_idx, partial, counts);
    launch_k(stats_final_kernel, dim3(1), dim3(256), 0, st, partial, nblk, T, n, K, alpha, counts, f, P, aux);
    return cudaGetLastError();
}

}  // namespace moe
