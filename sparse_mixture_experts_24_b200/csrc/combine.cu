// combine.cu -- the gate-weighted additive combine: y[t] = sum_k g[t][k] *
// O[row of (t, k)], accumulated in fp32 in slot order k = 0..K-1 (a fixed
// order, so the result is deterministic; no atomics).
//
// Source: "Mixture of Experts: Why Mixtral Only Wakes Up Two Specialists",
// Part 3, Step 4 (each chosen expert's output is multiplied by its weight and
// the products are added), and the sum over experts in the layer equation of
// "Mixtral of Experts" section 2.1.
//
// One thread per 16-byte vector of y (grid-stride): it reads the K matching
// vectors of O and writes one vector of y, so every load of a small batch is
// in flight at once and large batches stream at HBM speed.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// kChunk slots at a time: their row indices and gates are loaded first, then
// all their O vectors, so that a thread has kChunk loads of O in flight (the
// row lookups make each load depend on an earlier one); the products are
// still added in slot order.
template <int kChunk>
__global__ void __launch_bounds__(256) combine_bf16_kernel(const uint4* __restrict__ O,
                                                           const int32_t* __restrict__ token_row,
                                                           const float* __restrict__ topk_w,
                                                           int64_t T, int K, int vec_per_row,
                                                           uint4* __restrict__ y) {
    griddep_wait();
    const int64_t total = T * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
        const int64_t t = i / vec_per_row;
        const int64_t v = i - t * vec_per_row;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int k0 = 0; k0 < K; k0 += kChunk) {
            int32_t r[kChunk];
            float g[kChunk];
            uint4 o[kChunk];
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
                const bool in = k0 + j < K;
                r[j] = in ? __ldg(token_row + t * K + k0 + j) : -1;
                g[j] = in ? __ldg(topk_w + t * K + k0 + j) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < kChunk; ++j)
                o[j] = r[j] >= 0 ? __ldg(O + static_cast<int64_t>(r[j]) * vec_per_row + v) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j = 0; j < kChunk; ++j)
                if (r[j] >= 0) fma_bf16x8(acc, g[j], o[j]);
        }
        y[i] = pack_bf16x8(acc);
    }
    griddep_launch_dependents();
}

__global__ void __launch_bounds__(256) combine_f32_kernel(const float4* __restrict__ O,
                                                          const int32_t* __restrict__ token_row,
                                                          const float* __restrict__ topk_w,
                                                          int64_t T, int K, int vec_per_row,
                                                          float4* __restrict__ y) {
    griddep_wait();
    const int64_t total = T * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
        const int64_t t = i / vec_per_row;
        const int64_t v = i - t * vec_per_row;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < K; ++k) {
            const int32_t r = __ldg(token_row + t * K + k);
            if (r < 0) continue;
            const float g = __ldg(topk_w + t * K + k);
            const float4 q = __ldg(O + static_cast<int64_t>(r) * vec_per_row + v);
            acc.x = fmaf(g, q.x, acc.x);
            acc.y = fmaf(g, q.y, acc.y);
            acc.z = fmaf(g, q.z, acc.z);
            acc.w = fmaf(g, q.w, acc.w);
        }
        y[i] = acc;
    }
    griddep_launch_dependents();
}

cudaError_t launch_combine(const void* O, bool bf16, const int32_t* token_row, const float* topk_w,
                           int64_t T, int K, int d, void* y, int num_sms, cudaStream_t st) {
    const int64_t vecs = T * (bf16 ? d / 8 : d / 4);
    int64_t blocks = (vecs + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (bf16) {
        const dim3 grid(static_cast<unsigned>(blocks));
        const uint4* o = static_cast<const uint4*>(O);
        uint4* yv = static_cast<uint4*>(y);
        if (K == 1)
            launch_k(combine_bf16_kernel<1>, grid, dim3(256), 0, st, o, token_row, topk_w, T, K, d / 8, yv);
        else if (K == 2)
            launch_k(combine_bf16_kernel<2>, grid, dim3(256), 0, st, o, token_row, topk_w, T, K, d / 8, yv);
        else
            launch_k(combine_bf16_kernel<4>, grid, dim3(256), 0, st, o, token_row, topk_w, T, K, d / 8, yv);
    } else
        launch_k(combine_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, 
            static_cast<const float4*>(O), token_row, topk_w, T, K, d / 4, static_cast<float4*>(y));
    return cudaGetLastError();
}

}  // namespace moe
