// router.cu -- the MoE gate on CUDA cores in fp32: logits L = x . W_g, the K
// largest logits per token (descending; equal logits keep the lower expert
// index), and the softmax over those K.
//
// Source: "Mixture of Experts: Why Mixtral Only Wakes Up Two Specialists",
// Part 3, Step 1 (a bias-free linear layer scores every expert), Step 2 (keep
// the two highest scores and their positions) and Step 3 (softmax over the two
// kept scores); the layer equation of "Mixtral of Experts" section 2.1 (the
// dropped logits are -inf, so the softmax runs over the kept ones only).
//
// Kernels:
//   router_token_kernel  n <= 32, T < 512: one block per token (up to 1,024
//                        threads), W_g rows read straight from global memory,
//                        block reduction.
//   router_small_kernel  n <= 32: W_g staged through shared memory transposed
//                        to [expert][row]; one warp per group of TPW tokens,
//                        the lanes split d four rows at a time, every lane
//                        keeps all n partial logits of its tokens in
//                        registers, a shuffle butterfly sums them, lane 0
//                        picks the top K.
//   router_logits_kernel + router_topk_kernel  n > 32: a 64x64 register-tiled
//                        fp32 GEMM writes the logits to the workspace, then a
//                        warp per token selects the top K with shuffles.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace moe {

// 4 consecutive x elements widened to fp32 (8 bytes of bf16, 16 of fp32).
template <typename XT>
__device__ __forceinline__ void load_x4(const XT* p, float (&v)[4]);

template <>
__device__ __forceinline__ void load_x4<uint16_t>(const uint16_t* p, float (&v)[4]) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    unpack_bf16x2(q.x, v[0], v[1]);
    unpack_bf16x2(q.y, v[2], v[3]);
}

template <>
__device__ __forceinline__ void load_x4<float>(const float* p, float (&v)[4]) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = q.x;
    v[1] = q.y;
    v[2] = q.z;
    v[3] = q.w;
}

// Top-K of one token's logits held in registers (NE slots, n valid), written
// with the softmax over the kept logits.  Strict '>' while scanning upwards
// keeps the lower index on ties (NaN logits arrive here as -inf).
template <int NE>
__device__ __forceinline__ void topk_softmax_regs(const float (&L)[NE], int n, int K,
                                                  int32_t* idx_out, float* w_out) {
    uint32_t taken = 0;
    float m = 0.f, s = 0.f;
    for (int k = 0; k < K; ++k) {
        int best = -1;
        float bv = 0.f;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            if (e < n && !((taken >> e) & 1u)) {
                if (best < 0 || L[e] > bv) {
                    best = e;
                    bv = L[e];
                }
            }
        }
        taken |= 1u << best;
        if (k == 0) m = bv;
        const float ex = expf(bv - m);
        s += ex;
        idx_out[k] = best;
        w_out[k] = ex;
    }
    const float inv = 1.f / s;
    for (int k = 0; k < K; ++k) w_out[k] *= inv;
}

// Below this many tokens the router runs one block per token.
constexpr int64_t kTokenKernelMaxT = 512;

// Rows of W_g staged per pass: NE x (chunk + 4) floats stay under 48 KB.
template <int NE>
struct SmallRouterCfg {
    static constexpr int kChunk = NE <= 8 ? 1024 : (NE <= 16 ? 512 : 256);
    static constexpr int kPitch = kChunk + 4;  // floats per staged expert row
};

// n <= 32.  Each warp owns TPW tokens; W_g is staged through shared memory in
// chunks of kChunk rows, transposed to [expert][row], so that a warp reads 32
// consecutive float4 (512 contiguous bytes) per expert: lane l covers rows
// 4l .. 4l+3 of every 128-row slice of the chunk and the matching 4 columns
// of x (8 or 16 contiguous bytes per token).  Shuffles sum the lanes; lane 0
// selects the top K.
template <typename XT, int NE, int TPW>
__global__ void __launch_bounds__(256) router_small_kernel(const XT* __restrict__ x,
                                                           const float* __restrict__ Wg, int64_t T,
                                                           int d, int n, int K,
                                                           int32_t* __restrict__ topk_idx,
                                                           float* __restrict__ topk_w) {
    griddep_wait();
    using C = SmallRouterCfg<NE>;
    __shared__ __align__(16) float Ws[NE * C::kPitch];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * 8 + warp) * TPW;

    float acc[TPW][NE];
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
        for (int e = 0; e < NE; ++e) acc[t][e] = 0.f;

    for (int c0 = 0; c0 < d; c0 += C::kChunk) {
        const int rows = min(C::kChunk, d - c0);   // multiple of 64
        __syncthreads();
        if ((n & 3) == 0) {
            // float4 loads (4 experts of one row); rows * n is a multiple of 256 floats
            const float4* src = reinterpret_cast<const float4*>(Wg + static_cast<int64_t>(c0) * n);
            const int nv = rows * n / 4;
#pragma unroll 4
            for (int i = threadIdx.x; i < nv; i += 256) {
                const float4 v = __ldg(src + i);
                const int j = (i * 4) / n, e = (i * 4) - j * n;
                float* dst = &Ws[e * C::kPitch + j];
                dst[0] = v.x;
                dst[C::kPitch] = v.y;
                dst[2 * C::kPitch] = v.z;
                dst[3 * C::kPitch] = v.w;
            }
        } else {
            for (int i = threadIdx.x; i < rows * n; i += 256) {
                const int j = i / n, e = i - j * n;
                Ws[e * C::kPitch + j] = __ldg(Wg + static_cast<int64_t>(c0 + j) * n + e);
            }
        }
        __syncthreads();
        if (t0 >= T) continue;
        for (int j = lane * 4; j < rows; j += 128) {
            float xv[TPW][4];
#pragma unroll
            for (int t = 0; t < TPW; ++t) {
                if (t0 + t < T) {
                    load_x4<XT>(x + (t0 + t) * static_cast<int64_t>(d) + c0 + j, xv[t]);
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) xv[t][u] = 0.f;
                }
            }
#pragma unroll
            for (int e = 0; e < NE; ++e) {
                if (e < n) {
                    const float4 w = *reinterpret_cast<const float4*>(&Ws[e * C::kPitch + j]);
#pragma unroll
                    for (int t = 0; t < TPW; ++t) {
                        float a = acc[t][e];
                        a = fmaf(xv[t][0], w.x, a);
                        a = fmaf(xv[t][1], w.y, a);
                        a = fmaf(xv[t][2], w.z, a);
                        a = fmaf(xv[t][3], w.w, a);
                        acc[t][e] = a;
                    }
                }
            }
        }
    }
    if (t0 >= T) return;
#pragma unroll
    for (int t = 0; t < TPW; ++t)
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            float a = acc[t][e];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            acc[t][e] = (a != a) ? -INFINITY : a;  // NaN ranks lowest
        }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TPW; ++t)
            if (t0 + t < T)
                topk_softmax_regs<NE>(acc[t], n, K, topk_idx + (t0 + t) * K, topk_w + (t0 + t) * K);
    }
    griddep_launch_dependents();
}

// n <= 32, few tokens: one block per token (1,024 threads for n <= 8, 512 for
// n <= 16, else 256, so that d = 4,096 takes one or two passes and every
// thread's loads are in flight together).  Thread i covers rows 4i .. 4i+3 of
// every (4 x threads)-row slice of d, reading those rows of W_g straight from
// global memory (4n contiguous floats per thread, contiguous across the
// block); shuffles, then one lane per expert over the warps' partials in warp
// order, sum the partial logit vectors.
template <int NE>
struct TokenRouterCfg {
    static constexpr int kThreads = NE <= 8 ? 1024 : (NE <= 16 ? 512 : 256);
};

template <typename XT, int NE>
__global__ void __launch_bounds__(TokenRouterCfg<NE>::kThreads)
    router_token_kernel(const XT* __restrict__ x, const float* __restrict__ Wg, int64_t T, int d, int n, int K,
                        int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    griddep_wait();
    constexpr int kThreads = TokenRouterCfg<NE>::kThreads;
    constexpr int kWarps = kThreads / 32;
    __shared__ float red[kWarps][NE];
    __shared__ float logit[NE];
    const int64_t t = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float acc[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) acc[e] = 0.f;
    const XT* xr = x + t * static_cast<int64_t>(d);
    for (int j = threadIdx.x * 4; j < d; j += kThreads * 4) {
        float xv[4];
        load_x4<XT>(xr + j, xv);
        const float* w = Wg + static_cast<int64_t>(j) * n;
        if (n == NE) {
            // rows j .. j+3 are 4*NE contiguous floats
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < NE / 4; ++q) {
                    const float4 v = __ldg(reinterpret_cast<const float4*>(w + r * NE) + q);
                    acc[4 * q + 0] = fmaf(xv[r], v.x, acc[4 * q + 0]);
                    acc[4 * q + 1] = fmaf(xv[r], v.y, acc[4 * q + 1]);
                    acc[4 * q + 2] = fmaf(xv[r], v.z, acc[4 * q + 2]);
                    acc[4 * q + 3] = fmaf(xv[r], v.w, acc[4 * q + 3]);
                }
        } else {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int e = 0; e < NE; ++e)
                    if (e < n) acc[e] = fmaf(xv[r], __ldg(w + r * n + e), acc[e]);
        }
    }
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        float a = acc[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) red[warp][e] = a;
    }
    __syncthreads();
    if (warp == 0) {
        if (lane < NE) {
            float a = 0.f;
#pragma unroll
            for (int w8 = 0; w8 < kWarps; ++w8) a += red[w8][lane];
            logit[lane] = (a != a) ? -INFINITY : a;  // NaN ranks lowest
        }
        __syncwarp();
        if (lane == 0) {
            float L[NE];
#pragma unroll
            for (int e = 0; e < NE; ++e) L[e] = logit[e];
            topk_softmax_regs<NE>(L, n, K, topk_idx + t * K, topk_w + t * K);
        }
    }
    griddep_launch_dependents();
}

// ---- n > 32: tiled logits GEMM ---------------------------------------------
constexpr int kRT = 64;   // tokens per tile
constexpr int kRE = 64;   // experts per tile
constexpr int kRK = 32;   // d per smem chunk

template <typename XT>
__global__ void __launch_bounds__(256) router_logits_kernel(const XT* __restrict__ x,
                                                            const float* __restrict__ Wg,
                                                            int64_t T, int d, int n,
                                                            float* __restrict__ logits) {
    griddep_wait();
    __shared__ float xs[kRK][kRT + 4];
    __shared__ float ws[kRK][kRE + 4];
    const int tid = threadIdx.x;
    const int tx = tid & 15;   // expert group
    const int ty = tid >> 4;   // token group
    const int64_t tok0 = static_cast<int64_t>(blockIdx.x) * kRT;
    const int e0 = blockIdx.y * kRE;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kRK) {
        // x chunk: 64 tokens x 32 d, stored transposed (d-major).
        for (int i = tid; i < kRT * kRK; i += 256) {
            const int t = i / kRK, k = i % kRK;
            const int64_t tok = tok0 + t;
            float v = 0.f;
            if (tok < T) {
                const int64_t off = tok * d + k0 + k;
                if constexpr (sizeof(XT) == 2)
                    v = bf16_bits_to_float(x[off]);
                else
                    v = static_cast<float>(x[off]);
            }
            xs[k][t] = v;
        }
        for (int i = tid; i < kRK * kRE; i += 256) {
            const int k = i / kRE, e = i % kRE;
            ws[k][e] = (e0 + e < n) ? __ldg(Wg + static_cast<int64_t>(k0 + k) * n + e0 + e) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kRK; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[k][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = ws[k][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t tok = tok0 + ty * 4 + i;
        if (tok >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
            if (e < n) logits[tok * n + e] = acc[i][j];
        }
    }
    griddep_launch_dependents();
}

// One warp per token: lane l holds logits l, l+32, ... (NS per lane), each
// the in-order sum of `splits` partial logits [splits][T][n].
template <int NS>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits,
                                                          int splits, int64_t T, int n, int K,
                                                          int32_t* __restrict__ topk_idx,
                                                          float* __restrict__ topk_w) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const float* row = logits + t * n;
    const int64_t split_stride = T * n;
    float v[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        // all partials in flight at once, then summed in split order
        float part[kRouterMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kRouterMaxSplits; ++sp)
            part[sp] = (e < n && sp < splits) ? __ldg(row + sp * split_stride + e) : 0.f;
        float a = 0.f;
#pragma unroll
        for (int sp = 0; sp < kRouterMaxSplits; ++sp)
            if (sp < splits) a += part[sp];
        v[i] = (a != a) ? -INFINITY : a;  // NaN ranks lowest: keeps the order total
    }
    warp_topk_softmax<NS>(v, n, K, lane, topk_idx + t * K, topk_w + t * K);
    griddep_launch_dependents();
}

cudaError_t launch_router_topk(const float* logits, int splits, int64_t T, int n, int K,
                               int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    const dim3 grid(static_cast<unsigned>((T + 7) / 8));
    if (n <= 32)
        launch_k(router_topk_kernel<1>, grid, dim3(256), 0, st, logits, splits, T, n, K, topk_idx, topk_w);
    else if (n <= 64)
        launch_k(router_topk_kernel<2>, grid, dim3(256), 0, st, logits, splits, T, n, K, topk_idx, topk_w);
    else if (n <= 128)
        launch_k(router_topk_kernel<4>, grid, dim3(256), 0, st, logits, splits, T, n, K, topk_idx, topk_w);
    else
        launch_k(router_topk_kernel<8>, grid, dim3(256), 0, st, logits, splits, T, n, K, topk_idx, topk_w);
    return cudaGetLastError();
}

template <typename XT, int NE>
static void launch_small(const XT* x, const float* Wg, int64_t T, int d, int n, int K, int32_t* idx,
                         float* w, int num_sms, cudaStream_t st) {
    if (T < kTokenKernelMaxT) {
        // few tokens: a whole block per token keeps every SM's loads in flight
        launch_k(router_token_kernel<XT, NE>, dim3(static_cast<unsigned>(T)), dim3(TokenRouterCfg<NE>::kThreads), 0,
                 st, x, Wg, T, d, n, K, idx, w);
        return;
    }
    // many tokens: share each staged W_g chunk between TPW tokens per warp,
    // choosing TPW so that about two blocks land on every SM
    constexpr int kTpwMax = NE <= 8 ? 4 : (NE <= 16 ? 2 : 1);
    int tpw = 1;
    if (kTpwMax >= 4 && T >= static_cast<int64_t>(num_sms) * 8 * 4)
        tpw = 4;
    else if (kTpwMax >= 2 && T >= static_cast<int64_t>(num_sms) * 8 * 2)
        tpw = 2;
    const int64_t blocks = (T + 8 * tpw - 1) / (8 * tpw);
    const unsigned g = static_cast<unsigned>(blocks);
    if (tpw == 4)
        launch_k(router_small_kernel<XT, NE, (kTpwMax >= 4 ? 4 : 1)>, dim3(g), dim3(256), 0, st, x, Wg, T, d, n, K, idx, w);
    else if (tpw == 2)
        launch_k(router_small_kernel<XT, NE, (kTpwMax >= 2 ? 2 : 1)>, dim3(g), dim3(256), 0, st, x, Wg, T, d, n, K, idx, w);
    else
        launch_k(router_small_kernel<XT, NE, 1>, dim3(g), dim3(256), 0, st, x, Wg, T, d, n, K, idx, w);
}

template <typename XT>
static cudaError_t launch_router_t(const XT* x, const float* Wg, int64_t T, int d, int n, int K,
                                   int32_t* idx, float* w, float* logits_ws, int num_sms,
                                   cudaStream_t st) {
    if (n <= 8) {
        launch_small<XT, 8>(x, Wg, T, d, n, K, idx, w, num_sms, st);
        return cudaGetLastError();
    }
    if (n <= 16) {
        launch_small<XT, 16>(x, Wg, T, d, n, K, idx, w, num_sms, st);
        return cudaGetLastError();
    }
    if (n <= 32) {
        launch_small<XT, 32>(x, Wg, T, d, n, K, idx, w, num_sms, st);
        return cudaGetLastError();
    }
    dim3 g1(static_cast<unsigned>((T + kRT - 1) / kRT), static_cast<unsigned>((n + kRE - 1) / kRE));
    launch_k(router_logits_kernel<XT>, dim3(g1), dim3(256), 0, st, x, Wg, T, d, n, logits_ws);
    return launch_router_topk(logits_ws, 1, T, n, K, idx, w, st);
}

cudaError_t launch_router_logits_simt(const void* x, bool x_bf16, const float* Wg, int64_t T, int d,
                                      int n, float* logits, cudaStream_t st) {
    dim3 g1(static_cast<unsigned>((T + kRT - 1) / kRT), static_cast<unsigned>((n + kRE - 1) / kRE));
    if (x_bf16)
        launch_k(router_logits_kernel<uint16_t>, dim3(g1), dim3(256), 0, st, static_cast<const uint16_t*>(x), Wg, T, d, n,
                                                           logits);
    else
        launch_k(router_logits_kernel<float>, dim3(g1), dim3(256), 0, st, static_cast<const float*>(x), Wg, T, d, n, logits);
    return cudaGetLastError();
}

// Gates cast to bf16 (round to nearest even) and kept as fp32 values: the
// routing code quoted in Part 3 of "Mixture of Experts: Why Mixtral Only Wakes
// Up Two Specialists" computes the softmax in fp32 and casts the weights to
// the inputs' dtype.
__global__ void __launch_bounds__(256) gates_to_bf16_kernel(float* __restrict__ w, int64_t count) {
    griddep_wait();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride)
        w[i] = __bfloat162float(__float2bfloat16_rn(w[i]));
    griddep_launch_dependents();
}

cudaError_t launch_gates_to_bf16(float* topk_w, int64_t count, int num_sms, cudaStream_t st) {
    int64_t blocks = (count + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 4) blocks = static_cast<int64_t>(num_sms) * 4;
    if (blocks < 1) blocks = 1;
    launch_k(gates_to_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, topk_w, count);
    return cudaGetLastError();
}

cudaError_t launch_router(const void* x, bool x_bf16, const float* Wg, int64_t T, int d, int n,
                          int K, int32_t* topk_idx, float* topk_w, float* logits_ws, int num_sms,
                          cudaStream_t st) {
    if (x_bf16)
        return launch_router_t<uint16_t>(static_cast<const uint16_t*>(x), Wg, T, d, n, K, topk_idx,
                                         topk_w, logits_ws, num_sms, st);
    return launch_router_t<float>(static_cast<const float*>(x), Wg, T, d, n, K, topk_idx, topk_w,
                                  logits_ws, num_sms, st);
}

}  // namespace moe
