// expert_choice.cu -- expert-choice routing: every expert picks its own C
// tokens ("Mixtral of Experts? Mixture of Experts? Try to explain Mixtral
// 8x7B", section "How Experts Are Chosen", item 2: experts choose which tokens
// to process, each with a fixed capacity).
//
//   S[t][e]  = softmax over the n experts of the router logits of token t;
//   expert e keeps the C tokens with the largest S[.][e] (equal scores: lower
//   token first), laid out as rows e*C .. e*C+C-1 in ascending token order;
//   y[t]     = sum over the experts that kept t, in expert order, of
//              S[t][e] * SwiGLU_e(x_t)  (0 for a token no expert kept).
//
// Kernels: ec_softmax_kernel (probabilities, transposed to [n][T], and the
// row map reset), ec_select_kernel (one block per expert: exact radix select
// of the C largest unique 64-bit keys (score bits, inverted token), then an
// ordered compaction), ec_combine_kernel (one thread per 16-byte vector of y).
// The expert GEMMs and the row gather are the token-choice ones.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// logits [splits][T][n] -> St [n][T]; rowmap [T][n] = -1.
__global__ void __launch_bounds__(256) ec_softmax_kernel(const float* __restrict__ logits, int splits,
                                                         int64_t T, int n, float* __restrict__ St,
                                                         int32_t* __restrict__ rowmap) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    float v[8];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        float part[kRouterMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kRouterMaxSplits; ++sp)
            part[sp] = (e < n && sp < splits) ? logits[(static_cast<int64_t>(sp) * T + t) * n + e] : 0.f;
        float a = 0.f;
#pragma unroll
        for (int sp = 0; sp < kRouterMaxSplits; ++sp)
            if (sp < splits) a += part[sp];
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
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < n) {
            St[static_cast<int64_t>(e) * T + t] = v[i] * inv;
            rowmap[t * n + e] = -1;
        }
    }
    griddep_launch_dependents();
}

// Larger key = better: probability first (non-negative floats order like
// their bit patterns), then the lower token index.
__device__ __forceinline__ uint64_t ec_key(float s, int64_t t) {
    return (static_cast<uint64_t>(__float_as_uint(s)) << 32) |
           static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(t));
}

constexpr int kSelThreads = 1024;

// One block per expert.
__global__ void __launch_bounds__(kSelThreads) ec_select_kernel(const float* __restrict__ St, int64_t T,
                                                                int n, int C, int bm,
                                                                int32_t* __restrict__ sel_token,
                                                                float* __restrict__ sel_gate,
                                                                int32_t* __restrict__ row_token,
                                                                int32_t* __restrict__ rowmap,
                                                                int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ offsets,
                                                                int32_t* __restrict__ mblk_base) {
    griddep_wait();
    __shared__ int32_t hist[256];
    __shared__ uint64_t s_prefix;
    __shared__ int s_remaining;
    __shared__ int32_t s_warp_sum[kSelThreads / 32];
    __shared__ int32_t s_base;
    const int e = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const float* col = St + static_cast<int64_t>(e) * T;

    if (tid == 0) {
        const int mb = (C + bm - 1) / bm;
        counts[e] = C;
        offsets[e] = e * C;
        mblk_base[e] = e * mb;
        if (e == n - 1) {
            offsets[n] = n * C;
            mblk_base[n] = n * mb;
        }
        s_prefix = 0;
        s_remaining = C;
    }
    // exact radix select of the C-th largest key, 8 bits per pass from the top
    uint64_t mask = 0;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        const uint64_t prefix = s_prefix;
        for (int64_t t = tid; t < T; t += kSelThreads) {
            const uint64_t k = ec_key(col[t], t);
            if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 0xFF], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int need = s_remaining, cum = 0, digit = 0;
            for (int b = 255; b >= 0; --b) {
                if (cum + hist[b] >= need) {
                    digit = b;
                    break;
                }
                cum += hist[b];
            }
            s_remaining = need - cum;
            s_prefix = prefix | (static_cast<uint64_t>(digit) << shift);
        }
        mask |= static_cast<uint64_t>(0xFF) << shift;
        __syncthreads();
    }
    const uint64_t kth = s_prefix;  // the C-th largest key: exactly C keys are >= kth
    // ordered compaction: tokens with key >= kth, ascending
    if (tid == 0) s_base = 0;
    __syncthreads();
    for (int64_t t0 = 0; t0 < T; t0 += kSelThreads) {
        const int64_t t = t0 + tid;
        float s = 0.f;
        bool keep = false;
        if (t < T) {
            s = col[t];
            keep = ec_key(s, t) >= kth;
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) s_warp_sum[warp] = __popc(bal);
        __syncthreads();
        if (warp == 0) {
            const int v = s_warp_sum[lane];
            int inc = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += u;
            }
            s_warp_sum[lane] = inc - v;  // exclusive warp base
        }
        __syncthreads();
        if (keep) {
            const int pos = s_base + s_warp_sum[warp] + __popc(bal & ((1u << lane) - 1u));
            if (pos < C) {
                const int row = e * C + pos;
                sel_token[row] = static_cast<int32_t>(t);
                sel_gate[row] = s;
                row_token[row] = static_cast<int32_t>(t);
                rowmap[t * n + e] = row;
            }
        }
        __syncthreads();
        // the last thread holds the last warp's ballot: chunk total = its base + its count
        if (tid == kSelThreads - 1) s_base += s_warp_sum[kSelThreads / 32 - 1] + __popc(bal);
        __syncthreads();
    }
    griddep_launch_dependents();
}

// y[t] = sum_e [rowmap[t][e] >= 0] gate * O[row], expert order.
template <bool kBf16>
__global__ void __launch_bounds__(256) ec_combine_kernel(const void* __restrict__ Ov,
                                                         const int32_t* __restrict__ rowmap,
                                                         const float* __restrict__ gate_of_row,
                                                         int64_t T, int n, int vec_per_row,
                                                         void* __restrict__ yv) {
    griddep_wait();
    const int64_t total = T * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / vec_per_row;
        const int64_t v = i - t * vec_per_row;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int e = 0; e < n; ++e) {
            const int32_t r = __ldg(rowmap + t * n + e);
            if (r < 0) continue;
            const float g = __ldg(gate_of_row + r);
            if (kBf16) {
                const uint4 q = __ldg(static_cast<const uint4*>(Ov) + static_cast<int64_t>(r) * vec_per_row + v);
                float a, b;
                unpack_bf16x2(q.x, a, b);
                acc[0] = fmaf(g, a, acc[0]);
                acc[1] = fmaf(g, b, acc[1]);
                unpack_bf16x2(q.y, a, b);
                acc[2] = fmaf(g, a, acc[2]);
                acc[3] = fmaf(g, b, acc[3]);
                unpack_bf16x2(q.z, a, b);
                acc[4] = fmaf(g, a, acc[4]);
                acc[5] = fmaf(g, b, acc[5]);
                unpack_bf16x2(q.w, a, b);
                acc[6] = fmaf(g, a, acc[6]);
                acc[7] = fmaf(g, b, acc[7]);
            } else {
                const float4 q = __ldg(static_cast<const float4*>(Ov) + static_cast<int64_t>(r) * vec_per_row + v);
                acc[0] = fmaf(g, q.x, acc[0]);
                acc[1] = fmaf(g, q.y, acc[1]);
                acc[2] = fmaf(g, q.z, acc[2]);
                acc[3] = fmaf(g, q.w, acc[3]);
            }
        }
        if (kBf16) {
            uint4 out;
            out.x = pack_bf16x2(acc[0], acc[1]);
            out.y = pack_bf16x2(acc[2], acc[3]);
            out.z = pack_bf16x2(acc[4], acc[5]);
            out.w = pack_bf16x2(acc[6], acc[7]);
            static_cast<uint4*>(yv)[i] = out;
        } else {
            static_cast<float4*>(yv)[i] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
    }
    griddep_launch_dependents();
}

cudaError_t launch_ec_route(const float* logits, int splits, int64_t T, int n, int C, int bm, float* St,
                            int32_t* rowmap, int32_t* sel_token, float* sel_gate, int32_t* row_token,
                            int32_t* counts, int32_t* offsets, int32_t* mblk_base, cudaStream_t st) {
    launch_k(ec_softmax_kernel, dim3(static_cast<unsigned>((T + 7) / 8)), dim3(256), 0, st, logits, splits,
             T, n, St, rowmap);
    launch_k(ec_select_kernel, dim3(static_cast<unsigned>(n)), dim3(kSelThreads), 0, st, St, T, n, C, bm,
             sel_token, sel_gate, row_token, rowmap, counts, offsets, mblk_base);
    return cudaGetLastError();
}

cudaError_t launch_ec_combine(const void* O, bool bf16, const int32_t* rowmap, const float* gate_of_row,
                              int64_t T, int n, int d, void* y, int num_sms, cudaStream_t st) {
    const int vpr = bf16 ? d / 8 : d / 4;
    int64_t blocks = (T * vpr + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (bf16)
        launch_k(ec_combine_kernel<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, O, rowmap,
                 gate_of_row, T, n, vpr, y);
    else
        launch_k(ec_combine_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, O, rowmap,
                 gate_of_row, T, n, vpr, y);
    return cudaGetLastError();
}

}  // namespace moe
