// router_tc.cu -- the router logits x . W_g on the tensor cores, at fp32
// accuracy, for bf16 activations.
//
// Source: "Mixture of Experts: Why Mixtral Only Wakes Up Two Specialists",
// Part 3, Step 1: the router is one bias-free linear layer giving one score
// (logit) per expert; the top-K and softmax that follow run in
// router_topk_kernel (router.cu).
//
// x is bf16, so every x value is exact in bf16.  W_g is fp32: wg_split_kernel
// writes it as three bf16 parts, W_g = hi + mid + lo + e with |e| <= 2^-24 |W_g|
// (each part is the bf16 rounding of what the previous parts left), laid out
// expert-major ([3][Npad][d], K contiguous).  Each part's product with x is
// exact in fp32, and the three MMAs accumulate into one fp32 TMEM accumulator,
// so the logits carry fp32-class rounding, not bf16's.
//
// router_tc_kernel: one CTA per (128 tokens, slice of d): the d range is split
// over gridDim.y CTAs so that small token counts still fill the GPU; warp 0
// streams x (128 x 64) and the three W_g parts (Npad x 64 each) by TMA through
// a multi-stage ring; warp 1 issues tcgen05.mma M=128, N=Npad, K=16 three
// times per K step; warps 2-5 read the 128 x Npad fp32 accumulator from TMEM
// and store the slice's partial logits [split][T][n], which the top-K kernel
// sums in split order (deterministic).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// W_g [d][n] fp32 -> parts [3][npad][d] bf16 (rows n..npad-1 are zero).
__global__ void __launch_bounds__(256) wg_split_kernel(const float* __restrict__ Wg, int d, int n,
                                                       int npad, uint16_t* __restrict__ parts) {
    griddep_wait();
    const int64_t total = static_cast<int64_t>(npad) * d;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int e = static_cast<int>(i / d);
        const int j = static_cast<int>(i - static_cast<int64_t>(e) * d);
        const float w = (e < n) ? __ldg(Wg + static_cast<int64_t>(j) * n + e) : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
        parts[i] = __bfloat16_as_ushort(hi);
        parts[total + i] = __bfloat16_as_ushort(mid);
        parts[2 * total + i] = __bfloat16_as_ushort(lo);
    }
    griddep_launch_dependents();
}

constexpr int kRtThreads = 192;
constexpr int kRtBM = 128;
constexpr int kRtBK = 64;
constexpr int kRtMaxStages = 6;
constexpr int kRtStageBudget = 196608;  // shared memory for the ring

struct __align__(8) RtTail {
    uint64_t full[kRtMaxStages];
    uint64_t empty[kRtMaxStages];
    uint64_t accum_full;
    uint64_t done;
    uint32_t tmem_base;
};

__host__ __device__ inline int rt_stage_bytes(int npad) { return kRtBM * kRtBK * 2 + 3 * npad * kRtBK * 2; }

__host__ __device__ inline int rt_stages(int npad) {
    int s = kRtStageBudget / rt_stage_bytes(npad);
    return s > kRtMaxStages ? kRtMaxStages : s;
}

__host__ inline int rt_tmem_cols(int npad) {
    int c = 32;
    while (c < npad) c <<= 1;
    return c;
}

__global__ void __launch_bounds__(kRtThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     int64_t T, int d, int n, int npad, int tmem_cols, float* __restrict__ logits,
                     int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int stage_bytes = rt_stage_bytes(npad);
    const int stages = rt_stages(npad);
    RtTail* tail = reinterpret_cast<RtTail*>(smem + stages * stage_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb_total = d / kRtBK;
    const int kb_begin = static_cast<int>(static_cast<int64_t>(kb_total) * blockIdx.y / gridDim.y);
    const int kb_end = static_cast<int>(static_cast<int64_t>(kb_total) * (blockIdx.y + 1) / gridDim.y);
    const int k_blocks = kb_end - kb_begin;
    const int m0 = blockIdx.x * kRtBM;
    logits += static_cast<int64_t>(blockIdx.y) * T * n;
    const int part_bytes = npad * kRtBK * 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
        }
        mbar_init(smem_u32(&tail->accum_full), 1);
        mbar_init(smem_u32(&tail->done), 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tail->tmem_base), static_cast<uint32_t>(tmem_cols));
        tmem_relinquish();
    }
    griddep_wait();  // the W_g parts come from the previous kernel
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            int armed[kRtMaxStages];
            for (int s = 0; s < kRtMaxStages; ++s) armed[s] = -1;
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty))
                    break;
                const uint32_t fb = smem_u32(&tail->full[stage]);
                mbar_arrive_expect_tx(fb, static_cast<uint32_t>(stage_bytes));
                armed[stage] = static_cast<int>(phase);
                const uint32_t dst = smem_u32(smem + stage * stage_bytes);
                const int kx = (kb_begin + kb) * kRtBK;
                tma_load_2d(dst, &tm_x, fb, kx, m0);
#pragma unroll
                for (int p = 0; p < 3; ++p)
                    tma_load_2d(dst + kRtBM * kRtBK * 2 + p * part_bytes, &tm_w, fb, kx, p * npad);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            for (int s = 0; s < stages; ++s)
                if (armed[s] >= 0)
                    mbar_wait(smem_u32(&tail->full[s]), static_cast<uint32_t>(armed[s]), status,
                              kStatusTimeoutDrain);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc_bf16(kRtBM, npad, 0, 0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_base = smem_u32(smem + stage * stage_bytes);
                const uint32_t b_base = a_base + kRtBM * kRtBK * 2;
#pragma unroll
                for (int kk = 0; kk < kRtBK / 16; ++kk) {
                    const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const uint64_t bdesc =
                            make_smem_desc(b_base + p * part_bytes + kk * 32, 16, 1024, 2);
                        tc_mma_f16(tmem_base, adesc, bdesc, idesc, (kb | kk | p) != 0 ? 1u : 0u);
                    }
                }
                tc_commit(smem_u32(&tail->empty[stage]));
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) tc_commit(smem_u32(&tail->accum_full));
            // every MMA of this CTA must be finished before TMEM is freed
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const int64_t t = static_cast<int64_t>(m0) + r;
        if (mbar_wait(smem_u32(&tail->accum_full), 0, status, kStatusTimeoutAccum)) {
            tc_fence_after();
            for (int c = 0; c < npad; c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c, v);
                tmem_wait_ld();
                if (t < T) {
                    float* out = logits + t * n;
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        if (c + q < n) out[c + q] = __uint_as_float(v[q]);
                }
            }
            tc_fence_before();
        }
    }
    __syncthreads();
    griddep_launch_dependents();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(tmem_cols));
    }
}

int router_tc_smem_bytes(int n) {
    const int npad = (n + 15) / 16 * 16;
    return rt_stages(npad) * rt_stage_bytes(npad) + static_cast<int>(sizeof(RtTail)) + 1024;
}

cudaError_t launch_router_logits_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                                    uint16_t* parts, int64_t T, int d, int n, float* logits, int* status,
                                    int num_sms, cudaStream_t st, int* splits_out) {
    const int npad = (n + 15) / 16 * 16;
    const int64_t total = static_cast<int64_t>(npad) * d;
    int64_t sb = (total + 255) / 256;
    if (sb > static_cast<int64_t>(num_sms) * 8) sb = static_cast<int64_t>(num_sms) * 8;
    launch_k(wg_split_kernel, dim3(static_cast<unsigned>(sb)), dim3(256), 0, st, Wg, d, n, npad, parts);
    const int smem = router_tc_smem_bytes(n);
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    // split d so that the CTAs fill at most one wave (one CTA per SM: the ring
    // takes most of shared memory), at least 8 K blocks each
    const int64_t mtiles = (T + kRtBM - 1) / kRtBM;
    int splits = static_cast<int>(num_sms / mtiles);
    const int kb_total = d / kRtBK;
    if (splits > kRouterMaxSplits) splits = kRouterMaxSplits;
    if (splits > kb_total / 8) splits = kb_total / 8;
    if (splits < 1) splits = 1;
    dim3 grid(static_cast<unsigned>(mtiles), static_cast<unsigned>(splits));
    launch_k(router_tc_kernel, dim3(grid), dim3(kRtThreads), smem, st, tm_x, tm_w, T, d, n, npad, rt_tmem_cols(npad),
                                                     logits, status);
    *splits_out = splits;
    return cudaGetLastError();
}

cudaError_t launch_router_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                             uint16_t* parts, int64_t T, int d, int n, int K, float* logits,
                             int32_t* topk_idx, float* topk_w, int* status, int num_sms,
                             cudaStream_t st) {
    int splits = 1;
    cudaError_t e = launch_router_logits_tc(tm_x, tm_w, Wg, parts, T, d, n, logits, status, num_sms, st,
                                            &splits);
    if (e != cudaSuccess) return e;
    return launch_router_topk(logits, splits, T, n, K, topk_idx, topk_w, st);
}

}  // namespace moe
