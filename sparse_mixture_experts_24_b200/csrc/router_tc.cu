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
// streams x (128 x 64) and the three W_g parts (Npad x 64 each, adjacent in
// shared memory) by TMA through a multi-stage ring; warp 1 issues the
// tcgen05.mma (M=128, K=16) of every K step; warps 2-5 read the fp32
// accumulators from TMEM.  With Npad <= 128 each part has an accumulator of
// its own, so that the three parts are one B operand of N = 3 Npad (one MMA
// per K step for Npad <= 80; N = 2 Npad and N = Npad up to 128), and the
// epilogue adds (hi + mid) + lo; wider W_g keeps one accumulator that the
// three MMAs of a K step all add into.  A tcgen05.mma costs its issuing thread
// about the same whatever its N, so fewer, wider MMAs finish the K steps
// sooner when Npad is small.
//   Logits variant: each CTA stages its partial logits in shared memory and
//   writes them as whole rows to [split][T][n]; router_topk_kernel (router.cu)
//   sums the splits in order and selects.
//   Fused variant: the splits of one token block form a cluster (1 x splits);
//   every CTA stages its partial in its own shared memory, and after a cluster
//   barrier the cluster's CTAs share out the 128 tokens: for each of its
//   tokens a warp sums the splits' partials in split order (read over
//   distributed shared memory, lane = expert) and selects the top K with the
//   same warp selection as router_topk_kernel (topk.cuh).  The logits never
//   reach global memory and no second kernel runs.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace moe {

// W_g [d][n] fp32 -> parts [3][npad][d] bf16 (rows n..npad-1 are zero).  One
// block per 32 rows of d and 32 experts: the tile is read along the experts
// (W_g's contiguous dimension) into shared memory, four loads per thread in
// flight together, and written along d, two values per 32-bit store (d is a
// multiple of 64).
__global__ void __launch_bounds__(256) wg_split_kernel(const float* __restrict__ Wg, int d, int n,
                                                       int npad, uint16_t* __restrict__ parts) {
    griddep_wait();
    __shared__ float tile[32][33];
    const int j0 = static_cast<int>(blockIdx.x) * 32, e0 = static_cast<int>(blockIdx.y) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        v[u] = (e0 + tx < n) ? __ldg(Wg + static_cast<int64_t>(j0 + ty + 8 * u) * n + e0 + tx) : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) tile[ty + 8 * u][tx] = v[u];
    __syncthreads();
    const int64_t total = static_cast<int64_t>(npad) * d;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int q = static_cast<int>(threadIdx.x) + 256 * u;
        const int c = q >> 4, pr = q & 15;  // expert e0 + c, rows j0 + 2 pr, j0 + 2 pr + 1
        if (e0 + c >= npad) continue;
        const int64_t at = static_cast<int64_t>(e0 + c) * d + j0 + 2 * pr;
        uint32_t packed[3] = {0u, 0u, 0u};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float w = tile[2 * pr + h][c];
            const __nv_bfloat16 hi = __float2bfloat16_rn(w);
            const float r1 = w - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const float r2 = r1 - __bfloat162float(mid);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
            packed[0] |= static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << (16 * h);
            packed[1] |= static_cast<uint32_t>(__bfloat16_as_ushort(mid)) << (16 * h);
            packed[2] |= static_cast<uint32_t>(__bfloat16_as_ushort(lo)) << (16 * h);
        }
#pragma unroll
        for (int p = 0; p < 3; ++p) *reinterpret_cast<uint32_t*>(parts + p * total + at) = packed[p];
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

// Partial logits staged per CTA: 128 rows of npad rounded up to 32 plus one
// float (the odd pitch keeps a warp's 32 rows in 32 different banks).
__host__ __device__ inline int rt_stage_pitch(int npad) { return (npad + 31) / 32 * 32 + 1; }
__host__ __device__ inline int rt_ring_bytes(int npad) {
    const int ring = rt_stages(npad) * rt_stage_bytes(npad);
    const int staged = kRtBM * rt_stage_pitch(npad) * 4;
    return ring > staged ? ring : staged;
}

// volatile keeps these loads after the cluster barrier that publishes the
// partials; with no memory clobber, arithmetic may move around them, so that
// several loads are issued before their first use.
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// Accumulator columns: one group of Npad per part (Npad <= 128), else one.
__host__ __device__ inline int rt_groups(int npad) { return npad <= 128 ? 3 : 1; }

__host__ inline int rt_tmem_cols(int npad) {
    int c = 32;
    while (c < rt_groups(npad) * npad) c <<= 1;
    return c;
}

// kNS: 32-expert slots per lane in the fused selection (npad <= 32 * kNS).
template <bool kFused, int kNS>
__global__ void __launch_bounds__(kRtThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     int64_t T, int d, int n, int npad, int tmem_cols, float* __restrict__ logits,
                     int K, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int stage_bytes = rt_stage_bytes(npad);
    const int stages = rt_stages(npad);
    RtTail* tail = reinterpret_cast<RtTail*>(smem + rt_ring_bytes(npad));
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
            // the three parts: one MMA of N = 3 Npad (Npad <= 80), N = 2 Npad
            // plus N = Npad (Npad <= 128), or three of N = Npad into one
            // accumulator
            const int groups = rt_groups(npad);
            const int n_first = groups == 1 ? npad : (npad <= 80 ? 3 * npad : 2 * npad);
            const uint32_t idesc_first = make_idesc_bf16(kRtBM, n_first, 0, 0);
            const uint32_t idesc_part = make_idesc_bf16(kRtBM, npad, 0, 0);
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
                    const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                    tc_mma_f16(tmem_base, adesc, make_smem_desc(b_base + kk * 32, 16, 1024, 2), idesc_first, acc);
                    if (groups == 1) {
                        for (int p = 1; p < 3; ++p)
                            tc_mma_f16(tmem_base, adesc, make_smem_desc(b_base + p * part_bytes + kk * 32, 16, 1024, 2),
                                       idesc_part, 1u);
                    } else if (n_first == 2 * npad) {
                        tc_mma_f16(tmem_base + static_cast<uint32_t>(2 * npad), adesc,
                                   make_smem_desc(b_base + 2 * part_bytes + kk * 32, 16, 1024, 2), idesc_part, acc);
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
    }
    // ---- epilogue: warps 2-5, thread = accumulator row (TMEM lane) ----
    // After accum_full every MMA of this CTA has completed, so the ring's
    // shared memory is free for staging.
    const int pitch = rt_stage_pitch(npad);
    float* stage_rows = reinterpret_cast<float*>(smem);
    const uint32_t rank = kFused ? blockIdx.y : 0;  // cluster (1 x splits): rank = split
    bool have_acc = false;
    if (warp >= 2) {
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        have_acc = mbar_wait(smem_u32(&tail->accum_full), 0, status, kStatusTimeoutAccum);
        if (have_acc) {
            tc_fence_after();
            const int groups = rt_groups(npad);
            const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
            for (int c = 0; c < npad; c += 16) {
                float a[16];
                uint32_t v[16];
                tmem_ld_32x32b_x16(lane_base + c, v);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) a[q] = __uint_as_float(v[q]);
                for (int g = 1; g < groups; ++g) {  // (hi + mid) + lo
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(g * npad + c), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 16; ++q) a[q] += __uint_as_float(v[q]);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) stage_rows[r * pitch + c + q] = a[q];
            }
            tc_fence_before();
        }
        if (!kFused && have_acc) {
            // whole rows: lane l writes columns l, l+32, ... of each of the warp's 32 rows
            __syncwarp();
            for (int rr = 0; rr < 32; ++rr) {
                const int64_t t = static_cast<int64_t>(m0) + quad * 32 + rr;
                if (t >= T) break;
                const float* src = stage_rows + (quad * 32 + rr) * pitch;
                float* out = logits + t * n;
                for (int c = lane; c < n; c += 32) out[c] = src[c];
            }
        }
    }
    if (kFused) {
        cluster_sync();  // every split's partial is staged
        const int splits = static_cast<int>(gridDim.y);
        const int rows_per = (kRtBM + splits - 1) / splits;
        const int r_end = min(kRtBM, static_cast<int>(rank) * rows_per + rows_per);
        uint32_t part_base[kRouterMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kRouterMaxSplits; ++sp)
            part_base[sp] = mapa_shared(smem_u32(stage_rows), static_cast<uint32_t>(sp < splits ? sp : 0));
        // a warp takes kRows consecutive rows at a time: all their partials
        // are loaded before any selection, so that the remote loads of the
        // kRows rows are in flight together
        constexpr int kRows = kNS <= 4 ? 4 : 2;
        constexpr int kWarps = kRtThreads / 32;
        for (int r0 = static_cast<int>(rank) * rows_per + warp * kRows; r0 < r_end; r0 += kWarps * kRows) {
            float v[kRows][kNS];
#pragma unroll
            for (int j = 0; j < kRows; ++j) {
                const int r = r0 + j;
                const bool row_ok = r < r_end && static_cast<int64_t>(m0) + r < T;
#pragma unroll
                for (int i = 0; i < kNS; ++i) {
                    const int e = lane + 32 * i;
                    float part[kRouterMaxSplits];
#pragma unroll
                    for (int sp = 0; sp < kRouterMaxSplits; ++sp)
                        part[sp] = (row_ok && e < n && sp < splits)
                                       ? ld_shared_cluster_f32(part_base[sp] +
                                                               static_cast<uint32_t>(r * pitch + e) * 4u)
                                       : 0.f;
                    float a = 0.f;
#pragma unroll
                    for (int sp = 0; sp < kRouterMaxSplits; ++sp)
                        if (sp < splits) a += part[sp];
                    v[j][i] = (a != a) ? -INFINITY : a;  // NaN ranks lowest
                }
            }
#pragma unroll
            for (int j = 0; j < kRows; ++j) {
                const int r = r0 + j;
                const int64_t t = static_cast<int64_t>(m0) + r;
                if (r < r_end && t < T) warp_topk_softmax<kNS>(v[j], n, K, lane, topk_idx + t * K, topk_w + t * K);
            }
        }
        cluster_sync();  // no CTA leaves while another reads its staged partial
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
    return rt_ring_bytes(npad) + static_cast<int>(sizeof(RtTail)) + 1024;
}

// split d so that the CTAs fill at most one wave (one CTA per SM: the ring
// takes most of shared memory), at least 8 K blocks each
static int router_splits(int64_t T, int d, int num_sms) {
    const int64_t mtiles = (T + kRtBM - 1) / kRtBM;
    int splits = static_cast<int>(num_sms / mtiles);
    const int kb_total = d / kRtBK;
    if (splits > kRouterMaxSplits) splits = kRouterMaxSplits;
    if (splits > kb_total / 8) splits = kb_total / 8;
    if (splits < 1) splits = 1;
    return splits;
}

static void launch_wg_split(const float* Wg, uint16_t* parts, int d, int n, int num_sms, cudaStream_t st) {
    (void)num_sms;
    const int npad = (n + 15) / 16 * 16;
    const dim3 grid(static_cast<unsigned>(d / 32), static_cast<unsigned>((npad + 31) / 32));
    launch_k(wg_split_kernel, grid, dim3(256), 0, st, Wg, d, n, npad, parts);
}

cudaError_t launch_router_logits_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                                    uint16_t* parts, int64_t T, int d, int n, float* logits, int* status,
                                    int num_sms, cudaStream_t st, int* splits_out) {
    const int npad = (n + 15) / 16 * 16;
    launch_wg_split(Wg, parts, d, n, num_sms, st);
    const int smem = router_tc_smem_bytes(n);
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<false, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int splits = router_splits(T, d, num_sms);
    const int64_t mtiles = (T + kRtBM - 1) / kRtBM;
    dim3 grid(static_cast<unsigned>(mtiles), static_cast<unsigned>(splits));
    launch_k(router_tc_kernel<false, 1>, dim3(grid), dim3(kRtThreads), smem, st, tm_x, tm_w, T, d, n, npad,
             rt_tmem_cols(npad), logits, 0, static_cast<int32_t*>(nullptr), static_cast<float*>(nullptr), status);
    *splits_out = splits;
    return cudaGetLastError();
}

// The top-K runs in the router's epilogue unless MOE_ROUTER_TOPK=separate asks
// for the logits-then-top-K kernels.
static bool fuse_topk(int K) {
    (void)K;
    static const bool separate = [] {
        const char* e = getenv("MOE_ROUTER_TOPK");
        return e && strcmp(e, "separate") == 0;
    }();
    return !separate;
}

int router_tc_launches(int K) { return fuse_topk(K) ? 2 : 3; }

// The fused router as clusters of the d-splits of each 128-token block.
template <int kNS>
static cudaError_t launch_fused(const CUtensorMap& tm_x, const CUtensorMap& tm_w, int64_t T, int d, int n, int npad,
                                float* logits, int K, int32_t* topk_idx, float* topk_w, int* status, int num_sms,
                                cudaStream_t st) {
    const int smem = router_tc_smem_bytes(n);
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<true, kNS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem);
    if (e != cudaSuccess) return e;
    const int splits = router_splits(T, d, num_sms);
    const int64_t mtiles = (T + kRtBM - 1) / kRtBM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(mtiles), static_cast<unsigned>(splits));
    cfg.blockDim = dim3(kRtThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(splits);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (g_chain_started && pdl_enabled()) ? 2 : 1;
    g_chain_started = true;
    e = cudaLaunchKernelEx(&cfg, router_tc_kernel<true, kNS>, tm_x, tm_w, T, d, n, npad, rt_tmem_cols(npad), logits,
                           K, topk_idx, topk_w, status);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_router_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                             uint16_t* parts, int64_t T, int d, int n, int K, float* logits,
                             int32_t* topk_idx, float* topk_w, int* status, int num_sms,
                             cudaStream_t st) {
    if (!fuse_topk(K)) {
        int splits = 1;
        cudaError_t e = launch_router_logits_tc(tm_x, tm_w, Wg, parts, T, d, n, logits, status, num_sms, st,
                                                &splits);
        if (e != cudaSuccess) return e;
        return launch_router_topk(logits, splits, T, n, K, topk_idx, topk_w, st);
    }
    const int npad = (n + 15) / 16 * 16;
    launch_wg_split(Wg, parts, d, n, num_sms, st);
    if (npad <= 32)
        return launch_fused<1>(tm_x, tm_w, T, d, n, npad, logits, K, topk_idx, topk_w, status, num_sms, st);
    if (npad <= 64)
        return launch_fused<2>(tm_x, tm_w, T, d, n, npad, logits, K, topk_idx, topk_w, status, num_sms, st);
    if (npad <= 128)
        return launch_fused<4>(tm_x, tm_w, T, d, n, npad, logits, K, topk_idx, topk_w, status, num_sms, st);
    return launch_fused<8>(tm_x, tm_w, T, d, n, npad, logits, K, topk_idx, topk_w, status, num_sms, st);
}

}  // namespace moe
