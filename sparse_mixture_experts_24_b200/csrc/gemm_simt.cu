// gemm_simt.cu -- fp32 grouped expert GEMMs on CUDA cores, the path of fp32
// handles (tensor cores have no fp32 x fp32 kind that keeps full fp32
// products).
//
//   GEMM1: H[r] = silu(Xp[r] . w1[e]) * (Xp[r] . w3[e])   rows r of expert e
//   GEMM2: O[r] = H[r] . w2[e]
//
// Source: the expert of the layer equation, SwiGLU_i(x) = (silu(x.w1_i) (*)
// x.w3_i) . w2_i ("Mixtral of Experts" section 2.1 on the flash-card page; the
// expand / non-linear / compress description of the feed-forward block in
// Part 2 of the neobadger page).
//
// Each block owns one 64-row M-block of one expert's segment and 64 output
// columns; 256 threads hold 4x4 outputs each (two accumulators in GEMM1).
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSM = kSimtBM;  // 64 rows
constexpr int kSN = 64;       // columns
constexpr int kSK = 16;       // reduction chunk

// Expert owning M-block `mb` (binary search over the M-block prefix).
__device__ __forceinline__ int find_expert(const int32_t* mblk_base, int n, int mb) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mblk_base[mid] <= mb)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A,
                                                        const float* __restrict__ B0,
                                                        const float* __restrict__ B1,
                                                        float* __restrict__ C,
                                                        const int32_t* __restrict__ offsets,
                                                        const int32_t* __restrict__ mblk_base,
                                                        int n, int Kdim, int Ncols) {
    griddep_wait();
    __shared__ float As[kSK][kSM + 4];
    __shared__ float Bs0[kSK][kSN + 4];
    __shared__ float Bs1[kSK][kSN + 4];
    const int mb = blockIdx.x;
    if (mb >= mblk_base[n]) return;
    const int e = find_expert(mblk_base, n, mb);
    const int row0 = offsets[e] + (mb - mblk_base[e]) * kSM;
    const int rows = min(kSM, offsets[e + 1] - row0);
    const int col0 = blockIdx.y * kSN;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const float* b0 = B0 + static_cast<int64_t>(e) * Kdim * Ncols;
    const float* b1 = kSwiGLU ? B1 + static_cast<int64_t>(e) * Kdim * Ncols : nullptr;

    float acc0[4][4], acc1[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;

    for (int k0 = 0; k0 < Kdim; k0 += kSK) {
        for (int i = tid; i < kSM * kSK; i += 256) {
            const int r = i / kSK, k = i % kSK;
            As[k][r] = (r < rows) ? A[static_cast<int64_t>(row0 + r) * Kdim + k0 + k] : 0.f;
        }
        for (int i = tid; i < kSK * kSN; i += 256) {
            const int k = i / kSN, c = i % kSN;
            const bool in = col0 + c < Ncols;
            const int64_t off = static_cast<int64_t>(k0 + k) * Ncols + col0 + c;
            Bs0[k][c] = in ? b0[off] : 0.f;
            if (kSwiGLU) Bs1[k][c] = in ? b1[off] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kSK; ++k) {
            float a[4], w0[4], w1v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w0[j] = Bs0[k][tx * 4 + j];
                if (kSwiGLU) w1v[j] = Bs1[k][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc0[i][j] = fmaf(a[i], w0[j], acc0[i][j]);
                    if (kSwiGLU) acc1[i][j] = fmaf(a[i], w1v[j], acc1[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = col0 + tx * 4 + j;
            if (c >= Ncols) continue;
            float v = acc0[i][j];
            if (kSwiGLU) v = v / (1.f + expf(-v)) * acc1[i][j];
            C[static_cast<int64_t>(row0 + r) * Ncols + c] = v;
        }
    }
    griddep_launch_dependents();
}

static unsigned mblk_cap(int64_t R, int n) {
    return static_cast<unsigned>((R + kSM - 1) / kSM + n);
}

cudaError_t launch_simt_gemm1(const float* xp, const float* w1, const float* w3, float* h,
                              const int32_t* offsets, const int32_t* mblk_base, int n, int64_t R,
                              int d, int F, cudaStream_t st) {
    dim3 grid(mblk_cap(R, n), static_cast<unsigned>((F + kSN - 1) / kSN));
    launch_k(simt_gemm_kernel<true>, dim3(grid), dim3(256), 0, st, xp, w1, w3, h, offsets, mblk_base, n, d, F);
    return cudaGetLastError();
}

cudaError_t launch_simt_gemm2(const float* h, const float* w2, float* o, const int32_t* offsets,
                              const int32_t* mblk_base, int n, int64_t R, int d, int F,
                              cudaStream_t st) {
    dim3 grid(mblk_cap(R, n), static_cast<unsigned>((d + kSN - 1) / kSN));
    launch_k(simt_gemm_kernel<false>, dim3(grid), dim3(256), 0, st, h, w2, nullptr, o, offsets, mblk_base, n, F, d);
    return cudaGetLastError();
}

}  // namespace moe
