// e4m3.cu -- FP8 (E4M3) quantisation for the low-precision expert path:
// expert weights held in fewer bits than 16 to cut the memory they take and
// the bytes a decode step reads ("Mixture of Experts: Why Mixtral Only Wakes
// Up Two Specialists", Part 4, "Why total and active both matter": the
// weights loaded at lower precision).
//
// Format: E4M3 of the OCP 8-bit floating point specification (exponent bias
// 7, largest finite value 448, no infinities).  A group of values (one weight
// column over the reduction rows, one gathered activation row, one hidden
// row) shares the fp32 scale max|v| / 448 (1 for an all-zero group); a
// value's code is the E4M3 rounding (to nearest, ties to even, saturating at
// +-448) of the fp32 quotient v / scale.
//
// Kernels:
//   wq_amax_kernel     per-column max |w| over 64-row chunks (atomicMax on the
//                      fp32 bit patterns, which order like the non-negative
//                      values they encode);
//   wq_encode_kernel   codes of every weight, one thread per 16-byte vector;
//   wq_scale_kernel    max |w| -> scale, in place;
//   qrows_kernel       one block per row: max |v| over the row, then its codes
//                      (rows of up to 4 vectors per thread stay in registers;
//                      longer ones are read again, from L1/L2).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ float e4m3_scale(float amax) {
    return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
}

__device__ __forceinline__ uint32_t e4m3_code(float v, float scale) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v, scale), __NV_SATFINITE, __NV_E4M3));
}

// 16 bytes of bf16 (8 values) or fp32 (4 values) as floats.
template <bool kBf16>
__device__ __forceinline__ void unpack16(const uint4& q, float* f) {
    if (kBf16) {
        unpack_bf16x2(q.x, f[0], f[1]);
        unpack_bf16x2(q.y, f[2], f[3]);
        unpack_bf16x2(q.z, f[4], f[5]);
        unpack_bf16x2(q.w, f[6], f[7]);
    } else {
        f[0] = __uint_as_float(q.x);
        f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    }
}

// Codes of the 8 (bf16) or 4 (fp32) values of one vector, each with its scale.
template <bool kBf16>
__device__ __forceinline__ void store_codes(uint8_t* dst, const float* f, const float* sc) {
    if (kBf16) {
        uint2 c;
        c.x = e4m3_code(f[0], sc[0]) | (e4m3_code(f[1], sc[1]) << 8) | (e4m3_code(f[2], sc[2]) << 16) |
              (e4m3_code(f[3], sc[3]) << 24);
        c.y = e4m3_code(f[4], sc[4]) | (e4m3_code(f[5], sc[5]) << 8) | (e4m3_code(f[6], sc[6]) << 16) |
              (e4m3_code(f[7], sc[7]) << 24);
        *reinterpret_cast<uint2*>(dst) = c;
    } else {
        *reinterpret_cast<uint32_t*>(dst) = e4m3_code(f[0], sc[0]) | (e4m3_code(f[1], sc[1]) << 8) |
                                            (e4m3_code(f[2], sc[2]) << 16) | (e4m3_code(f[3], sc[3]) << 24);
    }
}

constexpr int kWqRows = 64;  // rows per amax block

template <bool kBf16>
__global__ void __launch_bounds__(256) wq_amax_kernel(const uint4* __restrict__ w, int rows, int vpr,
                                                      int cols, unsigned* __restrict__ amax_bits) {
    constexpr int kPer = kBf16 ? 8 : 4;
    const int v = blockIdx.x * 256 + threadIdx.x;
    const int e = blockIdx.z;
    const int r0 = blockIdx.y * kWqRows;
    if (v >= vpr) return;
    const int r1 = min(rows, r0 + kWqRows);
    float m[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) m[i] = 0.f;
    for (int r = r0; r < r1; ++r) {
        float f[kPer];
        unpack16<kBf16>(__ldg(w + (static_cast<int64_t>(e) * rows + r) * vpr + v), f);
#pragma unroll
        for (int i = 0; i < kPer; ++i) m[i] = fmaxf(m[i], fabsf(f[i]));  // NaN is ignored
    }
    unsigned* dst = amax_bits + static_cast<int64_t>(e) * cols + static_cast<int64_t>(v) * kPer;
#pragma unroll
    for (int i = 0; i < kPer; ++i) atomicMax(dst + i, __float_as_uint(m[i]));
}

template <bool kBf16>
__global__ void __launch_bounds__(256) wq_encode_kernel(const uint4* __restrict__ w, int64_t total_vec, int rows,
                                                        int vpr, int cols, const unsigned* __restrict__ amax_bits,
                                                        uint8_t* __restrict__ codes) {
    constexpr int kPer = kBf16 ? 8 : 4;
    const int64_t per_expert = static_cast<int64_t>(rows) * vpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_vec; i += stride) {
        const int64_t e = i / per_expert;
        const int v = static_cast<int>(i % vpr);
        const unsigned* ab = amax_bits + e * cols + static_cast<int64_t>(v) * kPer;
        float f[kPer], sc[kPer];
        unpack16<kBf16>(__ldg(w + i), f);
#pragma unroll
        for (int j = 0; j < kPer; ++j) sc[j] = e4m3_scale(__uint_as_float(__ldg(ab + j)));
        store_codes<kBf16>(codes + i * kPer, f, sc);
    }
}

__global__ void __launch_bounds__(256) wq_scale_kernel(float* __restrict__ scales, int64_t count) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < count) scales[i] = e4m3_scale(scales[i]);
}


// One block per row: max |v| over the row (block reduction), then its codes.
// kThreads = 512 for few rows (a row's vectors spread over more threads),
// 128 for many (four times the rows in flight per SM).  A row of at most
// 4 * kThreads vectors is read once and kept in registers for its codes.
template <bool kBf16, int kThreads>
__global__ void __launch_bounds__(kThreads) qrows_kernel(const uint4* __restrict__ src,
                                                         const int32_t* __restrict__ row_src,
                                                         int64_t src_rows, int64_t rows,
                                                         const int32_t* __restrict__ row_limit, int vpr,
                                                         uint8_t* __restrict__ codes,
                                                         float* __restrict__ scales) {
    griddep_wait();
    constexpr int kPer = kBf16 ? 8 : 4;
    __shared__ float s_max[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int64_t limit = rows;
    if (row_limit) limit = min(limit, static_cast<int64_t>(*row_limit));
    const int64_t cols = static_cast<int64_t>(vpr) * kPer;
    const bool one_pass = vpr <= 4 * kThreads;
    for (int64_t r = blockIdx.x; r < limit; r += gridDim.x) {
        int64_t s = r;
        if (row_src) {
            s = __ldg(row_src + r);
            if (s < 0 || s >= src_rows) continue;  // block-uniform
        }
        const uint4* row = src + s * vpr;
        // four vectors per thread in flight at once (zeros past the row end)
        float m = 0.f;
        uint4 q[4];
        for (int v0 = tid; v0 < vpr; v0 += 4 * kThreads) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + u * kThreads;
                q[u] = v < vpr ? __ldg(row + v) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float f[kPer];
                unpack16<kBf16>(q[u], f);
#pragma unroll
                for (int i = 0; i < kPer; ++i) m = fmaxf(m, fabsf(f[i]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_max[warp] = m;
        __syncthreads();
        m = s_max[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, s_max[w]);
        const float scale = e4m3_scale(m);
        float sc[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) sc[i] = scale;
        uint8_t* out = codes + r * cols;
        for (int v0 = tid; v0 < vpr; v0 += 4 * kThreads) {
            if (!one_pass) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int v = v0 + u * kThreads;
                    q[u] = v < vpr ? __ldg(row + v) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + u * kThreads;
                if (v < vpr) {
                    float f[kPer];
                    unpack16<kBf16>(q[u], f);
                    store_codes<kBf16>(out + static_cast<int64_t>(v) * kPer, f, sc);
                }
            }
        }
        if (tid == 0) scales[r] = scale;
        __syncthreads();  // s_max is reused by the next row
    }
    griddep_launch_dependents();
}

cudaError_t launch_quantize_weights_e4m3(const void* w, bool bf16, int n, int rows, int cols, uint8_t* codes,
                                         float* scales, int num_sms, cudaStream_t st) {
    const int per = bf16 ? 8 : 4;
    const int vpr = cols / per;
    const int64_t count = static_cast<int64_t>(n) * cols;
    cudaError_t e = cudaMemsetAsync(scales, 0, static_cast<size_t>(count) * sizeof(float), st);
    if (e != cudaSuccess) return e;
    unsigned* bits = reinterpret_cast<unsigned*>(scales);
    const dim3 ga(static_cast<unsigned>((vpr + 255) / 256), static_cast<unsigned>((rows + kWqRows - 1) / kWqRows),
                  static_cast<unsigned>(n));
    const int64_t total_vec = static_cast<int64_t>(n) * rows * vpr;
    int64_t blocks = (total_vec + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 32) blocks = static_cast<int64_t>(num_sms) * 32;
    if (blocks < 1) blocks = 1;
    if (bf16) {
        wq_amax_kernel<true><<<ga, 256, 0, st>>>(static_cast<const uint4*>(w), rows, vpr, cols, bits);
        wq_encode_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<const uint4*>(w), total_vec,
                                                                               rows, vpr, cols, bits, codes);
    } else {
        wq_amax_kernel<false><<<ga, 256, 0, st>>>(static_cast<const uint4*>(w), rows, vpr, cols, bits);
        wq_encode_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(static_cast<const uint4*>(w),
                                                                                total_vec, rows, vpr, cols, bits,
                                                                                codes);
    }
    wq_scale_kernel<<<static_cast<unsigned>((count + 255) / 256), 256, 0, st>>>(scales, count);
    return cudaGetLastError();
}

cudaError_t launch_quantize_rows_e4m3(const void* src, bool bf16, const int32_t* row_src, int64_t src_rows,
                                      int64_t rows, const int32_t* row_limit, int cols, uint8_t* codes,
                                      float* scales, int num_sms, cudaStream_t st) {
    const int vpr = cols / (bf16 ? 8 : 4);
    // 16 rows per SM in flight once there are enough rows (measured on the
    // prefill rows); a few long rows keep 512 threads each
    const bool many = rows >= 16LL * num_sms;
    int64_t blocks = rows;
    const int64_t cap = static_cast<int64_t>(num_sms) * (many ? 16 : 8);
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const dim3 g(static_cast<unsigned>(blocks));
    const uint4* s = static_cast<const uint4*>(src);
    if (bf16 && many)
        launch_k(qrows_kernel<true, 128>, g, dim3(128), 0, st, s, row_src, src_rows, rows, row_limit, vpr, codes,
                 scales);
    else if (bf16)
        launch_k(qrows_kernel<true, 512>, g, dim3(512), 0, st, s, row_src, src_rows, rows, row_limit, vpr, codes,
                 scales);
    else if (many)
        launch_k(qrows_kernel<false, 128>, g, dim3(128), 0, st, s, row_src, src_rows, rows, row_limit, vpr, codes,
                 scales);
    else
        launch_k(qrows_kernel<false, 512>, g, dim3(512), 0, st, s, row_src, src_rows, rows, row_limit, vpr, codes,
                 scales);
    return cudaGetLastError();
}

}  // namespace moe
