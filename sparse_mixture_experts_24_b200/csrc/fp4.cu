// fp4.cu -- 4-bit expert weights: E2M1 values with an E4M3 scale per 16
// reduction rows of one output column and an fp32 scale per expert matrix
// (the weights held at 4 bits, "Mixture of Experts: Why Mixtral Only Wakes Up
// Two Specialists", Part 4, "Why total and active both matter").
//
//   st   = max|w| over the matrix / (6 * 448)          (1 for an all-zero matrix)
//   sb   = E4M3( (max|w| over the 16-row block / 6) / st ), round to nearest even
//   code = E2M1( w / (sb * st) ), round to nearest even, saturating at +-6
//          (0 when sb is 0), every quotient and product rounded to fp32
//   codes [n][rows][cols/2]: column 2j in the low nibble of byte j, 2j+1 in the
//   high nibble; bscale [n][rows/16][cols] E4M3 codes; tscale [n] fp32.
//
// Kernels: fp4_amax_kernel (max |w| per matrix, atomicMax on the fp32 bit
// patterns), fp4_quant_kernel (one thread per 16-row block of a column pair:
// the two block scales, then 16 code bytes), fp4_tscale_kernel (max -> st).
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ float fp4_tensor_scale(float amax) {
    return amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f;
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

template <bool kBf16>
__device__ __forceinline__ float load_w(const void* w, int64_t i) {
    if (kBf16) {
        const uint16_t b = __ldg(static_cast<const uint16_t*>(w) + i);
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    return __ldg(static_cast<const float*>(w) + i);
}

template <bool kBf16>
__global__ void __launch_bounds__(256) fp4_amax_kernel(const void* __restrict__ w, int64_t per_matrix,
                                                       unsigned* __restrict__ amax_bits) {
    const int e = blockIdx.y;
    float m = 0.f;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < per_matrix;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        m = fmaxf(m, fabsf(load_w<kBf16>(w, e * per_matrix + i)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + e, __float_as_uint(m));
}

// Thread = (matrix e, block b, column pair j).
template <bool kBf16>
__global__ void __launch_bounds__(256) fp4_quant_kernel(const void* __restrict__ w, int rows, int cols,
                                                        const unsigned* __restrict__ amax_bits,
                                                        uint8_t* __restrict__ codes, uint8_t* __restrict__ bscale) {
    const int pairs = cols / 2;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int nb = rows / 16;
    const int e = blockIdx.y;
    if (item >= static_cast<int64_t>(nb) * pairs) return;
    const int b = static_cast<int>(item / pairs);
    const int j = static_cast<int>(item - static_cast<int64_t>(b) * pairs);
    const float st = fp4_tensor_scale(__uint_as_float(__ldg(amax_bits + e)));
    const int64_t base = (static_cast<int64_t>(e) * rows + 16 * b) * cols + 2 * j;
    float v[2][16];
    float amax[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 16; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            v[h][r] = load_w<kBf16>(w, base + static_cast<int64_t>(r) * cols + h);
            amax[h] = fmaxf(amax[h], fabsf(v[h][r]));
        }
    float denom[2];
    uint32_t sb_code[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float qb = __fdiv_rn(__fdiv_rn(amax[h], 6.f), st);
        sb_code[h] = static_cast<uint32_t>(__nv_cvt_float_to_fp8(qb, __NV_SATFINITE, __NV_E4M3));
        denom[h] = __fmul_rn(e4m3_value(sb_code[h]), st);
    }
    uint8_t* bs = bscale + (static_cast<int64_t>(e) * nb + b) * cols + 2 * j;
    bs[0] = static_cast<uint8_t>(sb_code[0]);
    bs[1] = static_cast<uint8_t>(sb_code[1]);
    uint8_t* out = codes + (static_cast<int64_t>(e) * rows + 16 * b) * pairs + j;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        uint32_t c[2];
#pragma unroll
        for (int h = 0; h < 2; ++h)
            c[h] = denom[h] == 0.f ? 0u
                                   : static_cast<uint32_t>(__nv_cvt_float_to_fp4(__fdiv_rn(v[h][r], denom[h]),
                                                                                 __NV_E2M1, cudaRoundNearest)) &
                                         0xFu;
        out[static_cast<int64_t>(r) * pairs] = static_cast<uint8_t>(c[0] | (c[1] << 4));
    }
}

__global__ void __launch_bounds__(256) fp4_tscale_kernel(float* __restrict__ tscale, int n) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < n) tscale[e] = fp4_tensor_scale(tscale[e]);
}

cudaError_t launch_quantize_weights_fp4(const void* w, bool bf16, int n, int rows, int cols, uint8_t* codes,
                                        uint8_t* bscale, float* tscale, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(tscale, 0, static_cast<size_t>(n) * sizeof(float), st);
    if (e != cudaSuccess) return e;
    unsigned* bits = reinterpret_cast<unsigned*>(tscale);
    const int64_t per = static_cast<int64_t>(rows) * cols;
    int64_t bx = (per + 255) / 256;
    const int64_t cap = (static_cast<int64_t>(num_sms) * 8 + n - 1) / n;
    if (bx > cap) bx = cap;
    if (bx < 1) bx = 1;
    const dim3 ga(static_cast<unsigned>(bx), static_cast<unsigned>(n));
    const int64_t items = static_cast<int64_t>(rows / 16) * (cols / 2);
    const dim3 gq(static_cast<unsigned>((items + 255) / 256), static_cast<unsigned>(n));
    if (bf16) {
        fp4_amax_kernel<true><<<ga, 256, 0, st>>>(w, per, bits);
        fp4_quant_kernel<true><<<gq, 256, 0, st>>>(w, rows, cols, bits, codes, bscale);
    } else {
        fp4_amax_kernel<false><<<ga, 256, 0, st>>>(w, per, bits);
        fp4_quant_kernel<false><<<gq, 256, 0, st>>>(w, rows, cols, bits, codes, bscale);
    }
    fp4_tscale_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(tscale, n);
    return cudaGetLastError();
}

}  // namespace moe
