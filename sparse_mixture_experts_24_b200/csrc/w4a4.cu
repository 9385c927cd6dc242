// w4a4.cu -- operand preparation for the 4-bit tensor-core expert path
// (4-bit weights and 4-bit activations, "Mixture of Experts: Why Mixtral Only
// Wakes Up Two Specialists", Part 4: the weights held at 4 bits).
//
// The tcgen05 block-scaled MMA (kind::mxf4nvf4, block 16) reads both operands
// K-major (two E2M1 codes per byte, the lower K index in the low nibble) and
// takes the E4M3 block scales from tensor memory, copied there from shared
// memory in 512-byte chunks: a chunk holds the 4 scales (one per 16 K) of 128
// rows for one 64-wide K step, row r's 4 bytes at 16 * (r % 32) + 4 * (r / 32).
//
//   w4a4_pack_kernel   4-bit weights in the layout of moe_quantize_weights_fp4
//                      (codes [n][K][N/2], scales [n][K/16][N]) -> K-major codes
//                      [n][N][K/2] and scale chunks [n][N/128][K/64][512].
//                      Pair mode (w1 and w3): the packed matrix has 2N rows,
//                      each 128-row block holding 64 columns of w1 followed by
//                      the same 64 columns of w3, so one 128-row tile of it
//                      yields both projections of 64 hidden columns.
//   w4a4_rows_kernel   rows (gathered x rows or hidden rows, bf16) -> E2M1 codes
//                      [R][K/2], a fp32 scale per row, and the scale chunks of
//                      the GEMM's tiles of 128 (or 32) rows: row r of expert
//                      e's segment lands in tile mblk_base[e] + (r -
//                      offsets[e]) / tile_rows.
//   Row quantisation: rs = max|row| / (6 * 448) (1 for a zero row), block scale
//   sb = E4M3((max|block| / 6) / rs), code = E2M1(v / (sb * rs)) (0 when the
//   product is 0), every quotient and product rounded to fp32.
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ int w4_chunk_byte(int r, int s) { return 16 * (r & 31) + 4 * ((r & 127) >> 5) + s; }

// Thread = (matrix e, packed row c, 16 K-rows kb16): 8 packed bytes and 1
// scale.  Packed row c reads column c of matrix 0, or in pair mode column
// 64 (c / 128) + c % 64 of matrix (c % 128) / 64.
__global__ void __launch_bounds__(256) w4a4_pack_kernel(const uint8_t* __restrict__ codes0,
                                                        const uint8_t* __restrict__ bscale0,
                                                        const uint8_t* __restrict__ codes1,
                                                        const uint8_t* __restrict__ bscale1, int K, int N,
                                                        int rows_out, uint8_t* __restrict__ packed,
                                                        uint8_t* __restrict__ chunks) {
    const int e = blockIdx.z;
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    const int kb16 = blockIdx.y;
    if (c >= rows_out) return;
    int col = c;
    const uint8_t* codes = codes0;
    const uint8_t* bscale = bscale0;
    if (codes1) {
        col = 64 * (c >> 7) + (c & 63);
        if (c & 64) {
            codes = codes1;
            bscale = bscale1;
        }
    }
    const int64_t in_base = (static_cast<int64_t>(e) * K + kb16 * 16) * (N / 2) + col / 2;
    const int sh = 4 * (col & 1);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t nib = (__ldg(codes + in_base + static_cast<int64_t>(i) * (N / 2)) >> sh) & 0xFu;
        if (i < 8)
            lo |= nib << (4 * i);
        else
            hi |= nib << (4 * (i - 8));
    }
    uint2* dst = reinterpret_cast<uint2*>(packed + (static_cast<int64_t>(e) * rows_out + c) * (K / 2) + kb16 * 8);
    *dst = make_uint2(lo, hi);
    const int KB = K / 64;
    const int64_t chunk = (static_cast<int64_t>(e) * (rows_out / 128) + c / 128) * KB + kb16 / 4;
    chunks[chunk * 512 + w4_chunk_byte(c, kb16 & 3)] =
        __ldg(bscale + (static_cast<int64_t>(e) * (K / 16) + kb16) * N + col);
}

cudaError_t launch_w4a4_pack(const uint8_t* codes, const uint8_t* bscale, const uint8_t* codes_pair,
                             const uint8_t* bscale_pair, int n, int K, int N, uint8_t* packed, uint8_t* chunks,
                             cudaStream_t st) {
    const int rows_out = codes_pair ? 2 * N : N;
    const dim3 grid(static_cast<unsigned>((rows_out + 255) / 256), static_cast<unsigned>(K / 16),
                    static_cast<unsigned>(n));
    w4a4_pack_kernel<<<grid, 256, 0, st>>>(codes, bscale, codes_pair, bscale_pair, K, N, rows_out, packed, chunks);
    return cudaGetLastError();
}

__device__ __forceinline__ float w4_tensor_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 2688.f) : 1.f; }

__device__ __forceinline__ float w4_e4m3_value(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __half2float(__half(h));
}

// One block per row; thread = blocks of 16 elements (bf16 source).  kThreads
// = 256 for few rows, 128 for many (twice the rows in flight per SM).
template <int kThreads>
__global__ void __launch_bounds__(kThreads) w4a4_rows_kernel(const uint16_t* __restrict__ src,
                                                                  const int32_t* __restrict__ row_src,
                                                                  int64_t src_rows, int K,
                                                                  const int32_t* __restrict__ offsets,
                                                                  const int32_t* __restrict__ mblk_base, int n,
                                                                  int tile_rows, uint8_t* __restrict__ codes,
                                                                  uint8_t* __restrict__ chunks,
                                                                  float* __restrict__ rscale) {
    griddep_wait();
    __shared__ float s_max[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rows = offsets[n];
    const int nblk = K / 16;
    const int KB = K / 64;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        int64_t s = r;
        if (row_src) {
            s = __ldg(row_src + r);
            if (s < 0 || s >= src_rows) continue;  // block-uniform
        }
        const uint4* row = reinterpret_cast<const uint4*>(src + s * K);
        float m = 0.f;
        for (int b = tid; b < nblk; b += kThreads) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 q = __ldg(row + 2 * b + h);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
                    m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_max[warp] = m;
        __syncthreads();
        m = s_max[0];
#pragma unroll
        for (int w = 1; w < kThreads / 32; ++w) m = fmaxf(m, s_max[w]);
        const float rs = w4_tensor_scale(m);
        // the row's tile and its row inside the tile
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= r)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t local = r - offsets[lo];
        const int64_t tile = mblk_base[lo] + local / tile_rows;
        const int tr = static_cast<int>(local % tile_rows);
        for (int b = tid; b < nblk; b += kThreads) {
            float v[16];
            float amax_b = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 q = __ldg(row + 2 * b + h);
                const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
                    v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) amax_b = fmaxf(amax_b, fabsf(v[i]));
            const uint32_t sb = static_cast<uint32_t>(
                __nv_cvt_float_to_fp8(__fdiv_rn(__fdiv_rn(amax_b, 6.f), rs), __NV_SATFINITE, __NV_E4M3));
            const float denom = __fmul_rn(w4_e4m3_value(sb), rs);
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t c =
                    denom == 0.f ? 0u
                                 : static_cast<uint32_t>(__nv_cvt_float_to_fp4(__fdiv_rn(v[i], denom), __NV_E2M1,
                                                                               cudaRoundNearest)) & 0xFu;
                packed[i >> 3] |= c << (4 * (i & 7));
            }
            *reinterpret_cast<uint2*>(codes + r * (K / 2) + 8 * b) = make_uint2(packed[0], packed[1]);
            chunks[(tile * KB + b / 4) * 512 + w4_chunk_byte(tr, b & 3)] = static_cast<uint8_t>(sb);
        }
        if (tid == 0) rscale[r] = rs;
        __syncthreads();  // s_max is reused by the next row
    }
    griddep_launch_dependents();
}

// Rows of up to 32 * 16 * kBPL elements: one warp per row, lane = blocks of 16
// (b = lane + 32 i), the whole row held in registers, so there is one read of
// the row, a warp-shuffle maximum and no block barrier.  Same arithmetic as
// w4a4_rows_kernel.
template <int kBPL>
__global__ void __launch_bounds__(256) w4a4_rows_warp_kernel(const uint16_t* __restrict__ src,
                                                             const int32_t* __restrict__ row_src,
                                                             int64_t src_rows, int K,
                                                             const int32_t* __restrict__ offsets,
                                                             const int32_t* __restrict__ mblk_base, int n,
                                                             int tile_rows, uint8_t* __restrict__ codes,
                                                             uint8_t* __restrict__ chunks,
                                                             float* __restrict__ rscale) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t rows = offsets[n];
    const int nblk = K / 16;
    const int KB = K / 64;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += warps) {
        int64_t s = r;
        if (row_src) {
            s = __ldg(row_src + r);
            if (s < 0 || s >= src_rows) continue;  // warp-uniform
        }
        const uint4* row = reinterpret_cast<const uint4*>(src + s * K);
        uint4 q[kBPL][2];
        float m = 0.f;
#pragma unroll
        for (int i = 0; i < kBPL; ++i) {
            const int b = lane + 32 * i;
            if (b < nblk) {
                q[i][0] = __ldg(row + 2 * b);
                q[i][1] = __ldg(row + 2 * b + 1);
            } else {
                q[i][0] = q[i][1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float amax_b[kBPL];
#pragma unroll
        for (int i = 0; i < kBPL; ++i) {
            float a = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w[4] = {q[i][h].x, q[i][h].y, q[i][h].z, q[i][h].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    a = fmaxf(a, fabsf(__uint_as_float(w[j] << 16)));
                    a = fmaxf(a, fabsf(__uint_as_float(w[j] & 0xFFFF0000u)));
                }
            }
            amax_b[i] = a;
            m = fmaxf(m, a);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float rs = w4_tensor_scale(m);
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (offsets[mid] <= r)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t local = r - offsets[lo];
        const int64_t tile = mblk_base[lo] + local / tile_rows;
        const int tr = static_cast<int>(local % tile_rows);
#pragma unroll
        for (int i = 0; i < kBPL; ++i) {
            const int b = lane + 32 * i;
            if (b >= nblk) continue;
            const uint32_t sb = static_cast<uint32_t>(
                __nv_cvt_float_to_fp8(__fdiv_rn(__fdiv_rn(amax_b[i], 6.f), rs), __NV_SATFINITE, __NV_E4M3));
            const float denom = __fmul_rn(w4_e4m3_value(sb), rs);
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w[4] = {q[i][h].x, q[i][h].y, q[i][h].z, q[i][h].w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float v = (j & 1) ? __uint_as_float(w[j >> 1] & 0xFFFF0000u) : __uint_as_float(w[j >> 1] << 16);
                    const uint32_t c =
                        denom == 0.f ? 0u
                                     : static_cast<uint32_t>(__nv_cvt_float_to_fp4(__fdiv_rn(v, denom), __NV_E2M1,
                                                                                   cudaRoundNearest)) & 0xFu;
                    packed[h] |= c << (4 * j);
                }
            }
            *reinterpret_cast<uint2*>(codes + r * (K / 2) + 8 * b) = make_uint2(packed[0], packed[1]);
            chunks[(tile * KB + b / 4) * 512 + w4_chunk_byte(tr, b & 3)] = static_cast<uint8_t>(sb);
        }
        if (lane == 0) rscale[r] = rs;
    }
    griddep_launch_dependents();
}

cudaError_t launch_w4a4_rows(const uint16_t* src, const int32_t* row_src, int64_t src_rows, int64_t rows_max, int K,
                             const int32_t* offsets, const int32_t* mblk_base, int n, int tile_rows, uint8_t* codes,
                             uint8_t* chunks, float* rscale, int num_sms, cudaStream_t st) {
    if (tile_rows != 128 && tile_rows != 32) return cudaErrorInvalidValue;
    // Many rows of at most 2,048 elements: a warp per row, the row in
    // registers (measured: many_expert x rows 82 -> 51 us, its H rows and
    // GEMM1 139 -> 85 us).  Longer rows, or few of them, keep a block per row:
    // a warp per 4,096-element row ran the decode x rows at half the speed
    // (64 rows: too few warps in flight) and the prefill ones 1.5x slower.
    const int bpl = (K / 16 + 31) / 32;
    if (bpl <= 4 && rows_max >= 4LL * num_sms) {
        int64_t wblocks = (rows_max + 7) / 8;
        if (wblocks > static_cast<int64_t>(num_sms) * 8) wblocks = static_cast<int64_t>(num_sms) * 8;
        if (wblocks < 1) wblocks = 1;
        const dim3 g(static_cast<unsigned>(wblocks));
        if (bpl <= 2)
            launch_k(w4a4_rows_warp_kernel<2>, g, dim3(256), 0, st, src, row_src, src_rows, K, offsets, mblk_base, n,
                     tile_rows, codes, chunks, rscale);
        else
            launch_k(w4a4_rows_warp_kernel<4>, g, dim3(256), 0, st, src, row_src, src_rows, K, offsets, mblk_base, n,
                     tile_rows, codes, chunks, rscale);
        return cudaGetLastError();
    }
    const bool many = rows_max >= 16LL * num_sms;
    int64_t blocks = rows_max;
    const int64_t cap = static_cast<int64_t>(num_sms) * (many ? 16 : 8);
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    if (many)
        launch_k(w4a4_rows_kernel<128>, dim3(static_cast<unsigned>(blocks)), dim3(128), 0, st, src, row_src,
                 src_rows, K, offsets, mblk_base, n, tile_rows, codes, chunks, rscale);
    else
        launch_k(w4a4_rows_kernel<256>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, src, row_src,
                 src_rows, K, offsets, mblk_base, n, tile_rows, codes, chunks, rscale);
    return cudaGetLastError();
}

}  // namespace moe
