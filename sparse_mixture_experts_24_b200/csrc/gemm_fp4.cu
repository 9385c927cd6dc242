// gemm_fp4.cu -- grouped expert GEMMs with 4-bit weights and bf16
// activations on the sm_100a tensor cores.
//
//   GEMM1: H[r] = bf16( silu(st1 * Xp[r] . W1q[e]) * (st3 * Xp[r] . W3q[e]) )
//   GEMM2: O[r] = bf16( st2 * H[r] . W2q[e] )
// where Wq = E2M1(code) * sb is the block-scaled weight without its per-matrix
// scale st (format in fp4.cu).  Wq has at most 6 significant bits, so it is
// exact in bf16 and the bf16 MMA computes x . Wq with exact products; st is
// applied to the fp32 accumulators.  Source: the SwiGLU expert of the layer
// equation ("Mixtral of Experts" section 2.1, flash-card page) with the
// weights held at 4 bits ("Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists", Part 4).
//
// One persistent CTA per SM, 480 threads:
//   warp 0     TMA producer of the raw weight tiles (8-deep ring): two halves
//              of 128 columns x 64 K-rows of packed codes (64 bytes per row)
//              and their 4 x 128 block scales (GEMM1: w1 and w3 of the same
//              columns; GEMM2: two adjacent column halves of w2).
//   warp 14    TMA producer of A (4-deep ring): 128 rows x 64 of bf16 Xp or
//              H, K-major, 128-byte swizzle.
//   warps 6-13 converters (raw slot -> one of two B slots): codes -> bf16
//              values (byte permutes of an 8-entry magnitude table, sign bits
//              moved into place), times the block scales (bf16x2 multiplies,
//              exact), stored as the N-major 128-byte-swizzled B tile the MMA
//              reads (same layout as a TMA load of bf16 weights); then a proxy
//              fence and an arrive.
//   warp 1     MMA issuer: tcgen05.mma kind::f16 M=128 N=256 K=16, 512 TMEM
//              columns (two accumulators).
//   warps 2-5  epilogue: accumulators x st, SwiGLU (GEMM1) or copy (GEMM2),
//              bf16 rows.
// Every wait is bounded (common.cuh).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace fp4gemm {

constexpr int kBM = kTcBM;   // 128
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kABytes = kBM * kBK * 2;           // 16 KB
constexpr int kBChunkBytes = kBK * 64 * 2;       // 8 KB: 64 K-rows x 64 bf16 columns
constexpr int kBBytes = 4 * kBChunkBytes;        // 32 KB
constexpr int kCodeHalfBytes = kBK * 64;         // 4 KB: 64 K-rows x 128 columns at 4 bits
constexpr int kScaleHalfBytes = (kBK / 16) * 128;  // 512 B
constexpr int kRawBytes = 2 * kCodeHalfBytes + 2 * kScaleHalfBytes;  // 9 KB
// Three rings: the small raw weight tiles run far ahead (their loads carry
// the HBM latency), A tiles four deep, converted B tiles two deep (the
// conversion is a shared-memory to shared-memory step).
constexpr int kRawStages = 8;
constexpr int kAStages = 4;
constexpr int kBStages = 2;
constexpr int kAOff = 0;
constexpr int kBOff = kAOff + kAStages * kABytes;
constexpr int kRawOff = kBOff + kBStages * kBBytes;
constexpr int kRingBytes = kRawOff + kRawStages * kRawBytes;   // 200 KB
constexpr int kTmemCols = 512;
constexpr int kConvWarps = 8;
constexpr int kAWarp = 14;                       // the A producer
constexpr int kThreads = (7 + kConvWarps) * 32;  // 480
constexpr int kMaxN = 256;

static_assert(kBOff % 1024 == 0 && kRawOff % 1024 == 0, "swizzled tiles keep 1 KB alignment");

struct __align__(8) SmemTail {
    uint64_t raw_full[kRawStages];
    uint64_t raw_empty[kRawStages];
    uint64_t a_full[kAStages];
    uint64_t a_empty[kAStages];
    uint64_t b_full[kBStages];
    uint64_t b_empty[kBStages];
    uint64_t accum_full[2];
    uint64_t accum_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kMaxN + 1];
    int32_t mblk[kMaxN + 1];
};

constexpr int kTailBytes = (static_cast<int>(sizeof(SmemTail)) + 127) / 128 * 128;
constexpr int kSmemBytes = kRingBytes + kTailBytes + 1024;

// Ring position: slot and phase of the i-th use of a ring of `depth` slots.
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void next(int depth) {
        if (++slot == depth) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

struct Tile {
    int e, n_tile, row0, rows;
};

__device__ __forceinline__ Tile tile_at(int t, const int32_t* off, const int32_t* mblk, int n, int n_tiles) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mblk[mid] * n_tiles <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    Tile ti;
    ti.e = lo;
    const int local = t - mblk[lo] * n_tiles;
    const int mb_count = mblk[lo + 1] - mblk[lo];
    ti.n_tile = local / mb_count;
    const int m_blk = local - ti.n_tile * mb_count;
    ti.row0 = off[lo] + m_blk * kBM;
    ti.rows = min(kBM, off[lo + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ float silu(float a) { return a / (1.f + __expf(-a)); }

// 8 E2M1 codes (code i in bits 4i .. 4i+3) -> 8 bf16 values, two per word
// (code 2k in the low half of word k).  Magnitude u = code & 7 indexes an
// 8-entry table of bf16 bit patterns split into low and high bytes:
//   u      0     1     2     3     4     5     6     7
//   value  0     0.5   1     1.5   2     3     4     6
//   bf16   0000  3F00  3F80  3FC0  4000  4040  4080  40C0
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t c, uint32_t (&out)[4]) {
    constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;
    constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const uint32_t s = c >> (16 * q);          // codes 4q .. 4q+3 in bits 0..15
        const uint32_t sel = s & 0x7777u;          // magnitudes; the selector msb must stay clear
        const uint32_t lo = __byte_perm(kLo0, kLo1, sel);
        const uint32_t hi = __byte_perm(kHi0, kHi1, sel);
        uint32_t w0 = __byte_perm(lo, hi, 0x5140);  // codes 4q, 4q+1
        uint32_t w1 = __byte_perm(lo, hi, 0x7362);  // codes 4q+2, 4q+3
        w0 |= ((s << 12) & 0x8000u) | ((s << 24) & 0x80000000u);
        w1 |= ((s << 4) & 0x8000u) | ((s << 16) & 0x80000000u);
        out[2 * q] = w0;
        out[2 * q + 1] = w1;
    }
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    const __nv_bfloat162 r =
        __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a), *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t e4m3_to_bf16_bits(uint32_t code) {
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
    return __float_as_uint(__half2float(__half(h))) >> 16;  // exact: 3 mantissa bits
}

}  // namespace fp4gemm

using namespace fp4gemm;

// kSwiGLU: GEMM1 (halves = w1 and w3 of 128 columns); else GEMM2 (halves = two
// adjacent 128-column halves of w2).
template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_c0,
                    const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_c1,
                    const __grid_constant__ CUtensorMap tm_s1, const Fp4GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    SmemTail* tail = reinterpret_cast<SmemTail*>(smem + kRingBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRawStages; ++s) {
            mbar_init(smem_u32(&tail->raw_full[s]), 1);
            mbar_init(smem_u32(&tail->raw_empty[s]), kConvWarps);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(smem_u32(&tail->a_full[s]), 1);
            mbar_init(smem_u32(&tail->a_empty[s]), 1);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(smem_u32(&tail->b_full[s]), kConvWarps);
            mbar_init(smem_u32(&tail->b_empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tail->accum_full[b]), 1);
            mbar_init(smem_u32(&tail->accum_empty[b]), 4);
        }
        mbar_init(smem_u32(&tail->done), 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_c0);
        tma_prefetch_desc(&tm_s0);
        tma_prefetch_desc(&tm_c1);
        tma_prefetch_desc(&tm_s1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tail->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    griddep_wait();  // segment offsets and A come from the previous kernels
    for (int i = threadIdx.x; i <= n; i += kThreads) {
        tail->off[i] = args.offsets[i];
        tail->mblk[i] = args.mblk_base[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->mblk[n] * args.n_tiles;
    const int stride = args.balanced ? balanced_ctas(total_tiles, static_cast<int>(gridDim.x))
                                     : static_cast<int>(gridDim.x);
    const int first = static_cast<int>(blockIdx.x) < stride ? static_cast<int>(blockIdx.x) : total_tiles;
    int* status = args.status;

    if (warp == 0 || warp == kAWarp) {
        if (lane == 0) {
            // ---------------- TMA producers: raw weight tiles (warp 0), A tiles (warp 14) ----------------
            const bool raw_side = warp == 0;
            const int depth = raw_side ? kRawStages : kAStages;
            uint64_t* full = raw_side ? tail->raw_full : tail->a_full;
            uint64_t* empty = raw_side ? tail->raw_empty : tail->a_empty;
            Ring ring;
            int armed[kRawStages];
            for (int s = 0; s < kRawStages; ++s) armed[s] = -1;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride) {
                const Tile ti = tile_at(t, tail->off, tail->mblk, n, args.n_tiles);
                const int c0 = kSwiGLU ? ti.n_tile * 128 : ti.n_tile * 256;
                const int c1 = kSwiGLU ? c0 : c0 + 128;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[ring.slot]), ring.phase ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[ring.slot]);
                    armed[ring.slot] = static_cast<int>(ring.phase);
                    const int k0 = kb * kBK;
                    if (raw_side) {
                        mbar_arrive_expect_tx(fb, kRawBytes);
                        const uint32_t raw = smem_u32(smem + kRawOff + ring.slot * kRawBytes);
                        tma_load_3d(raw, &tm_c0, fb, c0 / 2, k0, ti.e);
                        tma_load_3d(raw + kCodeHalfBytes, &tm_c1, fb, c1 / 2, k0, ti.e);
                        tma_load_3d(raw + 2 * kCodeHalfBytes, &tm_s0, fb, c0, k0 / 16, ti.e);
                        tma_load_3d(raw + 2 * kCodeHalfBytes + kScaleHalfBytes, &tm_s1, fb, c1, k0 / 16, ti.e);
                    } else {
                        mbar_arrive_expect_tx(fb, kABytes);
                        tma_load_2d(smem_u32(smem + kAOff + ring.slot * kABytes), &tm_a, fb, k0, ti.row0);
                    }
                    ring.next(depth);
                }
            }
            for (int s = 0; s < depth; ++s)
                if (armed[s] >= 0)
                    mbar_wait(smem_u32(&full[s]), static_cast<uint32_t>(armed[s]), status, kStatusTimeoutDrain);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = make_idesc_bf16(kBM, kBN, 0, 1);
            Ring ra, rb;
            int local = 0;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride, ++local) {
                const int buf = local & 1;
                const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait(smem_u32(&tail->accum_empty[buf]), bph ^ 1u, status, kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->a_full[ra.slot]), ra.phase, status, kStatusTimeoutFull) ||
                        !mbar_wait(smem_u32(&tail->b_full[rb.slot]), rb.phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + kAOff + ra.slot * kABytes);
                    const uint32_t b_base = smem_u32(smem + kBOff + rb.slot * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(b_base + kk * 2048, kBChunkBytes, 1024, 2);
                        tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&tail->a_empty[ra.slot]));
                    tc_commit(smem_u32(&tail->b_empty[rb.slot]));
                    ra.next(kAStages);
                    rb.next(kBStages);
                }
                if (ok) tc_commit(smem_u32(&tail->accum_full[buf]));
            }
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else if (warp >= 6) {
        // ---------------- converters (warps 6..13) ----------------
        // Per stage: 2 halves x 16 groups of 8 columns x 4 blocks of 16 K-rows
        // = 128 items, two threads per item, each taking every other row of
        // the block (rows 2i + sub).  Warp w takes half w / 4 and block w % 4;
        // lane = 16 sub + g, so each quarter-warp (the unit of a 16-byte
        // shared store) writes 8 different 16-byte slots of one row, and the
        // half-warps' code loads of one row step cover all 32 banks.
        const int cw_idx = warp - 6;           // 0 .. 7
        const int h = cw_idx >> 2;
        const int kb16 = cw_idx & 3;
        const int g = lane & 15;
        const int sub = lane >> 4;
        const int col = h * 128 + g * 8;       // first of the 8 output columns
        const int chunk = col >> 6;            // 64-column chunk of the B tile
        const int u = (col & 63) >> 3;         // 16-byte unit inside a 128-byte row
        Ring rr, rb;
        bool ok = true;
        for (int t = first; t < total_tiles && ok; t += stride) {
            for (int kb = 0; kb < args.k_blocks; ++kb) {
                if (!mbar_wait(smem_u32(&tail->raw_full[rr.slot]), rr.phase, status, kStatusTimeoutFull) ||
                    !mbar_wait(smem_u32(&tail->b_empty[rb.slot]), rb.phase ^ 1u, status, kStatusTimeoutEmpty)) {
                    ok = false;
                    break;
                }
                const uint8_t* raw = smem + kRawOff + rr.slot * kRawBytes;
                const uint8_t* codes = raw + h * kCodeHalfBytes;
                const uint8_t* scales = raw + 2 * kCodeHalfBytes + h * kScaleHalfBytes;
                const uint2 sb8 = *reinterpret_cast<const uint2*>(scales + kb16 * 128 + g * 8);
                uint32_t cw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    cw[i] = *reinterpret_cast<const uint32_t*>(codes + (kb16 * 16 + 2 * i + sub) * 64 + g * 4);
                // the raw slot is read: hand it back to the producer
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tail->raw_empty[rr.slot]));
                uint32_t sp[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t word = q < 2 ? sb8.x : sb8.y;
                    const uint32_t b0 = (word >> (16 * (q & 1))) & 0xFFu;
                    const uint32_t b1 = (word >> (16 * (q & 1) + 8)) & 0xFFu;
                    sp[q] = e4m3_to_bf16_bits(b0) | (e4m3_to_bf16_bits(b1) << 16);
                }
                uint8_t* bdst = smem + kBOff + rb.slot * kBBytes + chunk * kBChunkBytes;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int k = kb16 * 16 + 2 * i + sub;
                    uint32_t w[4];
                    e2m1x8_to_bf16(cw[i], w);
                    uint4 v;
                    v.x = bf16x2_mul(w[0], sp[0]);
                    v.y = bf16x2_mul(w[1], sp[1]);
                    v.z = bf16x2_mul(w[2], sp[2]);
                    v.w = bf16x2_mul(w[3], sp[3]);
                    *reinterpret_cast<uint4*>(bdst + k * 128 + ((u ^ (k & 7)) << 4)) = v;
                }
                fence_proxy_async_smem();  // the tensor core reads these stores
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&tail->b_full[rb.slot]));
                rr.next(kRawStages);
                rb.next(kBStages);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quad = warp & 3;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const Tile ti = tile_at(t, tail->off, tail->mblk, n, args.n_tiles);
            const int buf = local & 1;
            const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tail->accum_full[buf]), bph, status, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kBN);
            const int valid = min(32, ti.rows - quad * 32);
            const bool row_ok = lane < valid;
            const int64_t row_base = static_cast<int64_t>(ti.row0) + quad * 32;
            uint16_t* out = static_cast<uint16_t*>(args.out);
            const float g0 = __ldg(args.tscale0 + ti.e);
            if (kSwiGLU) {
                const float g1 = __ldg(args.tscale1 + ti.e);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t a[32], b[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, a);
                    tmem_ld_32x32b_x32(tbase + 128 + c * 32, b);
                    tmem_wait_ld();
                    const int col = ti.n_tile * 128 + c * 32;
                    if (row_ok && col < args.out_cols) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float h0 = silu(__uint_as_float(a[2 * j]) * g0) * (__uint_as_float(b[2 * j]) * g1);
                            const float h1 =
                                silu(__uint_as_float(a[2 * j + 1]) * g0) * (__uint_as_float(b[2 * j + 1]) * g1);
                            pk[j] = pack_bf16x2(h0, h1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(out + (row_base + lane) * args.out_cols + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t a[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, a);
                    tmem_wait_ld();
                    const int col = ti.n_tile * 256 + c * 32;
                    if (row_ok && col < args.out_cols) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            pk[j] = pack_bf16x2(__uint_as_float(a[2 * j]) * g0, __uint_as_float(a[2 * j + 1]) * g0);
                        uint4* dst = reinterpret_cast<uint4*>(out + (row_base + lane) * args.out_cols + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tail->accum_empty[buf]));
        }
    }

    tc_fence_before();
    __syncthreads();
    griddep_launch_dependents();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <bool kSwiGLU>
static cudaError_t launch_fp4(const CUtensorMap& ta, const CUtensorMap& c0, const CUtensorMap& s0,
                              const CUtensorMap& c1, const CUtensorMap& s1, const Fp4GemmArgs& a, int num_sms,
                              cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(fp4_gemm_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + kBM - 1) / kBM + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    if (g < 1) g = 1;
    launch_k(fp4_gemm_kernel<kSwiGLU>, dim3(static_cast<unsigned>(g)), dim3(kThreads), kSmemBytes, st, ta, c0, s0,
             c1, s1, a);
    return cudaGetLastError();
}

cudaError_t launch_fp4_gemm1(const CUtensorMap& tm_xp, const CUtensorMap& tm_c1, const CUtensorMap& tm_s1,
                             const CUtensorMap& tm_c3, const CUtensorMap& tm_s3, const Fp4GemmArgs& a, int num_sms,
                             cudaStream_t st) {
    return launch_fp4<true>(tm_xp, tm_c1, tm_s1, tm_c3, tm_s3, a, num_sms, st);
}

cudaError_t launch_fp4_gemm2(const CUtensorMap& tm_h, const CUtensorMap& tm_c2, const CUtensorMap& tm_s2,
                             const Fp4GemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_fp4<false>(tm_h, tm_c2, tm_s2, tm_c2, tm_s2, a, num_sms, st);
}

}  // namespace moe
