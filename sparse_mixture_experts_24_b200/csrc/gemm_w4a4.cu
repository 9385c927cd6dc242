// gemm_w4a4.cu -- grouped expert GEMMs with 4-bit weights and 4-bit
// activations on the sm_100a block-scaled tensor cores.
//
//   GEMM1: H[r] = bf16( silu(rx[r] st1[e] (Xq[r] . W1q[e])) * (rx[r] st3[e] (Xq[r] . W3q[e])) )
//   GEMM2: O[r] = bf16( rh[r] st2[e] (Hq[r] . W2q[e]) )
// where Xq, Hq, Wq are E2M1 codes times their E4M3 block scales (16 along K)
// -- the tensor core applies those -- and rx, rh, st are the fp32 row and
// matrix scales, applied to the accumulators.  Source: the SwiGLU expert of
// the layer equation ("Mixtral of Experts" section 2.1, flash-card page) with
// 4-bit weights ("Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists", Part 4).
//
// One persistent CTA per SM, 320 threads:
//   warp 0     TMA producer, 4-stage ring of 54 KB: per stage a K step of 256
//              (128 bytes of codes per row): A 128 rows (128-byte swizzle), B
//              256 rows of K-major weight codes (GEMM1: 128 columns of w1 and
//              the same of w3; GEMM2: 256 columns of w2), and by plain bulk
//              copies the matching 512-byte scale chunks (4 for A, 8 for B).
//   warp 1     allocates 512 TMEM columns (one 256-column accumulator, four
//              stages x 48 columns of scale factors); per 64-wide K step it
//              copies the scale chunks into TMEM (tcgen05.cp 32x128b.warpx4)
//              and issues tcgen05.mma kind::mxf4nvf4 block16 M=128 N=256.
//   warps 2-9  epilogue, two warps per TMEM lane quadrant splitting the
//              columns: accumulator x row scale x matrix scale, SwiGLU (GEMM1)
//              or a copy (GEMM2), bf16 rows.  With one accumulator the MMAs of
//              the next tile wait for the epilogue, so it is kept short.
// Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace w4gemm {

constexpr int kBM = kTcBM;   // 128
constexpr int kBN = 256;
constexpr int kABytes = kBM * 128;      // 16 KB
constexpr int kBHalfBytes = 128 * 128;  // 16 KB: 128 rows of 128 bytes
constexpr int kBBytes = 2 * kBHalfBytes;
constexpr int kSfaBytes = 4 * 512;
constexpr int kSfbBytes = 8 * 512;
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 54 KB
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, each taking half the columns
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int kMaxN = 256;
constexpr int kTmemCols = 512;
constexpr int kSfCols = 48;  // per stage: 4 K steps x (4 SFA + 8 SFB columns)

static_assert(kStageBytes % 1024 == 0, "stages keep the 1 KB alignment of the swizzled tiles");

struct __align__(8) SmemTail {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t accum_full;
    uint64_t accum_empty;
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kMaxN + 1];
    int32_t mblk[kMaxN + 1];
};

constexpr int kTailBytes = (static_cast<int>(sizeof(SmemTail)) + 127) / 128 * 128;
constexpr int kSmemBytes = kStages * kStageBytes + kTailBytes + 1024;

struct Tile {
    int e, n_tile, m_blk, row0, rows;
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
    ti.m_blk = local - ti.n_tile * mb_count;
    ti.row0 = off[lo] + ti.m_blk * kBM;
    ti.rows = min(kBM, off[lo + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ float silu(float a) { return __fdividef(a, 1.f + __expf(-a)); }

}  // namespace w4gemm

using namespace w4gemm;

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                     const __grid_constant__ CUtensorMap tm_b1, const W4a4GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    SmemTail* tail = reinterpret_cast<SmemTail*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
        }
        mbar_init(smem_u32(&tail->accum_full), 1);
        mbar_init(smem_u32(&tail->accum_empty), kEpiWarps);
        mbar_init(smem_u32(&tail->done), 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b0);
        tma_prefetch_desc(&tm_b1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tail->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    griddep_wait();
    for (int i = threadIdx.x; i <= n; i += kThreads) {
        tail->off[i] = args.offsets[i];
        tail->mblk[i] = args.mblk_base[i];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->mblk[n] * args.n_tiles;
    const int kb64_total = args.k_steps * 4;  // 64-wide K steps of the whole reduction
    int* status = args.status;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            int armed[kStages];
            for (int s = 0; s < kStages; ++s) armed[s] = -1;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const Tile ti = tile_at(t, tail->off, tail->mblk, n, args.n_tiles);
                // B rows (output columns) of the two halves and their scale-chunk blocks
                const int c0 = kSwiGLU ? ti.n_tile * 128 : ti.n_tile * 256;
                const int c1 = kSwiGLU ? c0 : c0 + 128;
                const int nb_per_e = args.n_cols / 128;
                const uint8_t* sfb0 = args.b_chunks0 + (static_cast<int64_t>(ti.e) * nb_per_e + c0 / 128) *
                                                           kb64_total * 512;
                const uint8_t* sfb1 = args.b_chunks1 + (static_cast<int64_t>(ti.e) * nb_per_e + c1 / 128) *
                                                           kb64_total * 512;
                const uint8_t* sfa =
                    args.a_chunks + (static_cast<int64_t>(tail->mblk[ti.e]) + ti.m_blk) * kb64_total * 512;
                for (int ks = 0; ks < args.k_steps; ++ks) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&tail->full[stage]);
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    armed[stage] = static_cast<int>(phase);
                    const uint32_t base = smem_u32(smem + stage * kStageBytes);
                    const int kx = ks * 128;  // byte column of the codes
                    tma_load_2d(base, &tm_a, fb, kx, ti.row0);
                    tma_load_3d(base + kABytes, &tm_b0, fb, kx, c0, ti.e);
                    tma_load_3d(base + kABytes + kBHalfBytes, &tm_b1, fb, kx, c1, ti.e);
                    const int64_t ck = static_cast<int64_t>(ks) * 4 * 512;
                    bulk_load(base + kABytes + kBBytes, sfa + ck, kSfaBytes, fb);
                    bulk_load(base + kABytes + kBBytes + kSfaBytes, sfb0 + ck, kSfbBytes / 2, fb);
                    bulk_load(base + kABytes + kBBytes + kSfaBytes + kSfbBytes / 2, sfb1 + ck, kSfbBytes / 2, fb);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0)
                    mbar_wait(smem_u32(&tail->full[s]), static_cast<uint32_t>(armed[s]), status, kStatusTimeoutDrain);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- scale-factor copies and MMA issue ----------------
            constexpr uint32_t idesc = make_idesc_fp4_block16(kBM, kBN);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++local) {
                if (!mbar_wait(smem_u32(&tail->accum_empty), (static_cast<uint32_t>(local) & 1u) ^ 1u, status,
                               kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < args.k_steps; ++ks) {
                    if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t base = smem_u32(smem + stage * kStageBytes);
                    const uint32_t sfa_smem = base + kABytes + kBBytes;
                    const uint32_t sfb_smem = sfa_smem + kSfaBytes;
                    const uint32_t sf_col = tmem_base + 256 + static_cast<uint32_t>(stage * kSfCols);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t sfa_t = sf_col + 4 * kk;
                        const uint32_t sfb_t = sf_col + 16 + 8 * kk;
                        tc_cp_32x128b_warpx4(sfa_t, make_smem_desc(sfa_smem + kk * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4(sfb_t, make_smem_desc(sfb_smem + kk * 512, 0, 128, 0));
                        tc_cp_32x128b_warpx4(sfb_t + 4, make_smem_desc(sfb_smem + kSfbBytes / 2 + kk * 512, 0, 128, 0));
                        const uint64_t adesc = make_smem_desc(base + kk * 32, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(base + kABytes + kk * 32, 16, 1024, 2);
                        tc_mma_fp4_block16(tmem_base, adesc, bdesc, idesc, sfa_t, sfb_t, (ks | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&tail->empty[stage]));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc_commit(smem_u32(&tail->accum_full));
            }
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        // warp w reads TMEM lanes 32 (w % 4) .. +31 and the column half (w - 2) / 4
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        int local = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++local) {
            const Tile ti = tile_at(t, tail->off, tail->mblk, n, args.n_tiles);
            const int valid = min(32, ti.rows - quad * 32);
            const bool row_ok = lane < valid;
            const int64_t row_base = static_cast<int64_t>(ti.row0) + quad * 32;
            // scales first: their loads overlap the wait for the accumulator
            const float rs = row_ok ? args.row_scale[row_base + lane] : 0.f;
            const float m0 = __ldg(args.mscale0 + ti.e);
            const float m1 = kSwiGLU ? __ldg(args.mscale1 + ti.e) : 0.f;
            if (!mbar_wait(smem_u32(&tail->accum_full), static_cast<uint32_t>(local) & 1u, status,
                           kStatusTimeoutAccum))
                break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
            uint16_t* out = static_cast<uint16_t*>(args.out);
            const float g0 = m0 * rs;
            if (kSwiGLU) {
                const float g1 = m1 * rs;
#pragma unroll 1
                for (int c = 2 * half; c < 2 * half + 2; ++c) {
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
                for (int c = 4 * half; c < 4 * half + 4; ++c) {
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
            if (lane == 0) mbar_arrive(smem_u32(&tail->accum_empty));
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
static cudaError_t launch_w4(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                             const W4a4GemmArgs& a, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + kBM - 1) / kBM + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    if (g < 1) g = 1;
    launch_k(w4a4_gemm_kernel<kSwiGLU>, dim3(static_cast<unsigned>(g)), dim3(kThreads), kSmemBytes, st, ta, tb0, tb1,
             a);
    return cudaGetLastError();
}

cudaError_t launch_w4a4_gemm1(const CUtensorMap& tm_xq, const CUtensorMap& tm_w1, const CUtensorMap& tm_w3,
                              const W4a4GemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_w4<true>(tm_xq, tm_w1, tm_w3, a, num_sms, st);
}

cudaError_t launch_w4a4_gemm2(const CUtensorMap& tm_hq, const CUtensorMap& tm_w2, const W4a4GemmArgs& a, int num_sms,
                              cudaStream_t st) {
    return launch_w4<false>(tm_hq, tm_w2, tm_w2, a, num_sms, st);
}

}  // namespace moe
