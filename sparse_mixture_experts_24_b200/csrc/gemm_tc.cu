// gemm_tc.cu -- bf16 grouped expert GEMMs on the sm_100a tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA).
//
//   GEMM1: H[r] = bf16( silu(Xp[r] . w1[e]) * (Xp[r] . w3[e]) )  rows r of expert e
//   GEMM2: O[r] = bf16( H[r] . w2[e] )
//
// Source: the SwiGLU expert of the layer equation, SwiGLU_i(x) = (silu(x.w1_i)
// (*) x.w3_i) . w2_i ("Mixtral of Experts" section 2.1, flash-card page), with
// three 4,096 x 14,336 matrices per expert (Part 4 of "Mixture of Experts: Why
// Mixtral Only Wakes Up Two Specialists"), run only on the rows routed to the
// expert (Part 3, Step 2: unchosen experts are not run).
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0   one thread issues TMA loads into a kStages-deep ring of shared
//            memory stages (A: 128 rows x 64 of Xp or H, K-major, 128-byte
//            swizzle; B: 64 x 256 of the weights, N-major, as four 64-column
//            boxes, 128-byte swizzle).  GEMM1's B is 128 columns of w1 next to
//            the same 128 columns of w3, so ONE N=256 MMA produces both the
//            gate and the up projection of a 128-column slice of H.
//   warp 1   allocates 512 TMEM columns (two 256-column fp32 accumulators);
//            one thread issues tcgen05.mma (M=128, N=256, K=16) and commits
//            to the stage's "empty" barrier and, per tile, to "accum full".
//   warps 2-5 epilogue: tcgen05.ld of the accumulator (thread = row),
//            silu(a)*b (GEMM1) or a copy (GEMM2), bf16 rounding, 16-byte
//            stores; rows past the expert's segment and columns past the
//            matrix are not stored.
// Tiles are (expert, column tile, 128-row block) ordered so that CTAs running
// at the same time share a weight tile through L2.  The tile list comes from
// the per-expert M-block prefix the dispatch wrote, so nothing returns to the
// host between routing and the experts.
//
// E4M3 variant (kFp8): the same pipeline over 8-bit operands (a stage is 128
// K-elements: A 128 x 128 bytes; B two 128-column boxes of 128 K-rows), four
// kind::f8f6f4 MMAs (K = 32) per stage, and epilogues that undo the scales:
// GEMM1 multiplies the accumulators by the row's activation scale and the
// column's weight scale before the SwiGLU, GEMM2 by the hidden row's scale and
// the column's w2 scale.
//
// Every wait is bounded (common.cuh): a pipeline that stops making progress
// sets a status bit and the CTA drains and exits instead of hanging.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBM = kTcBM;           // 128 rows per tile (MMA M)
constexpr int kBN = 256;             // MMA N
constexpr int kBK = 64;              // K per stage (one 128-byte swizzle row of bf16)
constexpr int kBK8 = 128;            // K per stage of the E4M3 kernels (128 bytes too)
constexpr int kB8ChunkBytes = kBK8 * 128;         // 16 KB: 128 K-rows x 128 one-byte columns
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;            // 16 KB
constexpr int kBChunkBytes = kBK * 64 * 2;        // 8 KB: 64 K-rows x 64 columns
constexpr int kBBytes = 4 * kBChunkBytes;         // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;    // 48 KB
constexpr int kTmemCols = 512;
constexpr int kThreads = 192;
constexpr int kMaxN = 256;

struct __align__(8) TcSmemTail {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t accum_full[2];
    uint64_t accum_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kMaxN + 1];
    int32_t mblk[kMaxN + 1];
};

constexpr int kTailBytes = (static_cast<int>(sizeof(TcSmemTail)) + 127) / 128 * 128;
constexpr int kSmemBytes = kStages * kStageBytes + kTailBytes + 4 * kWarpStageBytes + 1024;

struct TileInfo {
    int e, n_tile, row0, rows;
};

// Tile order.  Tile t -> (expert, column tile, row block).  Per expert, with
// A_e = its row blocks x a_blk_bytes and B_e = its column tiles x b_tile_bytes:
//   plain   (A_e fits in the band budget, or no bands): the row block runs
//           fastest over the whole expert; A_e stays in L2 while every
//           column tile streams past it once.
//   m-bands the row blocks are cut into bands of band_m blocks (the last may
//           be shorter), row block fastest within a band: a band's A rows
//           stay in L2, B_e streams once per band.
//   n-bands the column tiles are cut into bands of band_n tiles, column tile
//           fastest within a row block: a band's weight tiles stay in L2, A_e
//           streams once per band.
// Bands are chosen per expert by the smaller DRAM estimate (A_e + bands x B_e
// against B_e + bands x A_e), so experts of a few row blocks keep the plain
// order and a very large one (a skewed router's favourite) gets bands.
struct TileOrder {
    int band_m, band_n;             // 0: no bands
    int64_t a_blk_bytes, b_tile_bytes;
};

__device__ __forceinline__ TileInfo tile_info(int t, const int32_t* off, const int32_t* mblk, int n,
                                              int n_tiles, const TileOrder& ord) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (mblk[mid] * n_tiles <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int e = lo;
    const int local = t - mblk[e] * n_tiles;
    const int mb_count = mblk[e + 1] - mblk[e];
    int mode = 0;  // 0 plain, 1 m-bands, 2 n-bands
    if (ord.band_m > 0 && mb_count > ord.band_m) {
        const int64_t A = static_cast<int64_t>(mb_count) * ord.a_blk_bytes;
        const int64_t B = static_cast<int64_t>(n_tiles) * ord.b_tile_bytes;
        const int64_t cm = A + static_cast<int64_t>((mb_count + ord.band_m - 1) / ord.band_m) * B;
        const int64_t cn = ord.band_n > 0 ? B + static_cast<int64_t>((n_tiles + ord.band_n - 1) / ord.band_n) * A
                                          : cm + 1;
        mode = cn < cm ? 2 : 1;
    }
    int n_tile, m_blk;
    if (mode == 2) {
        const int band = ord.band_n;
        const int full = n_tiles / band * band;   // column tiles in whole bands
        if (local < full * mb_count) {
            const int b = local / (band * mb_count);
            const int r = local - b * band * mb_count;
            m_blk = r / band;
            n_tile = b * band + (r - m_blk * band);
        } else {
            const int rem = n_tiles - full;
            const int r = local - full * mb_count;
            m_blk = r / rem;
            n_tile = full + (r - m_blk * rem);
        }
    } else {
        const int band = mode == 1 ? ord.band_m : mb_count;
        const int full = mb_count / band * band;  // row blocks in whole bands
        if (local < full * n_tiles) {
            const int b = local / (band * n_tiles);
            const int r = local - b * band * n_tiles;
            n_tile = r / band;
            m_blk = b * band + (r - n_tile * band);
        } else {
            const int rem = mb_count - full;
            const int r = local - full * n_tiles;
            n_tile = r / rem;
            m_blk = full + (r - n_tile * rem);
        }
    }
    TileInfo ti;
    ti.e = e;
    ti.n_tile = n_tile;
    ti.row0 = off[e] + m_blk * kBM;
    ti.rows = min(kBM, off[e + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.f + __expf(-a)); }

// Order of the reduction blocks of a tile.  GEMM2 (kSwiGLU false) walks K
// downwards on odd column tiles: the tiles of one expert's row block that fall
// into consecutive persistent rounds then meet at the same end of K, where the
// H rows the previous round read last are still in L2 (measured on the prefill
// shapes: 1.16x the algorithmic DRAM bytes with one direction).  The direction
// depends only on the column tile, so every output element is summed in one
// fixed order however the rows are tiled.
template <bool kSwiGLU>
__device__ __forceinline__ int k_block_at_t(int kb, int k_blocks, int n_tile, int alternate) {
    return (!kSwiGLU && alternate && (n_tile & 1)) ? k_blocks - 1 - kb : kb;
}

// kSwiGLU: GEMM1 (two B maps, 128 output columns per tile); else GEMM2.
// kFp8: E4M3 operands with the scales of TcGemmArgs applied in the epilogue.
template <bool kSwiGLU, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                   const __grid_constant__ CUtensorMap tm_b1, const TcGemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    TcSmemTail* tail = reinterpret_cast<TcSmemTail*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
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
        tma_prefetch_desc(&tm_b0);
        if (kSwiGLU) tma_prefetch_desc(&tm_b1);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tail->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    // everything above overlaps the previous kernel; its outputs (segment
    // offsets, the A operand) are read only after this wait
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
    const int stride = args.balanced ? balanced_ctas(total_tiles, static_cast<int>(gridDim.x))
                                     : static_cast<int>(gridDim.x);
    const int first = static_cast<int>(blockIdx.x) < stride ? static_cast<int>(blockIdx.x) : total_tiles;
    TileOrder ord;
    ord.band_m = args.band_m;
    ord.band_n = args.band_n;
    ord.a_blk_bytes = static_cast<int64_t>(kBM) * args.k_blocks * (kFp8 ? kBK8 : kBK * 2);
    ord.b_tile_bytes = static_cast<int64_t>(kBN) * args.k_blocks * (kFp8 ? kBK8 : kBK * 2);
    int* status = args.status;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            int armed[kStages];
            for (int s = 0; s < kStages; ++s) armed[s] = -1;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride) {
                const TileInfo ti = tile_info(t, tail->off, tail->mblk, n, args.n_tiles, ord);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status,
                                   kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&tail->full[stage]);
                    mbar_arrive_expect_tx(fb, kStageBytes);
                    armed[stage] = static_cast<int>(phase);
                    const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b_dst = a_dst + kABytes;
                    const int k0 = k_block_at_t<kSwiGLU>(kb, args.k_blocks, ti.n_tile, args.k_alternate) * (kFp8 ? kBK8 : kBK);
                    tma_load_2d(a_dst, &tm_a, fb, k0, ti.row0);
                    if (kFp8) {
                        if (kSwiGLU) {
                            const int c0 = ti.n_tile * 128;
                            tma_load_3d(b_dst, &tm_b0, fb, c0, k0, ti.e);
                            tma_load_3d(b_dst + kB8ChunkBytes, &tm_b1, fb, c0, k0, ti.e);
                        } else {
                            const int c0 = ti.n_tile * 256;
                            tma_load_3d(b_dst, &tm_b0, fb, c0, k0, ti.e);
                            tma_load_3d(b_dst + kB8ChunkBytes, &tm_b0, fb, c0 + 128, k0, ti.e);
                        }
                    } else if (kSwiGLU) {
                        const int c0 = ti.n_tile * 128;
                        tma_load_3d(b_dst + 0 * kBChunkBytes, &tm_b0, fb, c0, k0, ti.e);
                        tma_load_3d(b_dst + 1 * kBChunkBytes, &tm_b0, fb, c0 + 64, k0, ti.e);
                        tma_load_3d(b_dst + 2 * kBChunkBytes, &tm_b1, fb, c0, k0, ti.e);
                        tma_load_3d(b_dst + 3 * kBChunkBytes, &tm_b1, fb, c0 + 64, k0, ti.e);
                    } else {
                        const int c0 = ti.n_tile * 256;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_3d(b_dst + c * kBChunkBytes, &tm_b0, fb, c0 + 64 * c, k0, ti.e);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Drain: no TMA write may still be in flight when the CTA exits.
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0)
                    mbar_wait(smem_u32(&tail->full[s]), static_cast<uint32_t>(armed[s]), status,
                              kStatusTimeoutDrain);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            constexpr uint32_t idesc = kFp8 ? make_idesc_e4m3(kBM, kBN, 0, 1) : make_idesc_bf16(kBM, kBN, 0, 1);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int t = first; t < total_tiles && ok; t += stride, ++local) {
                const int buf = local & 1;
                const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait(smem_u32(&tail->accum_empty[buf]), bph ^ 1u, status,
                               kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b_base = a_base + kABytes;
                    if (kFp8) {
#pragma unroll
                        for (int kk = 0; kk < kBK8 / 32; ++kk) {
                            // A: K-major, 128-byte swizzle; K by 32 one-byte elements moves 32
                            // bytes inside the swizzle row.  B: N-major, 128-byte swizzle, two
                            // 128-column chunks 16 KB apart (LBO); K by 32 = four 8-row groups.
                            const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
                            const uint64_t bdesc =
                                make_smem_desc(b_base + kk * 4096, kB8ChunkBytes, 1024, 2);
                            tc_mma_f8(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        // A: K-major, 128-byte swizzle; advancing K by 16 moves 32 bytes
                        // inside the swizzle row.  SBO = 1024 (8 rows x 128 B).
                        const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
                        // B: N-major, 128-byte swizzle; K by 16 = two 8-row groups (2 KB).
                        // LBO = 8 KB between 64-column chunks, SBO = 1 KB between 8-row groups.
                        const uint64_t bdesc =
                            make_smem_desc(b_base + kk * 2048, kBChunkBytes, 1024, 2);
                        tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    }
                    tc_commit(smem_u32(&tail->empty[stage]));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc_commit(smem_u32(&tail->accum_full[buf]));
            }
            // All MMAs of this CTA must be finished before TMEM is freed.
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
        uint8_t* stage = smem + kStages * kStageBytes + kTailBytes + (warp - 2) * kWarpStageBytes;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const TileInfo ti = tile_info(t, tail->off, tail->mblk, n, args.n_tiles, ord);
            const int buf = local & 1;
            const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tail->accum_full[buf]), bph, status, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kBN);
            // this warp's 32 rows: [row0 + 32*quad, ...), `valid` of them inside the segment
            const int valid = min(32, ti.rows - quad * 32);
            const int64_t row_base = static_cast<int64_t>(ti.row0) + quad * 32;
            uint16_t* out = static_cast<uint16_t*>(args.out);
            if (kSwiGLU) {
                // GEMM1: direct 16-byte stores of each lane's row (measured faster here
                // than staging through shared memory)
                const bool row_ok = lane < valid;
                const float rs = (kFp8 && row_ok) ? args.row_scale[row_base + lane] : 1.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t a[32], b[32];
                    tmem_ld_32x32b_x32(tbase + c * 32, a);
                    tmem_ld_32x32b_x32(tbase + 128 + c * 32, b);
                    tmem_wait_ld();
                    const int col = ti.n_tile * 128 + c * 32;
                    if (row_ok && col < args.out_cols) {
                        if (kFp8) {
                            // dequantise: accumulator x row scale x column scale
                            const float4* s0 = reinterpret_cast<const float4*>(
                                args.col_scale0 + static_cast<int64_t>(ti.e) * args.out_cols + col);
                            const float4* s1 = reinterpret_cast<const float4*>(
                                args.col_scale1 + static_cast<int64_t>(ti.e) * args.out_cols + col);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 u = __ldg(s0 + q), v = __ldg(s1 + q);
                                a[4 * q + 0] = __float_as_uint(__uint_as_float(a[4 * q + 0]) * rs * u.x);
                                a[4 * q + 1] = __float_as_uint(__uint_as_float(a[4 * q + 1]) * rs * u.y);
                                a[4 * q + 2] = __float_as_uint(__uint_as_float(a[4 * q + 2]) * rs * u.z);
                                a[4 * q + 3] = __float_as_uint(__uint_as_float(a[4 * q + 3]) * rs * u.w);
                                b[4 * q + 0] = __float_as_uint(__uint_as_float(b[4 * q + 0]) * rs * v.x);
                                b[4 * q + 1] = __float_as_uint(__uint_as_float(b[4 * q + 1]) * rs * v.y);
                                b[4 * q + 2] = __float_as_uint(__uint_as_float(b[4 * q + 2]) * rs * v.z);
                                b[4 * q + 3] = __float_as_uint(__uint_as_float(b[4 * q + 3]) * rs * v.w);
                            }
                        }
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float h0 = silu_f(__uint_as_float(a[2 * j])) * __uint_as_float(b[2 * j]);
                            const float h1 =
                                silu_f(__uint_as_float(a[2 * j + 1])) * __uint_as_float(b[2 * j + 1]);
                            pk[j] = pack_bf16x2(h0, h1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(out + (row_base + lane) * args.out_cols + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            } else {
                const float rs = (kFp8 && lane < valid) ? args.row_scale[row_base + lane] : 1.f;
#pragma unroll 1
                for (int g = 0; g < 4; ++g) {
                    uint32_t pk[32];
                    const int col = ti.n_tile * 256 + g * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t a[32];
                        tmem_ld_32x32b_x32(tbase + g * 64 + c * 32, a);
                        tmem_wait_ld();
                        if (kFp8 && col < args.out_cols) {
                            const float4* s0 = reinterpret_cast<const float4*>(
                                args.col_scale0 + static_cast<int64_t>(ti.e) * args.out_cols + col + c * 32);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 u = __ldg(s0 + q);
                                a[4 * q + 0] = __float_as_uint(__uint_as_float(a[4 * q + 0]) * rs * u.x);
                                a[4 * q + 1] = __float_as_uint(__uint_as_float(a[4 * q + 1]) * rs * u.y);
                                a[4 * q + 2] = __float_as_uint(__uint_as_float(a[4 * q + 2]) * rs * u.z);
                                a[4 * q + 3] = __float_as_uint(__uint_as_float(a[4 * q + 3]) * rs * u.w);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            pk[c * 16 + j] = pack_bf16x2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1]));
                    }
                    if (col < args.out_cols && valid > 0)
                        warp_store_rows_64(stage, pk, lane, out, args.out_cols, row_base, valid, col);
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

static int grid_for(const TcGemmArgs& a, int num_sms) {
    const int64_t max_tiles = ((a.R + kBM - 1) / kBM + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    return static_cast<int>(g < 1 ? 1 : g);
}

template <bool kSwiGLU, bool kFp8>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                             const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<kSwiGLU, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    launch_k(tc_gemm_kernel<kSwiGLU, kFp8>, dim3(grid_for(a, num_sms)), dim3(kThreads), kSmemBytes, st, ta, tb0,
             tb1, a);
    return cudaGetLastError();
}

cudaError_t launch_tc_gemm1(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1,
                            const CUtensorMap& tm_w3, const TcGemmArgs& a, int num_sms,
                            cudaStream_t st) {
    return launch_tc<true, false>(tm_xp, tm_w1, tm_w3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a,
                            int num_sms, cudaStream_t st) {
    return launch_tc<false, false>(tm_h, tm_w2, tm_w2, a, num_sms, st);
}

cudaError_t launch_tc_gemm1_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1,
                                 const CUtensorMap& tm_q3, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st) {
    return launch_tc<true, true>(tm_x8, tm_q1, tm_q3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                 int num_sms, cudaStream_t st) {
    return launch_tc<false, true>(tm_h8, tm_q2, tm_q2, a, num_sms, st);
}

}  // namespace moe
