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
//            swizzle; B: 64 x 256 of the weights, N-major, four 64-column
//            chunks, 128-byte swizzle).  The bf16 weight maps are 4-D (64
//            columns, K rows, 64-column chunk, expert) so that one copy brings
//            several chunks: a stage is 2 copies (GEMM2) or 3 (GEMM1) instead
//            of 5 (fewer copies for the one producer thread to issue).  GEMM1's
//            B is 128 columns of w1 next to the same 128 columns of w3, so ONE
//            N=256 MMA produces both the gate and the up projection of a
//            128-column slice of H.
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
constexpr int kGatherThreads = 320;  // + 4 warps gathering A rows from x (GEMM1, bf16)
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

// Tile order.  Tile t -> (expert, column tile, row block).  An expert's row
// blocks are cut into bands of `band` blocks (the last may be shorter); within
// a band the row block runs fastest, then the column tile, so a band's A rows
// stay in L2 while every weight column tile of the expert streams past them
// once per band.  An expert of at most `band` blocks is one band: its A rows
// stay in L2 for all its column tiles.  Bands matter when one expert takes
// far more rows than L2 holds (a skewed router's favourite): unbanded, every
// round of persistent tiles would stream all of that expert's A rows again
// (measured on the skewed prefill: 11.9 GB of DRAM reads in GEMM1 against
// 2.9 GB with bands of 32 MB of A rows).
__device__ __forceinline__ TileInfo tile_info(int t, const int32_t* off, const int32_t* mblk, int n,
                                              int n_tiles, int band_limit) {
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
    const int band = min(mb_count, band_limit);
    const int full = mb_count / band * band;  // row blocks in whole bands
    int n_tile, m_blk;
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
    TileInfo ti;
    ti.e = e;
    ti.n_tile = n_tile;
    ti.row0 = off[e] + m_blk * kBM;
    ti.rows = min(kBM, off[e + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.f + __expf(-a)); }

// kSwiGLU: GEMM1 (two B maps, 128 output columns per tile); else GEMM2.
// kFp8: E4M3 operands with the scales of TcGemmArgs applied in the epilogue.
// 16-byte copy global -> shared (zero-filled when src_bytes is 0), in the
// thread's current cp.async group.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}
// Arrive on the mbarrier once every cp.async this thread has issued so far has
// landed; .noinc: the arrival counts toward the barrier's expected count.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// kGather (GEMM1, bf16 only): A is not read from Xp by TMA; warps 6-9 gather
// the tile's rows straight from x (row r of the tile = token row_token[row0 +
// r]) with 16-byte cp.async copies into the same 128-byte-swizzled layout,
// so the gather kernel and the Xp round trip through HBM are gone.  Each
// gather thread owns one 16-byte column chunk of 8 rows; after issuing a
// stage's copies it makes their completion arrive on the stage's full barrier
// (cp.async.mbarrier.arrive.noinc: 128 such arrivals plus the TMA producer's),
// so the gather warps never wait for their own copies and run as far ahead as
// the ring allows; the MMA thread fences the async proxy after each full wait.
template <bool kSwiGLU, bool kFp8, bool kGather>
__global__ void __launch_bounds__(kGather ? kGatherThreads : kThreads, 1)
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
            mbar_init(smem_u32(&tail->full[s]), kGather ? 129 : 1);  // TMA (+ the 128 gather threads)
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
    for (int i = threadIdx.x; i <= n; i += static_cast<int>(blockDim.x)) {
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
    const int band_limit = args.band_m > 0 ? args.band_m : 0x40000000;
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
                const TileInfo ti = tile_info(t, tail->off, tail->mblk, n, args.n_tiles, band_limit);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status,
                                   kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&tail->full[stage]);
                    mbar_arrive_expect_tx(fb, kGather ? kBBytes : kStageBytes);
                    armed[stage] = static_cast<int>(phase);
                    const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b_dst = a_dst + kABytes;
                    const int k0 = kb * (kFp8 ? kBK8 : kBK);
                    if (!kGather) tma_load_2d(a_dst, &tm_a, fb, k0, ti.row0);
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
                        // the weight maps are 4-D (64 columns, K rows, 64-column chunk,
                        // expert): one copy brings two whole 64-column chunks
                        tma_load_4d(b_dst, &tm_b0, fb, 0, k0, ti.n_tile * 2, ti.e);
                        tma_load_4d(b_dst + 2 * kBChunkBytes, &tm_b1, fb, 0, k0, ti.n_tile * 2, ti.e);
                    } else {
                        tma_load_4d(b_dst, &tm_b0, fb, 0, k0, ti.n_tile * 4, ti.e);  // four chunks
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
                    if (kGather) fence_proxy_async_smem();  // the gathered rows came by cp.async
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
    } else if (kGather && warp >= 6) {
        // ---------------- A gather (warps 6..9) ----------------
        const int gt = static_cast<int>(threadIdx.x) - kThreads;  // 0..127
        const int c = gt & 7;                                      // 16-byte chunk of a 128-byte row slice
        const int r0 = gt >> 3;                                    // rows r0, r0 + 16, ..., r0 + 112
        const uint16_t* x = args.x;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = first; t < total_tiles && ok; t += stride) {
            const TileInfo ti = tile_info(t, tail->off, tail->mblk, n, args.n_tiles, band_limit);
            const uint16_t* src[8];
            uint32_t bytes[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = r0 + 16 * i;
                const int tok = r < ti.rows ? __ldg(args.row_token + ti.row0 + r) : -1;
                const bool valid = tok >= 0 && tok < args.x_rows;
                src[i] = x + (valid ? static_cast<int64_t>(tok) * args.x_cols : 0) + c * 8;
                bytes[i] = valid ? 16u : 0u;
            }
            for (int kb = 0; kb < args.k_blocks; ++kb) {
                uint32_t okw = 1;
                if (lane == 0)
                    okw = mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty) ? 1u : 0u;
                okw = __shfl_sync(0xffffffffu, okw, 0);
                if (!okw) {
                    ok = false;
                    break;
                }
                const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = r0 + 16 * i;
                    cp_async_16(a_dst + r * 128 + ((c ^ (r & 7)) << 4), src[i] + kb * kBK, bytes[i]);
                }
                cp_async_mbar_arrive_noinc(smem_u32(&tail->full[stage]));
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        cp_async_wait<0>();  // no copy of this thread may still be landing when the CTA exits
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
        uint8_t* stage = smem + kStages * kStageBytes + kTailBytes + (warp - 2) * kWarpStageBytes;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const TileInfo ti = tile_info(t, tail->off, tail->mblk, n, args.n_tiles, band_limit);
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

template <bool kSwiGLU, bool kFp8, bool kGather = false>
static cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                             const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<kSwiGLU, kFp8, kGather>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    launch_k(tc_gemm_kernel<kSwiGLU, kFp8, kGather>, dim3(grid_for(a, num_sms)),
             dim3(kGather ? kGatherThreads : kThreads), kSmemBytes, st, ta, tb0, tb1, a);
    return cudaGetLastError();
}

cudaError_t launch_tc_gemm1_gather(const CUtensorMap& tm_w1, const CUtensorMap& tm_w3, const TcGemmArgs& a,
                                   int num_sms, cudaStream_t st) {
    return launch_tc<true, false, true>(tm_w1, tm_w1, tm_w3, a, num_sms, st);
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
