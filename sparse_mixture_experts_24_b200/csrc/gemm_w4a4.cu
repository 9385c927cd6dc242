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
// One persistent CTA per SM, 384 threads, tiles of kTM rows x kBN columns of
// the packed B (kBN = 128: two accumulators, 6 stages of 36 KB, or 8 of 24 KB
// with 32-row tiles; kBN = 256: one accumulator, 4 stages of 54 KB, or 5 of 42
// KB with 32-row tiles -- the block scales take the rest of TMEM):
//   warp 0     TMA producer: per stage a K step of 256 (128 bytes of codes per
//              row): A 128 rows (128-byte swizzle), the kBN K-major weight rows
//              in one copy (GEMM1: the w1|w3 pair pack, 64 hidden columns per
//              128-row block; GEMM2: w2), and by plain bulk copies the matching
//              512-byte scale chunks (4 for A, 4 per 128-row B block).
//   warps 10-11 per stage (warp 10 the even stages, 11 the odd ones), copy
//              the scale chunks into that stage's TMEM columns (tcgen05.cp
//              32x128b.warpx4, 3 or 2 per 64-wide K step) and commit them to
//              the stage's scales-ready barrier.
//   warp 1     allocates 512 TMEM columns; once a stage's scales are in TMEM
//              it issues tcgen05.mma kind::mxf4nvf4 block16 M=128 N=kBN.
//              With the scale copies on warps of their own, the MMA thread
//              issues only the stage's 4 MMAs.
//   warps 2-9  epilogue, two warps per TMEM lane quadrant splitting the
//              columns: accumulator x row scale x matrix scale, SwiGLU (GEMM1)
//              or a copy (GEMM2), bf16 rows.
// Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace w4gemm {

constexpr int kBM = kTcBM;   // 128: MMA M
constexpr int kBBlockBytes = 128 * 128; // 16 KB: one 128-row block of B
constexpr int kSfaBytes = 4 * 512;      // 4 chunks (64-wide K steps) of A scales
constexpr int kSfbBlockBytes = 4 * 512; // the same for one 128-row block of B
constexpr int kMaxN = 256;
constexpr int kMaxStages = 8;
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 8;  // two per TMEM lane quadrant, each taking half the columns
constexpr int kCpWarp = 2 + kEpiWarps;  // the scale-factor copies: warps kCpWarp, kCpWarp + 1
constexpr int kCpWarps = 2;             // each owns the stages s with s % 2 == its index
constexpr int kThreads = (2 + kEpiWarps + kCpWarps) * 32;

// Tile width kBN (128 or 256 output columns of the packed B, i.e. 64 or 128
// hidden columns of GEMM1's w1|w3 pairs) and tile height kTM (rows of A per
// tile: 128, or 32 for batches of a few rows per expert): B blocks per stage,
// stages, and TMEM: accumulators from column 0 (two of 128 columns, or one of
// 256), the scale factors of every stage after them.  The MMA is always
// M = 128; with kTM = 32 the A rows past 32 are whatever follows in shared
// memory (finite codes), and their accumulator rows are never stored.
template <int kBN, int kTM>
struct Cfg {
    static constexpr int kBlocks = kBN / 128;
    static constexpr int kABytes = kTM * 128;  // kTM rows of 128 bytes (a K step of 256)
    static constexpr int kStageBytes = kABytes + kBlocks * kBBlockBytes + kSfaBytes + kBlocks * kSfbBlockBytes;
    static constexpr int kStages = kBN == 128 ? (kTM == 32 ? 8 : 6) : (kTM == 32 ? 5 : 4);
    static constexpr int kAccBufs = kBN == 128 ? 2 : 1;
    static constexpr int kSfCols = 4 * (4 + 4 * kBlocks);  // per stage: 4 K steps x (A + B chunks)
    static constexpr int kSfBase = kAccBufs * kBN;
    static_assert(kStageBytes % 1024 == 0, "stages keep the 1 KB alignment of the swizzled tiles");
    static_assert(kSfBase + kStages * kSfCols <= kTmemCols, "TMEM budget");
    static_assert(kStages <= kMaxStages, "barrier arrays");
};

struct __align__(8) SmemTail {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t sf_ready[kMaxStages];  // the stage's scale chunks are in TMEM
    uint64_t cp_done[kCpWarps];
    uint64_t accum_full[2];
    uint64_t accum_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kMaxN + 1];
    int32_t mblk[kMaxN + 1];
};

constexpr int kTailBytes = (static_cast<int>(sizeof(SmemTail)) + 127) / 128 * 128;

template <int kBN, int kTM>
constexpr int smem_bytes() {
    return Cfg<kBN, kTM>::kStages * Cfg<kBN, kTM>::kStageBytes + kTailBytes + 1024;
}

struct Tile {
    int e, n_tile, m_blk, row0, rows;
};

template <int kTM>
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
    ti.row0 = off[lo] + ti.m_blk * kTM;
    ti.rows = min(kTM, off[lo + 1] - ti.row0);
    return ti;
}

__device__ __forceinline__ float silu(float a) { return __fdividef(a, 1.f + __expf(-a)); }

}  // namespace w4gemm

using namespace w4gemm;

// kSwiGLU: GEMM1 over the w1|w3 pair pack (accumulator column j of block
// j / 128 is w1 for j % 128 < 64, w3 otherwise; hidden column = 64 x block +
// j % 64); else GEMM2 over w2.
template <bool kSwiGLU, int kBN, int kTM>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const W4a4GemmArgs args) {
    using C = Cfg<kBN, kTM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    SmemTail* tail = reinterpret_cast<SmemTail*>(smem + C::kStages * C::kStageBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
            mbar_init(smem_u32(&tail->sf_ready[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tail->accum_full[b]), 1);
            mbar_init(smem_u32(&tail->accum_empty[b]), kEpiWarps);
        }
        mbar_init(smem_u32(&tail->done), 1);
        for (int c = 0; c < kCpWarps; ++c) mbar_init(smem_u32(&tail->cp_done[c]), 1);
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
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
    const int stride = args.balanced ? balanced_ctas(total_tiles, static_cast<int>(gridDim.x))
                                     : static_cast<int>(gridDim.x);
    const int first = static_cast<int>(blockIdx.x) < stride ? static_cast<int>(blockIdx.x) : total_tiles;
    const int kb64_total = args.k_steps * 4;  // 64-wide K steps of the whole reduction
    int* status = args.status;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0;
            int armed[kMaxStages];
            for (int s = 0; s < kMaxStages; ++s) armed[s] = -1;
            bool ok = true;
            const int blocks_per_e = args.n_rows_b / 128;
            for (int t = first; t < total_tiles && ok; t += stride) {
                const Tile ti = tile_at<kTM>(t, tail->off, tail->mblk, n, args.n_tiles);
                const int r0 = ti.n_tile * kBN;  // first packed B row of the tile
                const uint8_t* sfb = args.b_chunks +
                                     (static_cast<int64_t>(ti.e) * blocks_per_e + r0 / 128) * kb64_total * 512;
                const uint8_t* sfa =
                    args.a_chunks + (static_cast<int64_t>(tail->mblk[ti.e]) + ti.m_blk) * kb64_total * 512;
                for (int ks = 0; ks < args.k_steps; ++ks) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&tail->full[stage]);
                    mbar_arrive_expect_tx(fb, C::kStageBytes);
                    armed[stage] = static_cast<int>(phase);
                    const uint32_t base = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t sf_smem = base + C::kABytes + C::kBlocks * kBBlockBytes;
                    const int kx = ks * 128;  // byte column of the codes
                    const int64_t ck = static_cast<int64_t>(ks) * 4 * 512;
                    tma_load_2d(base, &tm_a, fb, kx, ti.row0);
                    bulk_load(sf_smem, sfa + ck, kSfaBytes, fb);
                    // the map's box is kBN rows: the tile's B blocks in one copy
                    tma_load_3d(base + C::kABytes, &tm_b, fb, kx, r0, ti.e);
#pragma unroll
                    for (int b = 0; b < C::kBlocks; ++b)
                        bulk_load(sf_smem + kSfaBytes + b * kSfbBlockBytes,
                                  sfb + static_cast<int64_t>(b) * kb64_total * 512 + ck, kSfbBlockBytes, fb);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < C::kStages; ++s)
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
            for (int t = first; t < total_tiles && ok; t += stride, ++local) {
                const int buf = C::kAccBufs == 2 ? (local & 1) : 0;
                const uint32_t use = C::kAccBufs == 2 ? static_cast<uint32_t>(local >> 1) : static_cast<uint32_t>(local);
                if (!mbar_wait(smem_u32(&tail->accum_empty[buf]), (use & 1u) ^ 1u, status, kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
                for (int ks = 0; ks < args.k_steps; ++ks) {
                    // the scale copies of this stage are complete (so are its TMA copies)
                    if (!mbar_wait(smem_u32(&tail->sf_ready[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t base = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(C::kSfBase + stage * C::kSfCols);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t sfa_t = sf_col + 4 * kk;
                        const uint32_t sfb_t = sf_col + 16 + 4 * C::kBlocks * kk;
                        const uint64_t adesc = make_smem_desc(base + kk * 32, 16, 1024, 2);
                        const uint64_t bdesc = make_smem_desc(base + C::kABytes + kk * 32, 16, 1024, 2);
                        tc_mma_fp4_block16(d_tmem, adesc, bdesc, idesc, sfa_t, sfb_t, (ks | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(smem_u32(&tail->empty[stage]));
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc_commit(smem_u32(&tail->accum_full[buf]));
            }
            tc_commit(smem_u32(&tail->done));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else if (warp >= kCpWarp) {
        if (lane == 0) {
            // ---------------- scale chunks -> TMEM ----------------
            // Two warps, each owning the stages s with s % 2 == its index (one
            // thread issuing every copy was busy 70% of the time at decode and
            // 91% at prefill, and a stage is released only after its copies
            // and MMAs).  A stage keeps its owner for every use, so each full
            // barrier is waited on by one thread, phase after phase: a waiter
            // that reached a later phase of a barrier still in its earlier one
            // would see the earlier parity as complete.  A stage's TMEM scale
            // columns are written again only after its next full barrier,
            // which follows the empty barrier that the MMAs reading them
            // committed to.
            const int cw = warp - kCpWarp;
            int stage = 0;
            uint32_t phase = 0;
            for (int t = first; t < total_tiles; t += stride) {
                bool ok = true;
                for (int ks = 0; ks < args.k_steps; ++ks) {
                    if (stage % kCpWarps != cw) {
                        if (++stage == C::kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                        continue;
                    }
                    if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t base = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t sfa_smem = base + C::kABytes + C::kBlocks * kBBlockBytes;
                    const uint32_t sfb_smem = sfa_smem + kSfaBytes;
                    const uint32_t sf_col = tmem_base + static_cast<uint32_t>(C::kSfBase + stage * C::kSfCols);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        tc_cp_32x128b_warpx4(sf_col + 4 * kk, make_smem_desc(sfa_smem + kk * 512, 0, 128, 0));
#pragma unroll
                        for (int b = 0; b < C::kBlocks; ++b)
                            tc_cp_32x128b_warpx4(sf_col + 16 + 4 * C::kBlocks * kk + 4 * b,
                                                 make_smem_desc(sfb_smem + b * kSfbBlockBytes + kk * 512, 0, 128, 0));
                    }
                    tc_commit(smem_u32(&tail->sf_ready[stage]));
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // every copy of this thread is complete before TMEM is freed
            tc_commit(smem_u32(&tail->cp_done[cw]));
            mbar_wait(smem_u32(&tail->cp_done[cw]), 0, status, kStatusTimeoutDrain);
        }
    } else {
        // ---------------- epilogue (warps 2..9) ----------------
        // warp w reads TMEM lanes 32 (w % 4) .. +31 and the column half (w - 2) / 4
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const Tile ti = tile_at<kTM>(t, tail->off, tail->mblk, n, args.n_tiles);
            const int buf = C::kAccBufs == 2 ? (local & 1) : 0;
            const uint32_t use = C::kAccBufs == 2 ? static_cast<uint32_t>(local >> 1) : static_cast<uint32_t>(local);
            const int valid = min(32, ti.rows - quad * 32);
            const bool row_ok = lane < valid;
            const int64_t row_base = static_cast<int64_t>(ti.row0) + quad * 32;
            // scales first: their loads overlap the wait for the accumulator
            const float rs = row_ok ? args.row_scale[row_base + lane] : 0.f;
            const float m0 = __ldg(args.mscale0 + ti.e);
            const float m1 = kSwiGLU ? __ldg(args.mscale1 + ti.e) : 0.f;
            if (!mbar_wait(smem_u32(&tail->accum_full[buf]), use & 1u, status, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kBN);
            uint16_t* out = static_cast<uint16_t*>(args.out);
            const float g0 = m0 * rs;
            // This warp's accumulator columns go to registers first and the
            // accumulator is handed back to the MMA warp before any math or
            // store: with one accumulator the next tile's MMAs wait only for
            // these TMEM reads.
            constexpr int kRegChunks = kBN / 64;  // 32-column chunks per warp
            uint32_t acc[kRegChunks][32];
            // warp-uniform: a quadrant past the tile's rows only hands back
            const bool any_row = valid > 0;
#pragma unroll
            for (int i = 0; i < kRegChunks; ++i) {
                if (!any_row) break;
                int col;
                if (kSwiGLU) {
                    // chunk pair q (q = half * kRegChunks / 2 + i / 2): w1 columns
                    // 128 (q / 2) + 32 (q % 2) + 0..31, the w3 ones 64 later
                    const int q = half * (kRegChunks / 2) + (i >> 1);
                    col = 128 * (q >> 1) + 32 * (q & 1) + ((i & 1) ? 64 : 0);
                } else {
                    col = (half * kRegChunks + i) * 32;
                }
                tmem_ld_32x32b_x32(tbase + col, acc[i]);
            }
            if (any_row) tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tail->accum_empty[buf]));
            if (kSwiGLU) {
                const float g1 = m1 * rs;
#pragma unroll
                for (int i = 0; i < kRegChunks / 2; ++i) {
                    const int q = half * (kRegChunks / 2) + i;
                    const int col = ti.n_tile * (kBN / 2) + 32 * q;
                    const uint32_t* a = acc[2 * i];
                    const uint32_t* b = acc[2 * i + 1];
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
                        for (int p = 0; p < 4; ++p)
                            dst[p] = make_uint4(pk[4 * p], pk[4 * p + 1], pk[4 * p + 2], pk[4 * p + 3]);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < kRegChunks; ++i) {
                    const int col = ti.n_tile * kBN + (half * kRegChunks + i) * 32;
                    const uint32_t* a = acc[i];
                    if (row_ok && col < args.out_cols) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            pk[j] = pack_bf16x2(__uint_as_float(a[2 * j]) * g0, __uint_as_float(a[2 * j + 1]) * g0);
                        uint4* dst = reinterpret_cast<uint4*>(out + (row_base + lane) * args.out_cols + col);
#pragma unroll
                        for (int p = 0; p < 4; ++p)
                            dst[p] = make_uint4(pk[4 * p], pk[4 * p + 1], pk[4 * p + 2], pk[4 * p + 3]);
                    }
                }
            }
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

int w4a4_tile_cols(bool wide) { return wide ? 256 : 128; }

template <bool kSwiGLU, int kBN, int kTM>
static cudaError_t launch_w4(const CUtensorMap& ta, const CUtensorMap& tb, const W4a4GemmArgs& a, int num_sms,
                             cudaStream_t st) {
    constexpr int smem = smem_bytes<kBN, kTM>();
    cudaError_t e = cudaFuncSetAttribute(w4a4_gemm_kernel<kSwiGLU, kBN, kTM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + kTM - 1) / kTM + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    if (g < 1) g = 1;
    launch_k(w4a4_gemm_kernel<kSwiGLU, kBN, kTM>, dim3(static_cast<unsigned>(g)), dim3(kThreads), smem, st, ta, tb,
             a);
    return cudaGetLastError();
}

template <bool kSwiGLU>
static cudaError_t launch_w4_any(const CUtensorMap& ta, const CUtensorMap& tb, const W4a4GemmArgs& a, bool wide,
                                 int tile_rows, int num_sms, cudaStream_t st) {
    if (!wide) {
        if (tile_rows == 32) return launch_w4<kSwiGLU, 128, 32>(ta, tb, a, num_sms, st);
        if (tile_rows == 128) return launch_w4<kSwiGLU, 128, 128>(ta, tb, a, num_sms, st);
        return cudaErrorInvalidValue;
    }
    if (tile_rows == 32) return launch_w4<kSwiGLU, 256, 32>(ta, tb, a, num_sms, st);
    if (tile_rows == 128) return launch_w4<kSwiGLU, 256, 128>(ta, tb, a, num_sms, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_w4a4_gemm1(const CUtensorMap& tm_xq, const CUtensorMap& tm_w13, const W4a4GemmArgs& a, bool wide,
                              int tile_rows, int num_sms, cudaStream_t st) {
    return launch_w4_any<true>(tm_xq, tm_w13, a, wide, tile_rows, num_sms, st);
}

cudaError_t launch_w4a4_gemm2(const CUtensorMap& tm_hq, const CUtensorMap& tm_w2, const W4a4GemmArgs& a, bool wide,
                              int tile_rows, int num_sms, cudaStream_t st) {
    return launch_w4_any<false>(tm_hq, tm_w2, a, wide, tile_rows, num_sms, st);
}

}  // namespace moe
