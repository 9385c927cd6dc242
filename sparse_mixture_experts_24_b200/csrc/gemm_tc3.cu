// gemm_tc3.cu -- the bf16 grouped expert GEMMs of gemm_tc.cu with two row
// blocks per tile: one SM computes a 256 x 256 tile as two 128 x 256 MMAs
// that share the stage's B operand.
//
//   GEMM1: H[r] = bf16( silu(Xp[r] . w1[e]) * (Xp[r] . w3[e]) )  rows r of expert e
//   GEMM2: O[r] = bf16( H[r] . w2[e] )
//
// Source: the SwiGLU expert of the layer equation ("Mixtral of Experts"
// section 2.1 on the flash-card page), run only on the rows routed to each
// expert (Part 3, Step 2 of "Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists").
//
// Why.  Timed inside gemm_tc.cu's kernel, the MMA thread waits for its stage's
// data about a fifth of the time while the producer waits for a free stage a
// third to a half of the time: the four 48 KB stages are all in flight and the
// copies take about four stage-times to land, so the tensor pipe's busy share
// follows the ring's bytes in flight (a 3-stage ring measured 62% busy, the
// 4-stage one 82%).  A stage of two row blocks and one weight tile carries 64
// KB for 1,024 tensor cycles instead of 48 KB for 512: three such stages (192
// KB) cover 3,072 tensor cycles of copy latency instead of 2,048.  The price:
// the two 256-column accumulators fill the 512 TMEM columns, so the next
// tile's MMAs wait while the epilogue reads the accumulators out.
//
// Roles (one persistent CTA per SM; 320 threads for GEMM1, 192 for GEMM2):
//   warp 0   TMA producer: per 64-deep K step, A rows of both row blocks (the
//            second skipped when the segment ends inside the first) and the
//            256 weight columns (4-D maps: GEMM1 two chunks of w1 and two of
//            w3, GEMM2 four chunks of w2).
//   warp 1   allocates 512 TMEM columns; one thread issues, per 16-deep K
//            slice, tcgen05.mma M=128 N=256 for row block 0 into columns
//            0-255 and for row block 1 into columns 256-511, both reading the
//            same B descriptor.
//   warps 2.. epilogue, thread = accumulator row, as gemm_tc.cu: GEMM1's
//            SwiGLU with direct 16-byte stores, warps 2-5 on row block 0 and 6-9
//            on row block 1; GEMM2's copy through per-warp staging blocks, warps
//            2-5 on both blocks in turn; then they hand the accumulators back.
// Tiles are (expert, column tile, pair of row blocks) in gemm_tc.cu's banded
// order over pairs.  E4M3 form (kFp8): a stage is 128 K-elements of one-byte
// codes (A 128 x 128 bytes per row block; B two 128 x 128 boxes), four
// kind::f8f6f4 MMAs (K = 32) per block, and gemm_tc.cu's E4M3 scaling in the
// epilogue.  Every wait is bounded (common.cuh).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace dual {

constexpr int kBM = kTcBM;                         // rows per MMA (one row block)
constexpr int kBN = 256;                           // MMA N
constexpr int kBK = 64;                            // K per stage (bf16)
constexpr int kBK8 = 128;                          // K per stage of the E4M3 form (128 bytes too)
constexpr int kB8ChunkBytes = kBK8 * 128;          // 16 KB: 128 K-rows x 128 one-byte columns
constexpr int kStages = 3;
constexpr int kABytes = kBM * kBK * 2;             // 16 KB per row block
constexpr int kBChunkBytes = kBK * 64 * 2;         // 8 KB: 64 K-rows x 64 columns
constexpr int kBBytes = 4 * kBChunkBytes;          // 32 KB
constexpr int kStageBytes = 2 * kABytes + kBBytes; // 64 KB
constexpr int kTmemCols = 512;
constexpr int kMaxN = 256;
// GEMM1's SwiGLU epilogue has two warps per TMEM lane quadrant, one per row
// block (it stores straight from registers); GEMM2's four warps take the two
// blocks in turn through their shared-memory staging blocks.
template <bool kSwiGLU>
struct Epi {
    static constexpr int kWarps = kSwiGLU ? 8 : 4;
    static constexpr int kThreads = (2 + kWarps) * 32;
    static constexpr int kStagingBytes = kSwiGLU ? 0 : 4 * kWarpStageBytes;
};

struct __align__(8) Tail {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t accum_full;
    uint64_t accum_empty;
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kMaxN + 1];
    int32_t pblk[kMaxN + 1];  // per-expert prefix of row-block pairs
};

constexpr int kTailBytes = (static_cast<int>(sizeof(Tail)) + 127) / 128 * 128;
template <bool kSwiGLU>
constexpr int smem_bytes() {
    return kStages * kStageBytes + kTailBytes + Epi<kSwiGLU>::kStagingBytes + 1024;
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory");

struct Tile {
    int e, n_tile, row0, rows;  // rows: up to 256 (two row blocks)
};

// Tile t -> (expert, column tile, pair of row blocks): an expert's pairs are
// cut into bands of `band` pairs, the pair fastest inside a band, then the
// column tile (the order of gemm_tc.cu's tile_info, over pairs).
__device__ __forceinline__ Tile tile_of(int t, const int32_t* off, const int32_t* pblk, int n, int n_tiles,
                                        int band_limit) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pblk[mid] * n_tiles <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int e = lo;
    const int local = t - pblk[e] * n_tiles;
    const int pb_count = pblk[e + 1] - pblk[e];
    const int band = min(pb_count, band_limit);
    const int full = pb_count / band * band;
    int n_tile, p;
    if (local < full * n_tiles) {
        const int b = local / (band * n_tiles);
        const int r = local - b * band * n_tiles;
        n_tile = r / band;
        p = b * band + (r - n_tile * band);
    } else {
        const int rem = pb_count - full;
        const int r = local - full * n_tiles;
        n_tile = r / rem;
        p = full + (r - n_tile * rem);
    }
    Tile ti;
    ti.e = e;
    ti.n_tile = n_tile;
    ti.row0 = off[e] + p * 2 * kBM;
    ti.rows = min(2 * kBM, off[e + 1] - ti.row0);
    return ti;
}

// silu(a) = a / (1 + e^-a) with the fast division: the accumulators wait for
// this epilogue, so its cost is the MMA's (exact to a few fp32 ulps before the
// bf16 rounding of H; for a below about -88, e^-a is infinite and the quotient
// is zero, the limit of silu).
__device__ __forceinline__ float silu_d(float a) { return __fdividef(a, 1.f + __expf(-a)); }

// The epilogue of one 128-row block: this warp's 32 accumulator rows (TMEM
// lanes from tbase), `valid` of them inside the segment, rows from row_base.
// E4M3 (kFp8): the accumulators are multiplied by the row's activation scale
// and the column's weight scale first, as gemm_tc.cu's E4M3 epilogues do.
template <bool kFp8>
__device__ __forceinline__ void dequant32(uint32_t (&a)[32], float rs, const float* col_scale) {
    if (!kFp8) return;
    const float4* sc = reinterpret_cast<const float4*>(col_scale);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 u = __ldg(sc + q);
        a[4 * q + 0] = __float_as_uint(__uint_as_float(a[4 * q + 0]) * rs * u.x);
        a[4 * q + 1] = __float_as_uint(__uint_as_float(a[4 * q + 1]) * rs * u.y);
        a[4 * q + 2] = __float_as_uint(__uint_as_float(a[4 * q + 2]) * rs * u.z);
        a[4 * q + 3] = __float_as_uint(__uint_as_float(a[4 * q + 3]) * rs * u.w);
    }
}

template <bool kSwiGLU, bool kFp8>
__device__ __forceinline__ void epilogue_block(uint32_t tbase, int valid, int64_t row_base, int n_tile, int e,
                                               const TcGemmArgs& args, uint8_t* stage, int lane) {
    uint16_t* out = static_cast<uint16_t*>(args.out);
    const float rs = (kFp8 && lane < valid) ? args.row_scale[row_base + lane] : 1.f;
    if (kSwiGLU) {
        // the TMEM loads of chunk c + 1 are in flight while chunk c is computed
        const bool row_ok = lane < valid;
        uint32_t a[2][32], b[2][32];
        tmem_ld_32x32b_x32(tbase, a[0]);
        tmem_ld_32x32b_x32(tbase + 128, b[0]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (c + 1 < 4) {
                tmem_ld_32x32b_x32(tbase + (c + 1) * 32, a[(c + 1) & 1]);
                tmem_ld_32x32b_x32(tbase + 128 + (c + 1) * 32, b[(c + 1) & 1]);
            }
            const int col = n_tile * 128 + c * 32;
            if (row_ok && col < args.out_cols) {
                const int64_t sc = static_cast<int64_t>(e) * args.out_cols + col;
                dequant32<kFp8>(a[c & 1], rs, args.col_scale0 + (kFp8 ? sc : 0));
                dequant32<kFp8>(b[c & 1], rs, args.col_scale1 + (kFp8 ? sc : 0));
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float h0 = silu_d(__uint_as_float(a[c & 1][2 * j])) * __uint_as_float(b[c & 1][2 * j]);
                    const float h1 =
                        silu_d(__uint_as_float(a[c & 1][2 * j + 1])) * __uint_as_float(b[c & 1][2 * j + 1]);
                    pk[j] = pack_bf16x2(h0, h1);
                }
                uint4* dst = reinterpret_cast<uint4*>(out + (row_base + lane) * args.out_cols + col);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            if (c + 1 < 4) tmem_wait_ld();
        }
    } else {
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
            uint32_t pk[32];
            const int col = n_tile * 256 + g * 64;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t a[32];
                tmem_ld_32x32b_x32(tbase + g * 64 + c * 32, a);
                tmem_wait_ld();
                if (kFp8 && col < args.out_cols)
                    dequant32<kFp8>(a, rs, args.col_scale0 + static_cast<int64_t>(e) * args.out_cols + col + c * 32);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    pk[c * 16 + j] = pack_bf16x2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1]));
            }
            if (col < args.out_cols && valid > 0) warp_store_rows_64(stage, pk, lane, out, args.out_cols, row_base, valid, col);
        }
    }
}

}  // namespace dual

using namespace dual;

template <bool kSwiGLU, bool kFp8>
__global__ void __launch_bounds__(dual::Epi<kSwiGLU>::kThreads, 1)
    tc_gemm_dual_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                        const __grid_constant__ CUtensorMap tm_b1, const TcGemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Tail* tail = reinterpret_cast<Tail*>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
        }
        mbar_init(smem_u32(&tail->accum_full), 1);
        mbar_init(smem_u32(&tail->accum_empty), Epi<kSwiGLU>::kWarps);
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
    griddep_wait();  // segment offsets and the A operand come from earlier kernels
    for (int i = threadIdx.x; i <= n; i += Epi<kSwiGLU>::kThreads) tail->off[i] = args.offsets[i];
    if (threadIdx.x == 0) {
        // pairs of row blocks per expert, from the dispatch's 128-row block prefix
        int acc = 0;
        for (int e = 0; e < n; ++e) {
            tail->pblk[e] = acc;
            acc += (args.mblk_base[e + 1] - args.mblk_base[e] + 1) / 2;
        }
        tail->pblk[n] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->pblk[n] * args.n_tiles;
    const int stride = args.balanced ? balanced_ctas(total_tiles, static_cast<int>(gridDim.x))
                                     : static_cast<int>(gridDim.x);
    const int first = static_cast<int>(blockIdx.x) < stride ? static_cast<int>(blockIdx.x) : total_tiles;
    // args.band_m counts 128-row blocks; a tile's row unit here is a pair
    const int band_limit = args.band_m > 0 ? max(1, args.band_m / 2) : 0x40000000;
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
                const Tile ti = tile_of(t, tail->off, tail->pblk, n, args.n_tiles, band_limit);
                const bool two = ti.rows > kBM;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&tail->full[stage]);
                    mbar_arrive_expect_tx(fb, static_cast<uint32_t>((two ? 2 : 1) * kABytes + kBBytes));
                    armed[stage] = static_cast<int>(phase);
                    const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b_dst = a_dst + 2 * kABytes;
                    const int k0 = kb * (kFp8 ? kBK8 : kBK);
                    tma_load_2d(a_dst, &tm_a, fb, k0, ti.row0);
                    if (two) tma_load_2d(a_dst + kABytes, &tm_a, fb, k0, ti.row0 + kBM);
                    if (kFp8) {
                        // E4M3 weights [K][cols] per expert: 128 x 128-byte boxes
                        if (kSwiGLU) {
                            tma_load_3d(b_dst, &tm_b0, fb, ti.n_tile * 128, k0, ti.e);
                            tma_load_3d(b_dst + kB8ChunkBytes, &tm_b1, fb, ti.n_tile * 128, k0, ti.e);
                        } else {
                            tma_load_3d(b_dst, &tm_b0, fb, ti.n_tile * 256, k0, ti.e);
                            tma_load_3d(b_dst + kB8ChunkBytes, &tm_b0, fb, ti.n_tile * 256 + 128, k0, ti.e);
                        }
                    } else if (kSwiGLU) {
                        tma_load_4d(b_dst, &tm_b0, fb, 0, k0, ti.n_tile * 2, ti.e);
                        tma_load_4d(b_dst + 2 * kBChunkBytes, &tm_b1, fb, 0, k0, ti.n_tile * 2, ti.e);
                    } else {
                        tma_load_4d(b_dst, &tm_b0, fb, 0, k0, ti.n_tile * 4, ti.e);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be writing shared memory when the CTA exits
            for (int s = 0; s < kStages; ++s)
                if (armed[s] >= 0)
                    mbar_wait(smem_u32(&tail->full[s]), static_cast<uint32_t>(armed[s]), status, kStatusTimeoutDrain);
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
                const Tile ti = tile_of(t, tail->off, tail->pblk, n, args.n_tiles, band_limit);
                const bool two = ti.rows > kBM;
                // one set of accumulators: the previous tile's epilogue must have read them
                if (!mbar_wait(smem_u32(&tail->accum_empty), (static_cast<uint32_t>(local) & 1u) ^ 1u, status,
                               kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b_base = a_base + 2 * kABytes;
                    if (kFp8) {
#pragma unroll
                        for (int kk = 0; kk < kBK8 / 32; ++kk) {
                            // A: K-major, K by 32 one-byte codes = 32 bytes; B: N-major, two
                            // 128-column chunks 16 KB apart, K by 32 = four 8-row groups
                            const uint64_t bdesc = make_smem_desc(b_base + kk * 4096, kB8ChunkBytes, 1024, 2);
                            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                            tc_mma_f8(tmem_base, make_smem_desc(a_base + kk * 32, 16, 1024, 2), bdesc, idesc, acc);
                            if (two)
                                tc_mma_f8(tmem_base + static_cast<uint32_t>(kBN),
                                          make_smem_desc(a_base + kABytes + kk * 32, 16, 1024, 2), bdesc, idesc, acc);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kBK / 16; ++kk) {
                            // A: K-major, 128-byte swizzle, K by 16 = 32 bytes; B: N-major,
                            // K by 16 = two 8-row groups (2 KB), 8 KB between chunks
                            const uint64_t bdesc = make_smem_desc(b_base + kk * 2048, kBChunkBytes, 1024, 2);
                            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                            tc_mma_f16(tmem_base, make_smem_desc(a_base + kk * 32, 16, 1024, 2), bdesc, idesc, acc);
                            if (two)
                                tc_mma_f16(tmem_base + static_cast<uint32_t>(kBN),
                                           make_smem_desc(a_base + kABytes + kk * 32, 16, 1024, 2), bdesc, idesc, acc);
                        }
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
        // ---------------- epilogue (warps 2..) ----------------
        const int quad = warp & 3;  // TMEM lanes [32*quad, 32*quad+32)
        uint8_t* stage = kSwiGLU ? nullptr : smem + kStages * kStageBytes + kTailBytes + (warp - 2) * kWarpStageBytes;
        // GEMM1: warps 2-5 take row block 0, warps 6-9 row block 1; GEMM2: both in turn
        const int blk_first = kSwiGLU ? (warp - 2) >> 2 : 0;
        const int blk_last = kSwiGLU ? blk_first : 1;
        int local = 0;
        for (int t = first; t < total_tiles; t += stride, ++local) {
            const Tile ti = tile_of(t, tail->off, tail->pblk, n, args.n_tiles, band_limit);
            if (!mbar_wait(smem_u32(&tail->accum_full), static_cast<uint32_t>(local) & 1u, status, kStatusTimeoutAccum))
                break;
            tc_fence_after();
            for (int blk = blk_first; blk <= blk_last; ++blk) {
                const int rows_b = ti.rows - blk * kBM;
                if (rows_b <= 0) break;  // the pair's second block is past the segment
                const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                       static_cast<uint32_t>(blk * kBN);
                const int valid = min(32, rows_b - quad * 32);
                const int64_t row_base = static_cast<int64_t>(ti.row0) + blk * kBM + quad * 32;
                epilogue_block<kSwiGLU, kFp8>(tbase, valid, row_base, ti.n_tile, ti.e, args, stage, lane);
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

template <bool kSwiGLU, bool kFp8>
static cudaError_t launch_dual(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                               const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    constexpr int kSmem = smem_bytes<kSwiGLU>();
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_dual_kernel<kSwiGLU, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + 2 * kBM - 1) / (2 * kBM) + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t g = num_sms;
    if (max_tiles < g) g = max_tiles;
    if (g < 1) g = 1;
    launch_k(tc_gemm_dual_kernel<kSwiGLU, kFp8>, dim3(static_cast<unsigned>(g)), dim3(Epi<kSwiGLU>::kThreads), kSmem,
             st, ta, tb0, tb1, a);
    return cudaGetLastError();
}

cudaError_t launch_tc_gemm1_dual(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1, const CUtensorMap& tm_w3,
                                 const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_dual<true, false>(tm_xp, tm_w1, tm_w3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2_dual(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st) {
    return launch_dual<false, false>(tm_h, tm_w2, tm_w2, a, num_sms, st);
}

cudaError_t launch_tc_gemm1_dual_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1, const CUtensorMap& tm_q3,
                                      const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    return launch_dual<true, true>(tm_x8, tm_q1, tm_q3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2_dual_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                      int num_sms, cudaStream_t st) {
    return launch_dual<false, true>(tm_h8, tm_q2, tm_q2, a, num_sms, st);
}

}  // namespace moe
