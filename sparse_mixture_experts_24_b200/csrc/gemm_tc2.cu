// gemm_tc2.cu -- the bf16 grouped expert GEMMs of gemm_tc.cu on CTA pairs
// (tcgen05 cta_group::2): two SMs of a cluster compute one 256 x 256 tile.
//
//   GEMM1: H[r] = bf16( silu(Xp[r] . w1[e]) * (Xp[r] . w3[e]) )  rows r of expert e
//   GEMM2: O[r] = bf16( H[r] . w2[e] )
//
// Source: the SwiGLU expert of the layer equation ("Mixtral of Experts"
// section 2.1 on the flash-card page), run only on the rows routed to each
// expert (Part 3, Step 2 of "Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists").
//
// Why pairs: with one SM per 128 x 256 tile every SM streams 48 KB of operands
// per 64-deep K step.  A pair MMA (M = 256, N = 256) takes 128 rows of A from
// each SM and N/2 columns of B from each SM, so each SM streams 32 KB per K
// step for the same tensor work, and a 6-stage ring fits in shared memory.
// For GEMM1 the leader's B half is 128 columns of w1 and the peer's half the
// same 128 columns of w3, so each SM's accumulator holds both projections of
// its 128 rows and the SwiGLU epilogue is unchanged.
//
// Roles (192 threads per CTA, one cluster of two CTAs per pair of SMs):
//   warp 0   (both CTAs) TMA of this CTA's A rows and B columns (bf16: one
//            copy of two 64-column chunks through a 4-D weight map) into its
//            own ring, in the banded tile order of gemm_tc.cu; completion is
//            counted on the LEADER's full barrier
//            (cp.async.bulk.tensor ... cta_group::2, no multicast); the leader
//            arms that barrier with the pair's byte count.
//   warp 1   (both CTAs) allocate 512 TMEM columns as a pair; the leader's lane
//            0 issues tcgen05.mma.cta_group::2 and commits to the empty barrier
//            of the stage in both CTAs and, per tile, to both accumulator-full
//            barriers.
//   warps 2-5 (both CTAs) epilogue of the CTA's own 128 rows; each warp then
//            arrives on the leader's accumulator-empty barrier (8 arrivals).
// Every wait is bounded; both CTAs pass a cluster barrier before exit so that
// no remote arrive can target a CTA that has already left.
//
// E4M3 variant (kFp8): a stage is 128 K-elements of one-byte codes (A: this
// CTA's 128 rows x 128 bytes; B: this CTA's 128 columns x 128 K-rows, N-major,
// one box), four tcgen05.mma.cta_group::2.kind::f8f6f4 (K = 32) per stage, and
// the epilogue of gemm_tc.cu's E4M3 kernels (accumulator x row scale x column
// scale).  At the fp8 rate the single-SM 128 x 256 tile has to stream its
// operands through shared memory twice as fast per FLOP as bf16; the pair tile
// halves the B bytes each SM streams.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPairBM = 256;                       // rows per pair tile
constexpr int kPairBN = 256;                       // pair MMA N
constexpr int kPairBK = 64;
constexpr int kPairBK8 = 128;                      // K per stage of the E4M3 pair kernels (128 bytes)
constexpr int kPairStages = 6;
constexpr int kPairABytes = 128 * kPairBK * 2;     // 16 KB: this CTA's 128 rows
constexpr int kPairBChunk = kPairBK * 64 * 2;      // 8 KB: 64 K-rows x 64 columns
constexpr int kPairBBytes = 2 * kPairBChunk;       // 16 KB: this CTA's 128 columns
constexpr int kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairTmemCols = 512;
constexpr int kPairThreads = 192;
constexpr int kPairMaxN = 256;

struct __align__(8) PairTail {
    uint64_t full[kPairStages];
    uint64_t empty[kPairStages];
    uint64_t accum_full[2];
    uint64_t accum_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t off[kPairMaxN + 1];
    int32_t mblk[kPairMaxN + 1];
};

constexpr int kPairTailBytes = (static_cast<int>(sizeof(PairTail)) + 127) / 128 * 128;
constexpr int kPairSmemBytes = kPairStages * kPairStageBytes + kPairTailBytes + 4 * kWarpStageBytes + 1024;

struct PairTile {
    int e, n_tile, row0, rows;
};

// Tile order: tile t -> (expert, column tile, 256-row block), an expert's row
// blocks cut into bands of `band` blocks with the row block fastest inside a
// band (the order of gemm_tc.cu's tile_info), so that a band's A rows stay in
// L2 while the expert's weight columns stream past them once per band.
__device__ __forceinline__ PairTile pair_tile(int t, const int32_t* off, const int32_t* mblk, int n,
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
    PairTile p;
    p.e = e;
    p.n_tile = n_tile;
    p.row0 = off[e] + m_blk * kPairBM;
    p.rows = min(kPairBM, off[e + 1] - p.row0);
    return p;
}

__device__ __forceinline__ float silu_pair(float a) { return a / (1.f + __expf(-a)); }

template <bool kSwiGLU, bool kFp8>
__global__ void __launch_bounds__(kPairThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                        const __grid_constant__ CUtensorMap tm_b1, const TcGemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    PairTail* tail = reinterpret_cast<PairTail*>(smem + kPairStages * kPairStageBytes);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n = args.n;
    const uint32_t rank = cluster_ctarank();
    const int cid = static_cast<int>(cluster_id_x());
    const int ncl = static_cast<int>(nclusters_x());

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(smem_u32(&tail->full[s]), 1);
            mbar_init(smem_u32(&tail->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tail->accum_full[b]), 1);
            mbar_init(smem_u32(&tail->accum_empty[b]), 8);
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
        tmem_alloc_pair(smem_u32(&tail->tmem_base), kPairTmemCols);
        tmem_relinquish_pair();
    }
    griddep_wait();  // segment offsets and the A operand come from earlier kernels
    for (int i = threadIdx.x; i <= n; i += kPairThreads) {
        tail->off[i] = args.offsets[i];
        tail->mblk[i] = args.mblk_base[i];
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barrier inits of both CTAs visible before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = tail->tmem_base;
    const int total_tiles = tail->mblk[n] * args.n_tiles;
    int* status = args.status;
    // args.band_m counts 128-row blocks; a pair tile's row block is 256 rows
    const int band_limit = args.band_m > 0 ? max(1, args.band_m / 2) : 0x40000000;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            int stage = 0;
            uint32_t phase = 0;
            int armed[kPairStages];
            for (int s = 0; s < kPairStages; ++s) armed[s] = -1;
            bool ok = true;
            for (int t = cid; t < total_tiles && ok; t += ncl) {
                const PairTile pt = pair_tile(t, tail->off, tail->mblk, n, args.n_tiles, band_limit);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->empty[stage]), phase ^ 1u, status, kStatusTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_local = smem_u32(&tail->full[stage]);
                    if (rank == 0) {
                        mbar_arrive_expect_tx(full_local, 2 * kPairStageBytes);
                        armed[stage] = static_cast<int>(phase);
                    }
                    const uint32_t full_leader = mapa_shared(full_local, 0);
                    const uint32_t a_dst = smem_u32(smem + stage * kPairStageBytes);
                    const uint32_t b_dst = a_dst + kPairABytes;
                    const int k0 = kb * (kFp8 ? kPairBK8 : kPairBK);
                    tma_load_2d_pair(a_dst, &tm_a, full_leader, k0, pt.row0 + 128 * static_cast<int>(rank));
                    if (kFp8) {
                        // one 128 x 128 box: 128 K-rows of this CTA's 128 columns
                        const CUtensorMap* src = (kSwiGLU && rank != 0) ? &tm_b1 : &tm_b0;
                        const int c0 = kSwiGLU ? pt.n_tile * 128 : pt.n_tile * kPairBN + 128 * static_cast<int>(rank);
                        tma_load_3d_pair(b_dst, src, full_leader, c0, k0, pt.e);
                    } else if (kSwiGLU) {
                        // bf16 weight maps are 4-D (64 columns, K rows, 64-column
                        // chunk, expert) with boxes of two chunks: this CTA's 128
                        // columns in one copy
                        const CUtensorMap* src = rank == 0 ? &tm_b0 : &tm_b1;
                        tma_load_4d_pair(b_dst, src, full_leader, 0, k0, pt.n_tile * 2, pt.e);
                    } else {
                        tma_load_4d_pair(b_dst, &tm_b0, full_leader, 0, k0, pt.n_tile * 4 + 2 * static_cast<int>(rank),
                                         pt.e);
                    }
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // The leader's full barriers count both CTAs' copies: draining them
            // covers every TMA write of the pair.
            if (rank == 0)
                for (int s = 0; s < kPairStages; ++s)
                    if (armed[s] >= 0)
                        mbar_wait(smem_u32(&tail->full[s]), static_cast<uint32_t>(armed[s]), status,
                                  kStatusTimeoutDrain);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- pair MMA issuer (leader only) ----------------
            constexpr uint32_t idesc =
                kFp8 ? make_idesc_e4m3(kPairBM, kPairBN, 0, 1) : make_idesc_bf16(kPairBM, kPairBN, 0, 1);
            int stage = 0;
            uint32_t phase = 0;
            int local = 0;
            bool ok = true;
            for (int t = cid; t < total_tiles && ok; t += ncl, ++local) {
                const int buf = local & 1;
                const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait(smem_u32(&tail->accum_empty[buf]), bph ^ 1u, status, kStatusTimeoutAccum)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kPairBN);
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!mbar_wait(smem_u32(&tail->full[stage]), phase, status, kStatusTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + stage * kPairStageBytes);
                    const uint32_t b_base = a_base + kPairABytes;
                    if (kFp8) {
#pragma unroll
                        for (int kk = 0; kk < kPairBK8 / 32; ++kk) {
                            // A: K-major, K by 32 one-byte codes = 32 bytes inside the swizzle
                            // row; B: N-major, one 128-column chunk, K by 32 = four 8-row groups
                            const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
                            const uint64_t bdesc = make_smem_desc(b_base + kk * 4096, kPairBBytes, 1024, 2);
                            tc_mma_f8_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kPairBK / 16; ++kk) {
                            const uint64_t adesc = make_smem_desc(a_base + kk * 32, 16, 1024, 2);
                            const uint64_t bdesc = make_smem_desc(b_base + kk * 2048, kPairBChunk, 1024, 2);
                            tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                        }
                    }
                    const uint32_t eb = smem_u32(&tail->empty[stage]);
                    tc_commit_pair(mapa_shared(eb, 0));
                    tc_commit_pair(mapa_shared(eb, 1));
                    if (++stage == kPairStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) {
                    const uint32_t fb = smem_u32(&tail->accum_full[buf]);
                    tc_commit_pair(mapa_shared(fb, 0));
                    tc_commit_pair(mapa_shared(fb, 1));
                }
            }
            tc_commit_pair(mapa_shared(smem_u32(&tail->done), 0));
            mbar_wait(smem_u32(&tail->done), 0, status, kStatusTimeoutDrain);
        }
    } else {
        // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
        const int quad = warp & 3;
        uint8_t* stage = smem + kPairStages * kPairStageBytes + kPairTailBytes + (warp - 2) * kWarpStageBytes;
        const uint32_t accum_empty_leader0 = mapa_shared(smem_u32(&tail->accum_empty[0]), 0);
        const uint32_t accum_empty_leader1 = mapa_shared(smem_u32(&tail->accum_empty[1]), 0);
        int local = 0;
        for (int t = cid; t < total_tiles; t += ncl, ++local) {
            const PairTile pt = pair_tile(t, tail->off, tail->mblk, n, args.n_tiles, band_limit);
            const int buf = local & 1;
            const uint32_t bph = static_cast<uint32_t>(local >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tail->accum_full[buf]), bph, status, kStatusTimeoutAccum)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(buf * kPairBN);
            // this warp's 32 rows of this CTA's half of the pair tile
            const int my_rows = pt.rows - 128 * static_cast<int>(rank);
            const int valid = min(32, my_rows - quad * 32);
            const int64_t row_base = static_cast<int64_t>(pt.row0) + 128 * static_cast<int>(rank) + quad * 32;
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
                    const int col = pt.n_tile * 128 + c * 32;
                    if (row_ok && col < args.out_cols) {
                        if (kFp8) {
                            // dequantise: accumulator x row scale x column scale
                            const float4* s0 = reinterpret_cast<const float4*>(
                                args.col_scale0 + static_cast<int64_t>(pt.e) * args.out_cols + col);
                            const float4* s1 = reinterpret_cast<const float4*>(
                                args.col_scale1 + static_cast<int64_t>(pt.e) * args.out_cols + col);
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
                            const float h0 = silu_pair(__uint_as_float(a[2 * j])) * __uint_as_float(b[2 * j]);
                            const float h1 =
                                silu_pair(__uint_as_float(a[2 * j + 1])) * __uint_as_float(b[2 * j + 1]);
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
                    const int col = pt.n_tile * kPairBN + g * 64;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t a[32];
                        tmem_ld_32x32b_x32(tbase + g * 64 + c * 32, a);
                        tmem_wait_ld();
                        if (kFp8 && col < args.out_cols) {
                            const float4* s0 = reinterpret_cast<const float4*>(
                                args.col_scale0 + static_cast<int64_t>(pt.e) * args.out_cols + col + c * 32);
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
            if (lane == 0) mbar_arrive_cluster(buf == 0 ? accum_empty_leader0 : accum_empty_leader1);
        }
    }

    tc_fence_before();
    __syncwarp();
    __syncthreads();
    cluster_sync();  // no remote arrive or commit may target a CTA that has left
    griddep_launch_dependents();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kPairTmemCols);
    }
}

template <bool kSwiGLU, bool kFp8>
static cudaError_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
                               const TcGemmArgs& a, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_pair_kernel<kSwiGLU, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t max_tiles = ((a.R + kPairBM - 1) / kPairBM + a.n) * static_cast<int64_t>(a.n_tiles);
    int64_t clusters = num_sms / 2;
    if (max_tiles < clusters) clusters = max_tiles;
    if (clusters < 1) clusters = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    cfg.blockDim = dim3(kPairThreads);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (g_chain_started && pdl_enabled()) ? 2 : 1;
    g_chain_started = true;
    return cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<kSwiGLU, kFp8>, ta, tb0, tb1, a);
}

cudaError_t launch_tc_gemm1_pair(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1,
                                 const CUtensorMap& tm_w3, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st) {
    return launch_pair<true, false>(tm_xp, tm_w1, tm_w3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2_pair(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a,
                                 int num_sms, cudaStream_t st) {
    return launch_pair<false, false>(tm_h, tm_w2, tm_w2, a, num_sms, st);
}

cudaError_t launch_tc_gemm1_pair_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1,
                                      const CUtensorMap& tm_q3, const TcGemmArgs& a, int num_sms,
                                      cudaStream_t st) {
    return launch_pair<true, true>(tm_x8, tm_q1, tm_q3, a, num_sms, st);
}

cudaError_t launch_tc_gemm2_pair_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                      int num_sms, cudaStream_t st) {
    return launch_pair<false, true>(tm_h8, tm_q2, tm_q2, a, num_sms, st);
}

}  // namespace moe
