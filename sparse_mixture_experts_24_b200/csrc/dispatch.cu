// dispatch.cu -- group the T*K (token, slot) pairs into contiguous per-expert
// segments so that each expert runs as one dense GEMM over only the tokens
// that chose it.
//
// Source: the Mixtral paper as quoted on the ainotis page ("How a
// mixture-of-experts model activates only part of its parameters"): when the
// gating vector is sparse, the outputs of experts with a zero gate are not
// computed; and Part 3, Step 2 of "Mixture of Experts: Why Mixtral Only Wakes
// Up Two Specialists" (the experts not kept are not run at all).  The layout
// (experts ascending, tokens ascending inside an expert) is this library's.
// An optional expert capacity (the Switch capacity described in Part 5 of the
// same page) keeps the first `capacity` pairs of each expert in that order and
// drops the rest (token_row = -1: the pair adds nothing to y).
//
// Kernels:
//   rank_kernel    per block of 256 pairs: expert histogram and the stable
//                  rank of every pair among the block's pairs of its expert
//                  (warp match + per-warp counts, no global atomics);
//   scan_kernel    one block: per-expert counts, segment offsets, each
//                  block's base inside each segment, and the M-block prefix
//                  the grouped GEMMs schedule from;
//   scatter_kernel row of every pair -> row_token, token_row;
//   gather_kernel  Xp[r] = x[row_token[r]], one thread per 16-byte vector.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kWarps = kPairsPerBlock / 32;

__global__ void __launch_bounds__(kPairsPerBlock) rank_kernel(const int32_t* __restrict__ idx,
                                                              int64_t R, int n,
                                                              int32_t* __restrict__ blockcounts,
                                                              int32_t* __restrict__ pair_rank) {
    griddep_wait();
    __shared__ int32_t whist[kWarps][kMaxExperts];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < kWarps * kMaxExperts; i += kPairsPerBlock) (&whist[0][0])[i] = 0;
    __syncthreads();

    const int64_t p = static_cast<int64_t>(blockIdx.x) * kPairsPerBlock + tid;
    int e = (p < R) ? idx[p] : -1;
    if (e < 0 || e >= n) e = -1;  // not a valid expert: ranked nowhere
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const uint32_t lt = (1u << lane) - 1u;
    const int wrank = __popc(peers & lt);
    if (e >= 0 && wrank == 0) whist[warp][e] = __popc(peers);
    __syncthreads();
    // exclusive prefix over the warps, per expert; block total
    for (int ex = tid; ex < n; ex += kPairsPerBlock) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int c = whist[w][ex];
            whist[w][ex] = run;
            run += c;
        }
        blockcounts[static_cast<int64_t>(blockIdx.x) * n + ex] = run;
    }
    __syncthreads();
    if (p < R) pair_rank[p] = (e >= 0) ? whist[warp][e] + wrank : -1;
    griddep_launch_dependents();
}

// Per-block counts are walked in chunks staged through shared memory, so
// the loads of a chunk are all in flight together (16 per thread); each expert's column is
// then scanned in place.  blockcounts ends up holding, for every block and
// expert, the block's first rank inside the expert's segment (the segment's
// offset is added by the scatter).
constexpr int kScanSmemInts = 8192;
constexpr int kScanUnroll = 16;

__global__ void __launch_bounds__(256) scan_kernel(int32_t* __restrict__ blockcounts, int nblk,
                                                   int n, int capacity, int bm,
                                                   int32_t* __restrict__ counts,
                                                   int32_t* __restrict__ offsets,
                                                   int32_t* __restrict__ mblk_base) {
    griddep_wait();
    __shared__ int s_warp[8];
    __shared__ int32_t s_chunk[kScanSmemInts];
    const int e = threadIdx.x;
    const int chunk_blocks = kScanSmemInts / n;
    int total = 0;
    for (int b0 = 0; b0 < nblk; b0 += chunk_blocks) {
        const int nb = min(chunk_blocks, nblk - b0);
        const int cnt = nb * n;
        int32_t* g = blockcounts + static_cast<int64_t>(b0) * n;
        __syncthreads();
        for (int i0 = 0; i0 < cnt; i0 += 256 * kScanUnroll) {
            int32_t v[kScanUnroll];  // all of a thread's loads in flight together
#pragma unroll
            for (int u = 0; u < kScanUnroll; ++u) {
                const int i = i0 + u * 256 + static_cast<int>(threadIdx.x);
                v[u] = i < cnt ? g[i] : 0;
            }
#pragma unroll
            for (int u = 0; u < kScanUnroll; ++u) {
                const int i = i0 + u * 256 + static_cast<int>(threadIdx.x);
                if (i < cnt) s_chunk[i] = v[u];
            }
        }
        __syncthreads();
        if (e < n) {
            for (int b = 0; b < nb; ++b) {
                const int v = s_chunk[b * n + e];
                s_chunk[b * n + e] = total;  // exclusive within the expert
                total += v;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < cnt; i += 256) g[i] = s_chunk[i];
    }
    total = min(total, capacity);  // pairs past the expert's capacity are dropped
    const int off = block_exclusive_scan(e < n ? total : 0, s_warp);
    const int mb = (e < n) ? (total + bm - 1) / bm : 0;
    const int mbase = block_exclusive_scan(mb, s_warp);
    if (e < n) {
        counts[e] = total;
        offsets[e] = off;
        mblk_base[e] = mbase;
    }
    if (e == n - 1) {
        offsets[n] = off + total;
        mblk_base[n] = mbase + mb;
    }
    griddep_launch_dependents();
}

__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ idx, int64_t R,
                                                      int K, int n, int capacity,
                                                      const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ blockbase,
                                                      const int32_t* __restrict__ pair_rank,
                                                      int32_t* __restrict__ row_token,
                                                      int32_t* __restrict__ token_row) {
    griddep_wait();
    const int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (p >= R) return;
    const int e = idx[p];
    const int rk = pair_rank[p];
    if (e < 0 || e >= n || rk < 0) {
        token_row[p] = -1;
        return;
    }
    const int rank_in_expert = blockbase[(p / kPairsPerBlock) * n + e] + rk;
    if (rank_in_expert >= capacity) {  // overflow: this pair skips its expert
        token_row[p] = -1;
        return;
    }
    const int dest = offsets[e] + rank_in_expert;
    row_token[dest] = static_cast<int32_t>(p / K);
    token_row[p] = dest;
    griddep_launch_dependents();
}

// Small batches (T*K <= kSmallDispatchPairs): the whole dispatch in one
// 1024-thread block -- counts, capped offsets, M-block prefix, stable ranks
// and the scatter -- with no global round trips between the steps.
constexpr int kSmallWarps = 32;

__global__ void __launch_bounds__(1024) dispatch_small_kernel(const int32_t* __restrict__ idx, int64_t R,
                                                              int K, int n, int capacity, int bm,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ mblk_base,
                                                              int32_t* __restrict__ row_token,
                                                              int32_t* __restrict__ token_row) {
    griddep_wait();
    __shared__ int32_t whist[kSmallWarps][kMaxExperts];   // per-warp counts, then warp bases
    __shared__ int32_t run[kMaxExperts];                  // pairs of each expert in earlier chunks
    __shared__ int32_t s_off[kMaxExperts];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < kMaxExperts; e += 1024) run[e] = 0;
    // pass 1: per-expert totals -> capped counts, offsets, M-block prefix
    for (int i = tid; i < kSmallWarps * kMaxExperts; i += 1024) (&whist[0][0])[i] = 0;
    __syncthreads();
    for (int64_t p = tid; p < R; p += 1024) {
        const int e = idx[p];
        if (e >= 0 && e < n) atomicAdd(&whist[0][e], 1);
    }
    __syncthreads();
    if (warp == 0) {
        // lane l scans experts 8l .. 8l+7; a shuffle scan joins the lanes
        int tot[8], mbs[8];
        int lane_tot = 0, lane_mb = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            tot[i] = (e < n) ? min(whist[0][e], capacity) : 0;
            mbs[i] = (tot[i] + bm - 1) / bm;
            lane_tot += tot[i];
            lane_mb += mbs[i];
        }
        int inc_tot = lane_tot, inc_mb = lane_mb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, inc_tot, o);
            const int b2 = __shfl_up_sync(0xffffffffu, inc_mb, o);
            if (lane >= o) {
                inc_tot += a;
                inc_mb += b2;
            }
        }
        int off = inc_tot - lane_tot, mbase = inc_mb - lane_mb;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane * 8 + i;
            if (e < n) {
                counts[e] = tot[i];
                offsets[e] = off;
                mblk_base[e] = mbase;
                s_off[e] = off;
            }
            if (e == n - 1) {
                offsets[n] = off + tot[i];
                mblk_base[n] = mbase + mbs[i];
            }
            off += tot[i];
            mbase += mbs[i];
        }
    }
    // pass 2: stable ranks chunk by chunk (1024 pairs per chunk, in pair order)
    for (int64_t c0 = 0; c0 < R; c0 += 1024) {
        __syncthreads();
        for (int i = tid; i < kSmallWarps * kMaxExperts; i += 1024) (&whist[0][0])[i] = 0;
        __syncthreads();
        const int64_t p = c0 + tid;
        int e = (p < R) ? idx[p] : -1;
        if (e < 0 || e >= n) e = -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int wrank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && wrank == 0) whist[warp][e] = __popc(peers);
        __syncthreads();
        for (int ex = tid; ex < n; ex += 1024) {
            int acc = run[ex];
            for (int w = 0; w < kSmallWarps; ++w) {
                const int cnt = whist[w][ex];
                whist[w][ex] = acc;
                acc += cnt;
            }
            run[ex] = acc;
        }
        __syncthreads();
        if (p < R) {
            if (e < 0) {
                token_row[p] = -1;
            } else {
                const int rank_in_expert = whist[warp][e] + wrank;
                if (rank_in_expert >= capacity) {
                    token_row[p] = -1;
                } else {
                    const int dest = s_off[e] + rank_in_expert;
                    row_token[dest] = static_cast<int32_t>(p / K);
                    token_row[p] = dest;
                }
            }
        }
    }
    griddep_launch_dependents();
}

cudaError_t launch_dispatch(const int32_t* topk_idx, int64_t T, int K, int n, int bm,
                            const DispatchBufs& b, cudaStream_t st, int capacity) {
    const int64_t R = T * K;
    if (R <= kSmallDispatchPairs) {
        launch_k(dispatch_small_kernel, dim3(1), dim3(1024), 0, st, topk_idx, R, K, n, capacity, bm, b.counts, b.offsets,
                                                  b.mblk_base, b.row_token, b.token_row);
        return cudaGetLastError();
    }
    const int nblk = static_cast<int>((R + kPairsPerBlock - 1) / kPairsPerBlock);
    launch_k(rank_kernel, dim3(nblk), dim3(kPairsPerBlock), 0, st, topk_idx, R, n, b.blockcounts, b.pair_rank);
    launch_k(scan_kernel, dim3(1), dim3(256), 0, st, b.blockcounts, nblk, n, capacity, bm, b.counts, b.offsets, b.mblk_base);
    launch_k(scatter_kernel, dim3(static_cast<unsigned>((R + 255) / 256)), dim3(256), 0, st, 
        topk_idx, R, K, n, capacity, b.offsets, b.blockcounts, b.pair_rank, b.row_token, b.token_row);
    return cudaGetLastError();
}

__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ x,
                                                     const int32_t* __restrict__ row_token,
                                                     int64_t R, int64_t T, int64_t vec_per_row,
                                                     uint4* __restrict__ xp) {
    griddep_wait();
    const int64_t total = R * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += stride) {
        const int64_t r = i / vec_per_row;
        const int64_t v = i - r * vec_per_row;
        const int64_t t = __ldg(row_token + r);
        if (t < 0 || t >= T) continue;  // a row no valid pair reached (bad expert ids)
        xp[i] = __ldg(x + t * vec_per_row + v);
    }
    griddep_launch_dependents();
}

cudaError_t launch_gather(const void* x, const int32_t* row_token, int64_t R, int64_t T,
                          int64_t row_bytes, void* xp, int num_sms, cudaStream_t st) {
    int64_t blocks = (R * (row_bytes / 16) + 255) / 256;
    const int64_t cap = static_cast<int64_t>(num_sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    launch_k(gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, 
        static_cast<const uint4*>(x), row_token, R, T, row_bytes / 16, static_cast<uint4*>(xp));
    return cudaGetLastError();
}

}  // namespace moe
