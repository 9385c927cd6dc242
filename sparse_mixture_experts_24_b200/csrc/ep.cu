// ep.cu -- expert parallelism: the n experts split over W ranks (rank q holds
// experts [q n/W, (q+1) n/W)), each rank routing its own tokens.  The
// exchange steps are fused with the copies and the combine that surround
// them, as stores to and loads from the other ranks' buffers (peer memory
// over NVLink; on one GPU, plain device memory):
//
//   ep_plan_kernel     from every rank's per-expert counts [W][n]: where this
//                      rank's rows of each expert start in the owner's
//                      receive buffer, and (as an owner) the segment offsets
//                      and M-block prefix of its own experts;
//   ep_scatter_kernel  (token, slot) pair -> its row of x stored straight into
//                      the owner rank's receive buffer, and its position
//                      recorded for the combine (the dispatch all-to-all);
//   ep_combine_kernel  y[t] = sum_k g[t][k] * O_owner[position of (t, k)], the
//                      rows loaded from the owners' output buffers (the
//                      combine all-to-all), slot order k = 0..K-1 in fp32.
//
// Receive layout on an owner: its experts in order; inside an expert the
// rows of rank 0, then rank 1, ...; inside a rank its pairs of that expert in
// token order -- so the owner's grouped GEMMs read contiguous segments.
//
// Source: the flash-card page on "Mixtral of Experts" names expert
// parallelism (experts placed on different GPUs) in section 2.1, with the
// warning that uneven routing overloads some GPUs, and again in section 5
// (temporal locality concentrates consecutive tokens on one expert).  The
// pages give no mechanics: the layout above, the fused exchange and the
// plan are this library's reading.  The layer computed is unchanged (the
// layer equation of section 2.1).
#include "common.cuh"
#include "kernels.h"

namespace moe {

// One block of 256 threads, thread = expert (n <= 256).
__global__ void __launch_bounds__(256) ep_plan_kernel(const int32_t* __restrict__ counts_all, int W, int n,
                                                      int rank, const int32_t* __restrict__ own_counts,
                                                      int64_t recv_rows, int32_t* __restrict__ dst_base,
                                                      int32_t* __restrict__ loff, int32_t* __restrict__ lmblk,
                                                      int* __restrict__ status) {
    griddep_wait();
    __shared__ int s_warp[8];
    __shared__ int s_ex[256];
    __shared__ int s_mb[256];
    __shared__ int s_bad;
    __shared__ unsigned long long s_owner_rows[kMaxEpRanks];
    const int e = threadIdx.x;
    const int nl = n / W;
    if (e == 0) s_bad = 0;
    if (e < kMaxEpRanks) s_owner_rows[e] = 0;
    __syncthreads();
    int tot = 0, pre = 0;
    if (e < n) {
        long long t64 = 0, p64 = 0;
        for (int s = 0; s < W; ++s) {
            const int c = counts_all[static_cast<int64_t>(s) * n + e];
            if (c < 0) s_bad = 1;
            if (s < rank) p64 += c;
            t64 += c;
        }
        if (own_counts && own_counts[e] != counts_all[static_cast<int64_t>(rank) * n + e]) s_bad = 1;
        // every owner's rows must fit its buffer (checked in 64 bits, so the
        // 32-bit offsets below cannot wrap)
        if (t64 > recv_rows) s_bad = 1;
        atomicAdd(&s_owner_rows[e / nl], static_cast<unsigned long long>(t64 > 0 ? t64 : 0));
        tot = static_cast<int>(t64 > recv_rows ? 0 : t64);
        pre = static_cast<int>(p64 > recv_rows ? 0 : p64);
    }
    __syncthreads();
    if (e < W && s_owner_rows[e] > static_cast<unsigned long long>(recv_rows)) s_bad = 1;
    if (e == 0) {  // all rows of all owners: the scan below runs in 32 bits
        unsigned long long all = 0;
        for (int q = 0; q < W; ++q) all += s_owner_rows[q];
        if (all > 2147483647ull) s_bad = 1;
    }
    const int ex = block_exclusive_scan(e < n ? tot : 0, s_warp);
    const int owner = e < n ? e / nl : -1;
    const int mb = (owner == rank) ? (tot + kTcBM - 1) / kTcBM : 0;
    const int mbx = block_exclusive_scan(mb, s_warp);
    s_ex[e] = ex;
    s_mb[e] = mbx;
    __syncthreads();
    const int seg = e < n ? ex - s_ex[owner * nl] : 0;  // start of expert e inside its owner's buffer
    __syncthreads();
    // on an error every segment is empty, so nothing downstream stores a row
    const bool bad = s_bad != 0;
    if (e < n) {
        dst_base[e] = bad ? 0 : seg + pre;
        if (owner == rank) {
            const int i = e - rank * nl;
            loff[i] = bad ? 0 : seg;
            lmblk[i] = bad ? 0 : mbx - s_mb[rank * nl];
            if (i == nl - 1) {
                loff[nl] = bad ? 0 : seg + tot;
                lmblk[nl] = bad ? 0 : mbx - s_mb[rank * nl] + mb;
            }
        }
    }
    if (e == 0 && bad) atomicOr(status, kStatusEpPlan);
    griddep_launch_dependents();
}

// One warp per (token, slot) pair: position = dst_base[e] + the pair's rank
// among this rank's pairs of e (token order, from the dispatch); the x row is
// copied to the owner's buffer in 16-byte vectors.  Nothing is stored when
// the plan flagged an error.
__global__ void __launch_bounds__(256) ep_scatter_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ token_row,
                                                         const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ dst_base, int64_t R, int K,
                                                         int n, int nl, const __grid_constant__ EpPeers recv, int64_t recv_rows,
                                                         int vec_per_row, int32_t* __restrict__ row_pos,
                                                         const int* __restrict__ status) {
    griddep_wait();
    const bool bad = (*status & kStatusEpPlan) != 0;
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int64_t p = first; p < R; p += warps) {
        const int e = __ldg(idx + p);
        const int j = __ldg(token_row + p);
        int64_t pos = -1;
        if (!bad && e >= 0 && e < n && j >= 0) {
            pos = static_cast<int64_t>(__ldg(dst_base + e)) + (j - __ldg(offsets + e));
            if (pos < 0 || pos >= recv_rows) pos = -1;
        }
        if (lane == 0) row_pos[p] = static_cast<int32_t>(pos);
        if (pos < 0) continue;
        const uint4* src = x + (p / K) * vec_per_row;
        uint4* dst = static_cast<uint4*>(recv.ptr[e / nl]) + pos * vec_per_row;
        for (int v = lane; v < vec_per_row; v += 32) dst[v] = __ldg(src + v);
    }
    // the stores reach the owners' memory before anything this grid precedes
    __threadfence_system();
    griddep_launch_dependents();
}

// One thread per 16-byte vector of y, as the single-GPU combine, the rows
// read from the owners' output buffers.
__global__ void __launch_bounds__(256) ep_combine_kernel(const int32_t* __restrict__ idx,
                                                         const float* __restrict__ topk_w,
                                                         const int32_t* __restrict__ row_pos, int64_t T, int K,
                                                         int n, int nl, const __grid_constant__ EpPeers out,
                                                         int vec_per_row, uint4* __restrict__ y) {
    griddep_wait();
    const int64_t total = T * vec_per_row;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / vec_per_row;
        const int64_t v = i - t * vec_per_row;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int k = 0; k < K; ++k) {
            const int32_t pos = __ldg(row_pos + t * K + k);
            const int e = __ldg(idx + t * K + k);
            if (pos < 0 || e < 0 || e >= n) continue;
            const float g = __ldg(topk_w + t * K + k);
            const uint4* o_row = static_cast<const uint4*>(out.ptr[e / nl]) + static_cast<int64_t>(pos) * vec_per_row;
            fma_bf16x8(acc, g, o_row[v]);
        }
        y[i] = pack_bf16x8(acc);
    }
    griddep_launch_dependents();
}

cudaError_t launch_ep_plan(const int32_t* counts_all, int W, int n, int rank, const int32_t* own_counts,
                           int64_t recv_rows, int32_t* dst_base, int32_t* loff, int32_t* lmblk, int* status,
                           cudaStream_t st) {
    launch_k(ep_plan_kernel, dim3(1), dim3(256), 0, st, counts_all, W, n, rank, own_counts, recv_rows, dst_base,
             loff, lmblk, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_scatter(const void* x, const int32_t* idx, const int32_t* token_row, const int32_t* offsets,
                              const int32_t* dst_base, int64_t T, int K, int n, int nl, const EpPeers& recv,
                              int64_t recv_rows, int d, int32_t* row_pos, const int* status, int num_sms,
                              cudaStream_t st) {
    const int64_t R = T * K;
    int64_t blocks = (R + 7) / 8;
    if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
    if (blocks < 1) blocks = 1;
    launch_k(ep_scatter_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
             static_cast<const uint4*>(x), idx, token_row, offsets, dst_base, R, K, n, nl, recv, recv_rows, d / 8,
             row_pos, status);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const int32_t* idx, const float* topk_w, const int32_t* row_pos, int64_t T, int K,
                              int n, int nl, const EpPeers& out, int d, void* y, int num_sms, cudaStream_t st) {
    const int64_t vecs = T * (d / 8);
    int64_t blocks = (vecs + 255) / 256;
    if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
    if (blocks < 1) blocks = 1;
    launch_k(ep_combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, idx, topk_w, row_pos, T,
             K, n, nl, out, d / 8, static_cast<uint4*>(y));
    return cudaGetLastError();
}

}  // namespace moe
