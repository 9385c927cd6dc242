// kernels.h -- host-side launchers of the MoE kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Kernels launched by one API call form a chain on its stream; every launch
// after the first carries the programmatic-stream-serialization attribute, so
// it can be scheduled while its predecessor drains (each kernel waits with
// griddepcontrol.wait before touching memory).  MOE_PDL=0 turns this off.
bool pdl_enabled();
extern thread_local bool g_chain_started;
inline void chain_begin() { g_chain_started = false; }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (g_chain_started && pdl_enabled()) ? 1 : 0;
    g_chain_started = true;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Rows of one M-block of the tensor-core GEMMs and of the CUDA-core GEMMs.
// Bits of the device status word (workspace): set by a kernel that gave up a
// bounded wait, read and cleared by moe_sync_status.
enum : int {
    kStatusTimeoutFull = 1,      // waited too long for a TMA stage to land
    kStatusTimeoutEmpty = 2,     // waited too long for the MMA to free a stage
    kStatusTimeoutAccum = 4,     // waited too long for an accumulator buffer
    kStatusTimeoutDrain = 8,     // waited too long while draining at exit
    kStatusSelfTest = 16,        // the self-test's wait ran out (as it should)
    kStatusEpPlan = 32,          // expert-parallel counts disagree, or a receive buffer is too small
};

constexpr int kTcBM = 128;
constexpr int kSimtBM = 64;
// (token, slot) pairs per dispatch block.
constexpr int kPairsPerBlock = 256;

// Router: logits (fp32), top-K, softmax over the kept K.
cudaError_t launch_router(const void* x, bool x_bf16, const float* Wg, int64_t T, int d, int n,
                          int K, int32_t* topk_idx, float* topk_w, float* logits_ws, int num_sms,
                          cudaStream_t st);

// Top-K + softmax of logits already in memory (warp per token): the logits
// are the sum, in order, of `splits` partial arrays [splits][T][n].
cudaError_t launch_router_topk(const float* logits, int splits, int64_t T, int n, int K,
                               int32_t* topk_idx, float* topk_w, cudaStream_t st);

// Largest number of K splits of the tensor-core router (workspace: logits
// [kRouterMaxSplits][T][n]).
constexpr int kRouterMaxSplits = 4;

// Tensor-core router for bf16 x: splits W_g into three bf16 parts
// (parts [3][npad][d], npad = n rounded up to 16), computes the logits
// [T][n] with tcgen05 (tm_x over x [T][d], tm_w over parts [3*npad][d], both
// with 64 x rows boxes: 128 rows for x, npad rows for the parts), then the
// top-K and softmax: in the router's own epilogue (the d-splits of a token
// block are one cluster), or, with MOE_ROUTER_TOPK=separate, by
// router_topk_kernel over logits in the workspace.
// Kernels launch_router_tc issues for a top-K of K: W_g split + fused router
// (K <= 8), or W_g split + logits + top-K.
int router_tc_launches(int K);
cudaError_t launch_router_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                             uint16_t* parts, int64_t T, int d, int n, int K, float* logits,
                             int32_t* topk_idx, float* topk_w, int* status, int num_sms,
                             cudaStream_t st);
int router_tc_smem_bytes(int n);

// Dispatch workspace (device, int32 unless noted).
struct DispatchBufs {
    int32_t* blockcounts;  // [nblk][n]: per-block counts, then each block's first rank in a segment
    int32_t* pair_rank;    // [R]: stable rank of each pair inside its block and expert
    int32_t* counts;       // [n]
    int32_t* offsets;      // [n+1]
    int32_t* mblk_base;    // [n+1]: exclusive prefix of M-blocks per expert
    int32_t* row_token;    // [R]
    int32_t* token_row;    // [R] = [T][K]
};

// Histogram + stable in-block ranks, scan, scatter.  bm = rows per M-block of
// the GEMM that consumes the segments; capacity = most pairs one expert takes
// (kNoCapacity: all).
constexpr int kNoCapacity = 2147483647;
// Up to this many pairs the dispatch is one single-block kernel (else three).
constexpr int kSmallDispatchPairs = 4096;
inline int dispatch_kernel_count(int64_t pairs) { return pairs <= kSmallDispatchPairs ? 1 : 3; }
cudaError_t launch_dispatch(const int32_t* topk_idx, int64_t T, int K, int n, int bm,
                            const DispatchBufs& b, cudaStream_t st, int capacity = kNoCapacity);

// Load-balancing statistics from logits [splits][T][n] (summed in split
// order) and the routing topk_idx [T][K]: f[n] (share of routed pairs),
// P[n] (mean softmax probability), aux[0] = alpha * n * sum f P.  partial is
// scratch of ceil(T/256) * n floats, counts scratch of n ints.
cudaError_t launch_router_stats(const float* logits, int splits, int64_t T, int n, int K,
                                const int32_t* topk_idx, float alpha, float* partial,
                                int32_t* counts, float* f, float* P, float* aux, cudaStream_t st);

// Logits only (no top-K) into logits [splits][T][n]; returns the split count.
cudaError_t launch_router_logits_tc(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const float* Wg,
                                    uint16_t* parts, int64_t T, int d, int n, float* logits, int* status,
                                    int num_sms, cudaStream_t st, int* splits_out);
cudaError_t launch_router_logits_simt(const void* x, bool x_bf16, const float* Wg, int64_t T, int d,
                                      int n, float* logits, cudaStream_t st);

// Xp[r] = x[row_token[r]] for r < R (row_bytes per row, multiple of 16);
// rows whose token is outside [0, T) are skipped.
cudaError_t launch_gather(const void* x, const int32_t* row_token, int64_t R, int64_t T,
                          int64_t row_bytes, void* xp, int num_sms, cudaStream_t st);

// y[t] = sum_k topk_w[t][k] * O[token_row[t][k]]; O and y bf16 (o_bf16) or fp32.
cudaError_t launch_combine(const void* O, bool bf16, const int32_t* token_row, const float* topk_w,
                           int64_t T, int K, int d, void* y, int num_sms, cudaStream_t st);

// Expert-choice routing: probabilities St [n][T], per-expert selection of C
// tokens (rows e*C .. e*C+C-1, tokens ascending) into sel_token / sel_gate /
// row_token, rowmap [T][n] (row of (t, e) or -1), and the dispatch arrays.
cudaError_t launch_ec_route(const float* logits, int splits, int64_t T, int n, int C, int bm, float* St,
                            int32_t* rowmap, int32_t* sel_token, float* sel_gate, int32_t* row_token,
                            int32_t* counts, int32_t* offsets, int32_t* mblk_base, cudaStream_t st);
// y[t] = sum_e gate_of_row[rowmap[t][e]] * O[rowmap[t][e]] (expert order).
cudaError_t launch_ec_combine(const void* O, bool bf16, const int32_t* rowmap, const float* gate_of_row,
                              int64_t T, int n, int d, void* y, int num_sms, cudaStream_t st);

// One thread waits on an mbarrier nothing arrives at, with the given budget;
// sets kStatusSelfTest in *status when the wait runs out.
cudaError_t launch_bounded_wait_probe(int* status, long long budget_cycles, cudaStream_t st);

// CUDA-core fp32 grouped GEMMs (fp32 handles).
//   H[r] = silu(Xp[r] . w1[e]) * (Xp[r] . w3[e]) for rows r of expert e
cudaError_t launch_simt_gemm1(const float* xp, const float* w1, const float* w3, float* h,
                              const int32_t* offsets, const int32_t* mblk_base, int n, int64_t R,
                              int d, int F, cudaStream_t st);
//   O[r] = H[r] . w2[e]
cudaError_t launch_simt_gemm2(const float* h, const float* w2, float* o, const int32_t* offsets,
                              const int32_t* mblk_base, int n, int64_t R, int d, int F,
                              cudaStream_t st);

// tcgen05 grouped GEMMs (bf16 handles).  Tensor maps are built by the host
// (see moe_api.cu) over: Xp [R_cap][d], w1/w3 [n][d][F], H [R_cap][F], w2 [n][F][d].
// Gates rounded to bf16 in place (router.cu).
cudaError_t launch_gates_to_bf16(float* topk_w, int64_t count, int num_sms, cudaStream_t st);

// Expert parallelism (ep.cu): one device pointer per rank, by value.
constexpr int kMaxEpRanks = 16;
struct EpPeers {
    void* ptr[kMaxEpRanks];
};
cudaError_t launch_ep_plan(const int32_t* counts_all, int W, int n, int rank, const int32_t* own_counts,
                           int64_t recv_rows, int32_t* dst_base, int32_t* loff, int32_t* lmblk, int* status,
                           cudaStream_t st);
cudaError_t launch_ep_scatter(const void* x, const int32_t* idx, const int32_t* token_row, const int32_t* offsets,
                              const int32_t* dst_base, int64_t T, int K, int n, int nl, const EpPeers& recv,
                              int64_t recv_rows, int d, int32_t* row_pos, const int* status, int num_sms,
                              cudaStream_t st);
cudaError_t launch_ep_combine(const int32_t* idx, const float* topk_w, const int32_t* row_pos, int64_t T, int K,
                              int n, int nl, const EpPeers& out, int d, void* y, int num_sms, cudaStream_t st);

struct TcGemmArgs {
    const int32_t* offsets;
    const int32_t* mblk_base;
    int n;
    int64_t R;         // rows (T*K): bounds the tile count
    int k_blocks;      // reduction length / 64
    int n_tiles;       // tiles along the output columns
    int out_cols;      // F (GEMM1) or d (GEMM2)
    void* out;         // H (GEMM1) or O (GEMM2), bf16 row-major [R][out_cols]
    int* status;       // device status word
    // E4M3 kernels only: row scale [R] and per-expert column scales [n][out_cols]
    // (GEMM1: w1 and w3; GEMM2: w2 in col_scale0)
    const float* row_scale;
    const float* col_scale0;
    const float* col_scale1;
    int balanced;      // 1: spread the tiles evenly over the fewest CTAs (balanced_ctas)
    int band_m;        // single-SM kernel: row blocks per band of the tile order (0: no bands)
    // launch_tc_gemm1_gather only: A rows gathered from x [x_rows][x_cols] bf16
    // (tile row r = token row_token[row0 + r])
    const uint16_t* x;
    const int32_t* row_token;
    int64_t x_rows;
    int64_t x_cols;
};

cudaError_t launch_tc_gemm1(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1,
                            const CUtensorMap& tm_w3, const TcGemmArgs& a, int num_sms,
                            cudaStream_t st);
cudaError_t launch_tc_gemm2(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a,
                            int num_sms, cudaStream_t st);
// GEMM1 with the A rows gathered from x by the kernel itself (no Xp).
cudaError_t launch_tc_gemm1_gather(const CUtensorMap& tm_w1, const CUtensorMap& tm_w3, const TcGemmArgs& a,
                                   int num_sms, cudaStream_t st);
cudaError_t launch_tc_gemm1_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1,
                                 const CUtensorMap& tm_q3, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st);
cudaError_t launch_tc_gemm2_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                 int num_sms, cudaStream_t st);

// 4-bit weights (fp4.cu, gemm_fp4.cu): codes [n][rows][cols/2] (column 2j in
// the low nibble of byte j), E4M3 block scales [n][rows/16][cols], fp32
// matrix scales [n].  Four launches (a memset, max, codes, matrix scale).
cudaError_t launch_quantize_weights_fp4(const void* w, bool bf16, int n, int rows, int cols, uint8_t* codes,
                                        uint8_t* bscale, float* tscale, int num_sms, cudaStream_t st);

struct Fp4GemmArgs {
    const int32_t* offsets;
    const int32_t* mblk_base;
    int n;
    int64_t R;
    int k_blocks;      // reduction length / 64
    int n_tiles;
    int out_cols;
    void* out;         // bf16 [R][out_cols]
    int* status;
    const float* tscale0;  // [n] matrix scales: w1 (GEMM1) or w2 (GEMM2)
    const float* tscale1;  // [n] w3 (GEMM1)
    int balanced;              // as TcGemmArgs::balanced
};

// tm_xp / tm_h: bf16 rows (64 x 128 boxes, 128-byte swizzle); tm_c*: codes
// [n][K][N/2] uint8 (64 x 64 boxes, no swizzle); tm_s*: block scales
// [n][K/16][N] uint8 (128 x 4 boxes, no swizzle).
cudaError_t launch_fp4_gemm1(const CUtensorMap& tm_xp, const CUtensorMap& tm_c1, const CUtensorMap& tm_s1,
                             const CUtensorMap& tm_c3, const CUtensorMap& tm_s3, const Fp4GemmArgs& a, int num_sms,
                             cudaStream_t st);
cudaError_t launch_fp4_gemm2(const CUtensorMap& tm_h, const CUtensorMap& tm_c2, const CUtensorMap& tm_s2,
                             const Fp4GemmArgs& a, int num_sms, cudaStream_t st);

// 4-bit weights and 4-bit activations on the block-scaled tensor cores
// (w4a4.cu, gemm_w4a4.cu).  Scale chunks: 512 bytes holding the 4 E4M3 scales
// (one per 16 K) of 128 rows for one 64-wide K step.
//   pack: codes [n][K][N/2] + scales [n][K/16][N] (moe_quantize_weights_fp4) ->
//   K-major codes [n][N][K/2] + chunks [n][N/128][K/64][512].  N % 128 == 0.
//   With codes_pair (w3 next to w1): [n][2N][K/2], 128-row blocks of 64 w1
//   columns then the same 64 w3 columns; chunks [n][2N/128][K/64][512].
cudaError_t launch_w4a4_pack(const uint8_t* codes, const uint8_t* bscale, const uint8_t* codes_pair,
                             const uint8_t* bscale_pair, int n, int K, int N, uint8_t* packed, uint8_t* chunks,
                             cudaStream_t st);
//   rows: bf16 rows (row r reads src row row_src[r], or r without row_src) ->
//   codes [R][K/2], row scales [R], and the chunks of the GEMM's tiles of
//   tile_rows rows (128 or 32) [tiles][K/64][512] (tile of row r: mblk_base[e]
//   + (r - offsets[e]) / tile_rows).  Rows past offsets[n] are skipped.
cudaError_t launch_w4a4_rows(const uint16_t* src, const int32_t* row_src, int64_t src_rows, int64_t rows_max, int K,
                             const int32_t* offsets, const int32_t* mblk_base, int n, int tile_rows, uint8_t* codes,
                             uint8_t* chunks, float* rscale, int num_sms, cudaStream_t st);

struct W4a4GemmArgs {
    const int32_t* offsets;
    const int32_t* mblk_base;
    int n;
    int64_t R;
    int k_steps;           // reduction length / 256
    int n_tiles;
    int out_cols;          // F (GEMM1) or d (GEMM2)
    int n_rows_b;          // rows of the packed weight matrix (2F for w1|w3, d for w2)
    void* out;             // bf16 [R][out_cols]
    int* status;
    const float* row_scale;    // [R] activation row scales
    const float* mscale0;      // [n] matrix scales: w1 (GEMM1) / w2 (GEMM2)
    const float* mscale1;      // [n] w3 (GEMM1)
    const uint8_t* a_chunks;   // activation scale chunks [tiles][K/64][512]
    const uint8_t* b_chunks;   // weight scale chunks [n][rows/128][K/64][512] (w1|w3 pairs, or w2)
    int balanced;              // as TcGemmArgs::balanced
};

// tm_a: activation codes [R][K/2] uint8 (boxes of tile_rows rows x 128 bytes,
// 128-byte swizzle); tm_b: packed weight codes [n][rows][K/2] uint8 (128 x 128
// x 1 boxes, same): the w1|w3 pair pack for GEMM1, w2 for GEMM2.  wide:
// 256-column tiles (one accumulator) instead of 128-column tiles (two
// accumulators); tile_rows: 128, or 32 (wide only) with the segments laid out
// in 32-row M-blocks.
int w4a4_tile_cols(bool wide);
cudaError_t launch_w4a4_gemm1(const CUtensorMap& tm_xq, const CUtensorMap& tm_w13, const W4a4GemmArgs& a, bool wide,
                              int tile_rows, int num_sms, cudaStream_t st);
cudaError_t launch_w4a4_gemm2(const CUtensorMap& tm_hq, const CUtensorMap& tm_w2, const W4a4GemmArgs& a, bool wide,
                              int tile_rows, int num_sms, cudaStream_t st);

// 4-bit weights with bf16 activations, the weights decoded into tensor
// memory (gemm_w4a16.cu).  Packed weights: per (expert, tile of 128 packed
// columns, 64 reduction rows) a 4,608-byte block of codes ([2][128][16]
// bytes, 8 rows per 32-bit word in the decoder's bit order) and block scales
// ([128][4] E4M3 codes).  With codes_pair (w3 beside w1) tile j holds columns
// 64j .. 64j+63 of w1 then the same columns of w3.  K % 64 == 0; N % 128 == 0
// (N % 64 == 0 with a pair).
cudaError_t launch_w4a16_pack(const uint8_t* codes, const uint8_t* bscale, const uint8_t* codes_pair,
                              const uint8_t* bscale_pair, int n, int K, int N, uint8_t* packed, cudaStream_t st);
struct W4a16GemmArgs {
    const int32_t* offsets;
    const int32_t* mblk_base;  // per-expert prefix of tile_rows-row blocks
    int n;
    int64_t R;
    int k_blocks;          // reduction length / 64
    int n_tiles;           // weight tiles per expert (F / 64 for GEMM1, d / 128 for GEMM2)
    int out_cols;          // F (GEMM1) or d (GEMM2)
    void* out;             // bf16 [R][out_cols]
    int* status;
    const uint8_t* wpack;  // packed weights [n][n_tiles][k_blocks][4608]
    const float* mscale0;  // [n] matrix scales: w1 (GEMM1) / w2 (GEMM2)
    const float* mscale1;  // [n] w3 (GEMM1)
    int balanced;          // as TcGemmArgs::balanced
};
// Token rows per tile: 32 when the experts average at most 32 rows, else 128.
int w4a16_tile_rows(int64_t R, int n);
// tm_xp / tm_h: bf16 rows as 3-D maps (64 columns, rows, 64-column chunk),
// boxes of 64 x tile_rows x (4 chunks for 32 rows, 2 for 128), 128-byte swizzle.
cudaError_t launch_w4a16_gemm1(const CUtensorMap& tm_xp, const W4a16GemmArgs& a, int tile_rows, int num_sms,
                               cudaStream_t st);
cudaError_t launch_w4a16_gemm2(const CUtensorMap& tm_h, const W4a16GemmArgs& a, int tile_rows, int num_sms,
                               cudaStream_t st);
// E4M3 quantisation (e4m3.cu).  Codes are those of v / scale with the quotient
// rounded to fp32, then to E4M3 by round-to-nearest-even with saturation to
// +-448; scale = max |v| / 448 over the group (1 for an all-zero group).
//   weights [n][rows][cols] -> codes of the same shape, scales [n][cols] (per
//   output column over the reduction rows); three launches.
cudaError_t launch_quantize_weights_e4m3(const void* w, bool bf16, int n, int rows, int cols,
                                         uint8_t* codes, float* scales, int num_sms, cudaStream_t st);
//   rows of src (bf16 or fp32, `cols` wide) -> codes [rows][cols] and one scale
//   per row.  With row_src, row r reads source row row_src[r] (a gather; rows
//   whose source is outside [0, src_rows) are skipped); with row_limit, rows at
//   or past *row_limit are skipped.
cudaError_t launch_quantize_rows_e4m3(const void* src, bool bf16, const int32_t* row_src, int64_t src_rows,
                                      int64_t rows, const int32_t* row_limit, int cols, uint8_t* codes,
                                      float* scales, int num_sms, cudaStream_t st);

// The same GEMMs with two 128-row blocks per single-SM tile (two MMAs share
// each stage's B; gemm_tc3.cu): mblk_base counts 128-row blocks as for
// launch_tc_gemm1/2, the weight maps are the same 4-D maps, and the tile order
// takes its bands from a.band_m (counted in 128-row blocks).
cudaError_t launch_tc_gemm1_dual(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1, const CUtensorMap& tm_w3,
                                 const TcGemmArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_tc_gemm2_dual(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st);
// The same on E4M3 operands (maps as launch_tc_gemm1_e4m3 / launch_tc_gemm2_e4m3).
cudaError_t launch_tc_gemm1_dual_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1, const CUtensorMap& tm_q3,
                                      const TcGemmArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_tc_gemm2_dual_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                      int num_sms, cudaStream_t st);

// The same GEMMs on CTA pairs (cta_group::2, 256-row tiles): mblk_base must
// count 256-row blocks; the weight maps are 4-D (64 columns, K rows, 64-column
// chunk, expert) with boxes of two chunks; the tile order takes its bands
// from a.band_m (counted in 128-row blocks).
constexpr int kTcPairBM = 256;
cudaError_t launch_tc_gemm1_pair(const CUtensorMap& tm_xp, const CUtensorMap& tm_w1,
                                 const CUtensorMap& tm_w3, const TcGemmArgs& a, int num_sms,
                                 cudaStream_t st);
cudaError_t launch_tc_gemm2_pair(const CUtensorMap& tm_h, const CUtensorMap& tm_w2, const TcGemmArgs& a,
                                 int num_sms, cudaStream_t st);
// The same on E4M3 operands (maps as launch_tc_gemm1_e4m3 / launch_tc_gemm2_e4m3).
cudaError_t launch_tc_gemm1_pair_e4m3(const CUtensorMap& tm_x8, const CUtensorMap& tm_q1,
                                      const CUtensorMap& tm_q3, const TcGemmArgs& a, int num_sms,
                                      cudaStream_t st);
cudaError_t launch_tc_gemm2_pair_e4m3(const CUtensorMap& tm_h8, const CUtensorMap& tm_q2, const TcGemmArgs& a,
                                      int num_sms, cudaStream_t st);

}  // namespace moe
