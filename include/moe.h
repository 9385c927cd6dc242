/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse mixture-of-experts layer.
 *
 * The layer (the equation of "Mixtral of Experts", section 2.1 "Sparse
 * Mixture of Experts", as given on the learn.ifs.name flash-card page):
 *
 *   y = sum_{i=0}^{n-1} Softmax(TopK(x . W_g))_i * SwiGLU_i(x)
 *   SwiGLU_i(x) = (silu(x . w1_i) (*) (x . w3_i)) . w2_i,  silu(z) = z * sigmoid(z)
 *
 * A bias-free linear router scores n experts per token, keeps the K largest
 * logits, normalises those K with a softmax, and sums the chosen experts'
 * SwiGLU outputs with those weights ("Mixture of Experts: Why Mixtral Only
 * Wakes Up Two Specialists", Part 3, Steps 1-4).
 *
 * Conventions shared by every entry point
 *   - All tensors are row-major and live in device memory of the current CUDA
 *     device; every pointer must be 16-byte aligned.
 *       x[T][d]            activations, dtype of the handle
 *       W_g[d][n]          router weights, always fp32 (column e scores expert e)
 *       w1[n][d][ffn]      gate projection of each expert, dtype of the handle
 *       w3[n][d][ffn]      up projection of each expert, dtype of the handle
 *       w2[n][ffn][d]      down projection of each expert, dtype of the handle
 *       y[T][d]            output, dtype of the handle (fp32 accumulation,
 *                          rounded once to bf16 for bf16 handles)
 *       topk_idx[T][K]     chosen experts, int32, by descending logit; equal
 *                          logits keep the lower expert index first
 *       topk_w[T][K]       their softmax weights, fp32, summing to 1 per token
 *   - The caller owns every tensor it passes.  The handle owns only its
 *     workspace (routing maps, permuted activations, the expert hidden layer
 *     and per-row expert outputs), which it allocates with cudaMalloc on the
 *     first call that needs more room and frees in moe_destroy.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; a returned MOE_OK reports launch-time
 *     success only.  moe_sync_status reports device-side failures.
 *   - A handle may be used by one host thread at a time, on the device on
 *     which its workspace was first allocated.  Calls on one handle must not
 *     overlap on the GPU (they share the workspace): issue them on one stream
 *     or order the streams.
 *   - On any error nothing is launched, the outputs are untouched, and
 *     moe_last_error() describes the failure.
 *   - After moe_reserve(T_max) (and, for moe_forward_e4m3 and
 *     moe_forward_w4a4, one earlier call of it, which sizes its part of the
 *     workspace), a forward call with T <= T_max only enqueues kernels: it
 *     allocates nothing and does not synchronise with the host, so it can be
 *     captured into a CUDA graph and replayed (the kernels keep their
 *     programmatic dependent launches).  The captured call reads x and the
 *     weights from the addresses it was given.
 *   - Environment switches, for measurement and tests (every setting is
 *     parity-tested against the same oracle and tolerances): MOE_PDL=0 (plain
 *     stream order) and MOE_ROUTER_TOPK=separate, read once per process;
 *     read per call: MOE_GEMM_PATH=single|pair|dual (the bf16 and E4M3 expert
 *     GEMMs on one-block, CTA-pair or two-block tiles for every batch),
 *     MOE_GEMM1_TILE / MOE_GEMM2_TILE=single|dual (one GEMM's tile),
 *     MOE_GATHER=separate|fused (x rows gathered by their own kernel or by
 *     GEMM1), MOE_GEMM1_BAND_KB / MOE_GEMM2_BAND_KB (the tile order's band of
 *     A rows; 0: no bands), MOE_GRID_BALANCE=0, MOE_W4A4_TILE=128|256,
 *     MOE_W4A4_ROWS=32|128 and MOE_W4A16_ROWS=32|128.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols stay visible when the library is built with hidden
 * default visibility. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Same object as cudaStream_t; declared here so that this header needs no
 * CUDA header. */
typedef struct CUstream_st *moe_stream_t;

typedef struct moe_handle moe_handle;

typedef enum {
    MOE_F32 = 0,  /* fp32 x, w1, w3, w2, y: CUDA-core fp32 path */
    MOE_BF16 = 1  /* bf16 x, w1, w3, w2, y: tcgen05 tensor-core path */
} moe_dtype;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer, wrong device */
    MOE_ERR_UNSUPPORTED = 2, /* not an sm_100 device, or a path the handle's dtype lacks */
    MOE_ERR_ALLOC = 3,       /* workspace cudaMalloc failed */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed */
    MOE_ERR_TIMEOUT = 5      /* a kernel gave up a bounded wait (see moe_sync_status) */
} moe_status;

/*
 * Create a handle for a layer with n experts, K experts per token, model dim
 * d and expert hidden dim ffn.  Sources: the roles of n and K in section 2.1
 * of "Mixtral of Experts" (flash cards); the router nn.Linear(dim, n,
 * bias=False) quoted in Part 3 Step 1 of the neobadger page.
 *   Constraints: 1 <= K <= n <= 256; d and ffn multiples of 64 in [64, 65536];
 *   dtype MOE_F32 or MOE_BF16; out != NULL.
 *   Touches no GPU state (no allocation happens here).
 *   Errors: MOE_ERR_INVALID_ARG; *out is set to NULL on error.
 */
MOE_API moe_status moe_create(int n, int K, int d, int ffn, moe_dtype dtype, moe_handle **out);

/*
 * Allocate the workspace for up to T_max tokens on the current device, so
 * that later moe_forward calls with T <= T_max allocate nothing (needed before
 * capturing a CUDA graph, and outside timed loops).
 *   Errors: MOE_ERR_INVALID_ARG (null handle, T_max < 0, T_max * K > 2^31 - 1,
 *   handle bound to another device), MOE_ERR_UNSUPPORTED (device is not
 *   sm_100), MOE_ERR_ALLOC.
 */
MOE_API moe_status moe_reserve(moe_handle *h, int64_t T_max);

/*
 * The whole layer forward on T tokens: router logits x . W_g (fp32), top-K,
 * softmax over the K kept logits, dispatch of (token, slot) pairs into
 * per-expert segments, SwiGLU experts on those segments, gate-weighted
 * combine into y.  Sources: the layer equation (flash cards, section 2.1);
 * the three routing lines and Steps 1-4 of Part 3 of the neobadger page.
 *   T = 0 is a no-op returning MOE_OK.  Grows the workspace if T exceeds the
 *   reservation.  topk_idx and topk_w are outputs.
 *   Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_ALLOC, MOE_ERR_CUDA.
 */
MOE_API moe_status moe_forward(moe_handle *h, int64_t T, const void *x, const float *W_g,
                       const void *w1, const void *w3, const void *w2, void *y,
                       int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/*
 * Router only: logits x . W_g in fp32, the K largest (descending; ties to the
 * lower index), softmax over those K.  Sources: Steps 1-3 of Part 3 of the
 * neobadger page and the routing lines quoted there (gate, topk, softmax).
 *   Errors: as moe_forward.
 */
MOE_API moe_status moe_route(moe_handle *h, int64_t T, const void *x, const float *W_g,
                     int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/*
 * Dispatch only: group the T*K (token, slot) pairs of topk_idx into
 * per-expert segments, expert by expert, tokens ascending inside an expert
 * (experts whose gate is zero compute nothing, as the ainotis page reports of
 * the Mixtral paper; this is that rule laid out for grouped GEMMs).  Outputs
 * (device, int32):
 *   counts[n]          rows of each expert
 *   offsets[n+1]       first row of each expert's segment; offsets[n] = T*K
 *   row_token[T*K]     token of each row
 *   token_row[T][K]    row of each (token, slot) pair
 * Any output pointer may be NULL to skip it.  topk_idx values must lie in
 * [0, n) and be distinct within a token; out-of-range values are counted into
 * no segment and make the results unspecified (never an out-of-bounds access).
 *   Errors: as moe_forward.
 */
MOE_API moe_status moe_dispatch(moe_handle *h, int64_t T, const int32_t *topk_idx, int32_t *counts,
                        int32_t *offsets, int32_t *row_token, int32_t *token_row,
                        moe_stream_t stream);

/*
 * Experts and combine under a routing supplied by the caller:
 * y[t] = sum_k topk_w[t][k] * SwiGLU_{topk_idx[t][k]}(x[t]).  Source: the
 * gate-weighted additive combine of Step 4 (Part 3, neobadger page) and the
 * sum over experts in the layer equation.  topk_idx must hold distinct experts
 * per token in [0, n).
 *   Errors: as moe_forward.
 */
MOE_API moe_status moe_forward_with_routing(moe_handle *h, int64_t T, const void *x,
                                    const int32_t *topk_idx, const float *topk_w,
                                    const void *w1, const void *w3, const void *w2, void *y,
                                    moe_stream_t stream);

/*
 * Gate precision.  bf16 = 1: after the fp32 softmax, every topk_w is rounded to
 * bf16 (nearest even) and kept as an fp32 value, as the routing code quoted in
 * Part 3 of the neobadger page casts the weights to the inputs' dtype; the
 * combine then uses those gates.  bf16 = 0 (the default): fp32 gates.  Applies
 * to every later call that routes (moe_forward, moe_route and the
 * low-precision forwards).
 *   Errors: MOE_ERR_INVALID_ARG (null handle, bf16 not 0 or 1).
 */
MOE_API moe_status moe_set_gate_rounding(moe_handle *h, int bf16);

/*
 * Expert capacity (Part 5 of the neobadger page, "What happens when an expert
 * is full", after the Switch paper: capacity = tokens in the batch / experts x
 * a capacity factor).  With factor > 0, each later forward / dispatch call on
 * T tokens gives every expert at most C = ceil(factor * T * K / n) (token,
 * slot) pairs: the first C in dispatch order (tokens ascending) are kept, the
 * overflow pairs skip their expert and add nothing to y (the caller's residual
 * carries those tokens on), and moe_dispatch reports them with token_row = -1.
 * Gates are not renormalised.  factor = 0 (the default) is the dropless layer
 * of the layer equation.
 *   Errors: MOE_ERR_INVALID_ARG (null handle, factor < 0 or not finite).
 */
MOE_API moe_status moe_set_capacity_factor(moe_handle *h, double factor);

/*
 * Expert-choice routing: every expert chooses its own tokens, up to a fixed
 * capacity ("Mixtral of Experts? Mixture of Experts? Try to explain Mixtral
 * 8x7B", section "How Experts Are Chosen", item 2).  With the router
 * probabilities S[t][e] = softmax over the n experts of x_t . W_g (fp32):
 *   - expert e keeps the `capacity` tokens with the largest S[.][e] (equal
 *     probabilities keep the lower token index); sel_token[e][0..capacity)
 *     lists them in ascending token order and sel_gate[e][j] = S[token][e];
 *   - y[t] = sum over the experts that kept t, in expert order, of
 *     S[t][e] * SwiGLU_e(x_t); a token no expert kept gets y[t] = 0.
 * The handle's K is not used.  x, W_g, w1, w3, w2, y as for moe_forward;
 * sel_token [n][capacity] int32 and sel_gate [n][capacity] fp32 are device
 * outputs.  1 <= capacity <= T.  The workspace grows to n * capacity rows.
 *   Errors: as moe_forward.
 */
MOE_API moe_status moe_forward_expert_choice(moe_handle *h, int64_t T, int64_t capacity,
                                             const void *x, const float *W_g, const void *w1,
                                             const void *w3, const void *w2, void *y,
                                             int32_t *sel_token, float *sel_gate,
                                             moe_stream_t stream);

/*
 * Load-balancing statistics of a routing (Part 5 of the neobadger page, "Tool
 * 2: a fine for favouritism", the Switch Transformers loss):
 *   f[i]  = share of the T*K routed (token, slot) pairs of topk_idx sent to
 *           expert i (the share of tokens when K = 1);
 *   P[i]  = mean over the T tokens of the router probability of expert i, the
 *           softmax over all n logits x . W_g (fp32);
 *   aux[0] = alpha * n * sum_i f[i] * P[i]  (alpha: 0.01 in the Switch paper,
 *           0.02 in the Hugging Face Mixtral configuration).
 * x, W_g as for moe_forward; topk_idx [T][K] an input (e.g. from moe_route);
 * f, P (n floats) and aux (1 float) device outputs.  Sums run in a fixed order
 * (deterministic).
 *   Errors: MOE_ERR_INVALID_ARG (also T = 0, alpha not finite), as moe_forward.
 */
MOE_API moe_status moe_router_stats(moe_handle *h, int64_t T, const void *x, const float *W_g,
                                    const int32_t *topk_idx, float alpha, float *f, float *P,
                                    float *aux, moe_stream_t stream);

/*
 * FP8 expert weights.  Part 4 of "Mixture of Experts: Why Mixtral Only Wakes
 * Up Two Specialists" ("Why total and active both matter") sizes the weights at
 * 16 bits and at lower precision; the pages fix no format.  This library
 * stores them as E4M3 (OCP 8-bit floating point: exponent bias 7, largest
 * finite 448, no infinities) with one fp32 scale per output column:
 *   scale[e][c] = max_r |w[e][r][c]| / 448   (1 for an all-zero column)
 *   code[e][r][c] = E4M3(fp32(w[e][r][c] / scale[e][c])), round to nearest,
 *                   ties to even, saturating at +-448
 * so w ~= decode(code) * scale.
 *
 * moe_quantize_weights_e4m3: w [n][rows][cols] (MOE_BF16 or MOE_F32, device)
 * -> codes [n][rows][cols] (uint8, device) and scales [n][cols] (fp32, device).
 * For the layer: w1 and w3 are [n][d][ffn] (scales [n][ffn]), w2 is
 * [n][ffn][d] (scales [n][d]).  Needs no handle; enqueued on `stream`.
 *   Errors: MOE_ERR_INVALID_ARG (n outside [1, 65535], rows < 1, cols not a
 *   positive multiple of 16, n*rows*cols > 2^40, null / misaligned pointer),
 *   MOE_ERR_UNSUPPORTED (not an sm_100 device), MOE_ERR_CUDA.
 */
MOE_API moe_status moe_quantize_weights_e4m3(int n, int rows, int cols, const void *w, moe_dtype dtype,
                                             uint8_t *codes, float *scales, moe_stream_t stream);

/*
 * The layer of moe_forward with E4M3 experts (MOE_BF16 handles only): the same
 * fp32 router, top-K, softmax and dispatch (and capacity, if set); then per
 * dispatched (token, slot) row
 *   x8  = E4M3 codes of x_t with the row scale sx = max|x_t| / 448;
 *   h   = bf16( silu(sx * s1 (*) (x8 . q1_e)) (*) (sx * s3 (*) (x8 . q3_e)) );
 *   h8  = E4M3 codes of h with the row scale sh = max|h| / 448;
 *   o   = bf16( sh * s2 (*) (h8 . q2_e) ),   y_t = sum_k gate_k * o_k
 * with fp32 tensor-core accumulation of the 8-bit products.  w*_q / w*_s are
 * the codes and scales of moe_quantize_weights_e4m3; x, W_g, y, topk_idx,
 * topk_w as for moe_forward.  The first call grows the workspace by
 * T*K*(ffn + 8) bytes.
 *   Errors: as moe_forward; MOE_ERR_UNSUPPORTED for an fp32 handle.
 */
MOE_API moe_status moe_forward_e4m3(moe_handle *h, int64_t T, const void *x, const float *W_g,
                                    const uint8_t *w1_q, const float *w1_s, const uint8_t *w3_q,
                                    const float *w3_s, const uint8_t *w2_q, const float *w2_s, void *y,
                                    int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/*
 * 4-bit expert weights (Part 4 of "Mixture of Experts: Why Mixtral Only Wakes
 * Up Two Specialists" sizes the weights at 4 bits; the format is this
 * library's): E2M1 values (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) with an E4M3
 * scale per 16 consecutive reduction rows of one output column and an fp32
 * scale per expert matrix:
 *   st[e]     = max|w[e]| / (6 * 448)                (1 for an all-zero matrix)
 *   sb[e][b][c] = E4M3( fp32(max|w[e][16b..16b+15][c]| / 6) / st[e] )
 *   code      = E2M1( fp32(w / fp32(sb * st)) ), round to nearest even,
 *               saturating at +-6 (0 where sb is 0)
 *   w ~= E2M1(code) * sb * st
 *
 * moe_quantize_weights_fp4: w [n][rows][cols] (MOE_BF16 or MOE_F32, device)
 * -> codes [n][rows][cols/2] uint8 (column 2j in the low nibble of byte j,
 * 2j+1 in the high nibble), block_scales [n][rows/16][cols] uint8 (E4M3
 * codes), matrix_scales [n] fp32, all device memory.  For the layer: w1, w3
 * [n][d][ffn] and w2 [n][ffn][d].  Needs no handle; enqueued on `stream`.
 *   Errors: MOE_ERR_INVALID_ARG (n outside [1, 65535], rows not a positive
 *   multiple of 16, cols not a positive multiple of 32, null / misaligned
 *   pointer), MOE_ERR_UNSUPPORTED (not an sm_100 device), MOE_ERR_CUDA.
 */
MOE_API moe_status moe_quantize_weights_fp4(int n, int rows, int cols, const void *w, moe_dtype dtype,
                                            uint8_t *codes, uint8_t *block_scales, float *matrix_scales,
                                            moe_stream_t stream);

/*
 * The layer of moe_forward with 4-bit experts (MOE_BF16 handles only): the same
 * router, dispatch (and capacity) and gather; each expert GEMM runs on bf16
 * activations and the weights E2M1(code) * sb, which are exact in bf16, and
 * multiplies the fp32 accumulators by the matrix scale st:
 *   h = bf16( silu(st1 * x . W1) (*) (st3 * x . W3) ),  o = bf16( st2 * h . W2 )
 * so the result is the bf16 layer of the dequantised weights.  Codes and
 * scales as moe_quantize_weights_fp4 writes them; x, W_g, y, topk_idx, topk_w
 * as for moe_forward.
 *   Errors: as moe_forward; MOE_ERR_UNSUPPORTED for an fp32 handle.
 */
MOE_API moe_status moe_forward_fp4(moe_handle *h, int64_t T, const void *x, const float *W_g,
                                   const uint8_t *w1_codes, const uint8_t *w1_block_scales,
                                   const float *w1_matrix_scales, const uint8_t *w3_codes,
                                   const uint8_t *w3_block_scales, const float *w3_matrix_scales,
                                   const uint8_t *w2_codes, const uint8_t *w2_block_scales,
                                   const float *w2_matrix_scales, void *y, int32_t *topk_idx, float *topk_w,
                                   moe_stream_t stream);

/*
 * 4-bit weights AND 4-bit activations on the block-scaled tensor cores
 * (tcgen05.mma kind::mxf4nvf4, block 16).  The weights are those of
 * moe_quantize_weights_fp4, repacked once by moe_pack_weights_w4a4 into the
 * layout the tensor core reads.  A single matrix [n][rows][cols] becomes
 *   packed_codes [n][cols][rows/2]: row-contiguous (K-major) codes, rows 2j
 *                and 2j+1 of a column in the low / high nibble of byte j;
 *   scale_chunks [n][cols/128][rows/64][512] (bytes): for 128 columns and one
 *                64-row step, the 4 block scales of column c at byte
 *                16 * (c % 32) + 4 * ((c % 128) / 32) + s (s = 16-row block).
 * A gate/up pair (w1 and w3, pair_codes / pair_block_scales = w3's) becomes
 * one matrix of 2*cols packed columns: packed column p holds column
 * 64 * (p / 128) + p % 64 of w1 when p % 128 < 64, else the same column of w3,
 * so each 128-column block carries both projections of 64 hidden columns;
 * packed_codes is then [n][2*cols][rows/2] and scale_chunks
 * [n][2*cols/128][rows/64][512], laid out as above for packed columns.
 * Arguments: codes / block_scales (and the pair's) as moe_quantize_weights_fp4
 * writes them; rows a multiple of 64; cols a multiple of 128 (64 for a
 * pair); pair_codes and pair_block_scales both null for a single matrix.
 * Needs no handle; enqueued on `stream`; the caller owns every buffer.
 *   Errors: MOE_ERR_INVALID_ARG (sizes, null / misaligned pointer, one of the
 *   pair pointers null), MOE_ERR_UNSUPPORTED (not an sm_100 device),
 *   MOE_ERR_CUDA.
 */
MOE_API moe_status moe_pack_weights_w4a4(int n, int rows, int cols, const uint8_t *codes,
                                         const uint8_t *block_scales, const uint8_t *pair_codes,
                                         const uint8_t *pair_block_scales, uint8_t *packed_codes,
                                         uint8_t *scale_chunks, moe_stream_t stream);

/*
 * 4-bit weights with bf16 activations, the fast form (the weights at 4 bits
 * as Part 4 of "Mixture of Experts: Why Mixtral Only Wakes Up Two
 * Specialists" loads them; the layout is this library's).  The weights of
 * moe_quantize_weights_fp4 are repacked once so that the GEMMs can decode
 * them straight into tensor memory.  A matrix [n][rows][cols] becomes
 *   packed [n][cols/128][rows/64][4608] bytes: for 128 columns and one 64-row
 *   step, 4,096 bytes of codes as [2][128][16] (half h = rows 32h .. 32h+31 of
 *   the step; per column four 32-bit words of 8 rows each, the bits of each
 *   word arranged for the decoder: rows 2i and 2i+1 of the word come out of it
 *   as one bf16 pair after a rotation by 0, 4, 10 bits (i = 0, 1, 2) or by 6
 *   and 14 bits (i = 3) and a mask), then the 4 E4M3 block scales of each
 *   column ([128][4] bytes).
 * A gate/up pair (w1 with pair_codes / pair_block_scales = w3's) becomes one
 * matrix of 2*cols packed columns whose tile j holds columns 64j .. 64j+63 of
 * w1 and then the same columns of w3: packed [n][cols/64][rows/64][4608].
 * Arguments: codes / block_scales (and the pair's) as moe_quantize_weights_fp4
 * writes them; rows a multiple of 64; cols a multiple of 128 (64 for a pair).
 * Needs no handle; enqueued on `stream`; the caller owns every buffer.
 *   Errors: MOE_ERR_INVALID_ARG (sizes, null / misaligned pointer, one of the
 *   pair pointers null), MOE_ERR_UNSUPPORTED (not an sm_100 device),
 *   MOE_ERR_CUDA.
 */
MOE_API moe_status moe_pack_weights_w4a16(int n, int rows, int cols, const uint8_t *codes,
                                          const uint8_t *block_scales, const uint8_t *pair_codes,
                                          const uint8_t *pair_block_scales, uint8_t *packed,
                                          moe_stream_t stream);

/*
 * The layer of moe_forward_fp4 (4-bit weights, bf16 activations: the bf16 layer
 * of the dequantised weights E2M1(code) * sb, the accumulators multiplied by
 * the matrix scales) on the packed weights of moe_pack_weights_w4a16: the
 * GEMMs decode the codes straight into tensor memory, where the tensor core
 * reads them, so the 4-bit weights cost 0.56 bytes each from memory and no
 * shared-memory round trip.  MOE_BF16 handles with d a multiple of 128.
 * w13_packed: the gate/up pair pack of w1 and w3 (rows = d, cols = ffn);
 * w2_packed: w2 packed alone (rows = ffn, cols = d); w*_matrix_scales from
 * moe_quantize_weights_fp4; x, W_g, y, topk_idx, topk_w as for moe_forward.
 * The GEMMs take tokens in blocks of 32 rows when the experts average at most
 * 32 rows per call (T*K <= 32*n), else 128 (MOE_W4A16_ROWS=32 or 128 forces
 * one; same results either way).
 *   Errors: as moe_forward; MOE_ERR_UNSUPPORTED for an fp32 handle or d not a
 *   multiple of 128.
 */
MOE_API moe_status moe_forward_w4a16(moe_handle *h, int64_t T, const void *x, const float *W_g,
                                     const uint8_t *w13_packed, const float *w1_matrix_scales,
                                     const float *w3_matrix_scales, const uint8_t *w2_packed,
                                     const float *w2_matrix_scales, void *y, int32_t *topk_idx,
                                     float *topk_w, moe_stream_t stream);

/*
 * The layer with 4-bit weights and 4-bit activations (MOE_BF16 handles with d
 * and ffn multiples of 256): the router, dispatch and capacity of moe_forward;
 * every gathered x row and every hidden row is quantised like a weight matrix
 * whose blocks run along the row (an fp32 scale max|row| / (6 * 448), E4M3
 * scales per 16 elements, E2M1 codes); the tensor core multiplies the codes
 * with their block scales and accumulates in fp32; the row and matrix scales
 * are applied to the accumulators:
 *   h = bf16( silu(rx st1 (Xq . W1q)) (*) (rx st3 (Xq . W3q)) ),
 *   o = bf16( rh st2 (Hq . W2q) ),   y_t = sum_k gate_k * o_k
 * w13_packed / w13_chunks: the gate/up pair pack of moe_pack_weights_w4a4
 * (w1 and w3, rows = d, cols = ffn); w2_packed / w2_chunks: w2 packed alone
 * (rows = ffn, cols = d); w*_matrix_scales from moe_quantize_weights_fp4;
 * x, W_g, y, topk_idx, topk_w as for moe_forward.  The GEMMs use tiles of
 * 256 packed columns, over 32 rows when the experts average at most 32 rows
 * per call (T*K <= 32*n) and over 128 rows otherwise; MOE_W4A4_TILE=128
 * selects 128-column tiles with two accumulators (the same row rule),
 * MOE_W4A4_ROWS=32 or 128 forces the row tiles (same results either way).
 * The first call grows the workspace by about T*K*(d + ffn)*0.6 bytes.
 *   Errors: as moe_forward; MOE_ERR_UNSUPPORTED for an fp32 handle or d, ffn
 *   not multiples of 256.
 */
MOE_API moe_status moe_forward_w4a4(moe_handle *h, int64_t T, const void *x, const float *W_g,
                                    const uint8_t *w13_packed, const uint8_t *w13_chunks,
                                    const float *w1_matrix_scales, const float *w3_matrix_scales,
                                    const uint8_t *w2_packed, const uint8_t *w2_chunks,
                                    const float *w2_matrix_scales, void *y, int32_t *topk_idx, float *topk_w,
                                    moe_stream_t stream);

/*
 * Expert parallelism over `world` ranks (1 <= world <= 16, world divides n):
 * rank q holds the weights of experts [q*n/world, (q+1)*n/world) and routes
 * its own tokens.  The flash-card page on "Mixtral of Experts" names this
 * placement (section 2.1: experts on different GPUs, uneven routing
 * overloading some of them; section 5: temporal locality); the pages give
 * no mechanics, so the exchange below is this library's design.  The two
 * all-to-all exchanges are fused into the kernels around them: the dispatch
 * STORES each routed x row into its expert owner's receive buffer, and the
 * combine LOADS each expert output row from its owner's output buffer.  Peer
 * buffers are device pointers the calling process can dereference (another
 * GPU's memory mapped through CUDA IPC with peer access, or, for ranks
 * emulated on one GPU, plain device memory).  Expert parallelism is dropless
 * (MOE_ERR_UNSUPPORTED while a capacity factor is set) and needs a MOE_BF16
 * handle created with the GLOBAL n.  One layer step on every rank:
 *   1. moe_route, then moe_dispatch(..., counts, ...) for this rank's counts[n];
 *   2. counts_all[world][n] = every rank's counts (row q = rank q's), on the
 *      device of every rank (e.g. an all-gather);
 *   3. moe_ep_dispatch;  4. a barrier across ranks;
 *   5. moe_ep_experts;   6. a barrier across ranks;   7. moe_ep_combine.
 * Receive layout on an owner: its experts in order; inside an expert the rows
 * of rank 0, then rank 1, ...; inside a rank its (token, slot) pairs of that
 * expert in token order.  An owner receives sum over ranks and over its
 * experts of counts_all rows; recv_rows (the rows every receive buffer holds,
 * the same on all ranks) must cover that, else moe_sync_status reports
 * MOE_ERR_INVALID_ARG and nothing is stored.  The y of a token is computed as
 * moe_forward_with_routing computes it (same kernels, same order), so with the
 * same routing the two agree bit for bit.
 *
 * moe_ep_dispatch: x [T][d], topk_idx [T][K] of this rank (device);
 * counts_all [world][n] int32 (device); recv_buffers: host array of `world`
 * device pointers, entry q = rank q's receive buffer [recv_rows][d] bf16;
 * row_pos [T][K] int32 (device, written): the row of each (token, slot) pair
 * inside its owner's buffer.  Also checks counts_all's row `rank` against
 * this rank's routing.
 */
MOE_API moe_status moe_ep_dispatch(moe_handle *h, int world, int rank, int64_t T, const void *x,
                                   const int32_t *topk_idx, const int32_t *counts_all,
                                   void *const *recv_buffers, int64_t recv_rows, int32_t *row_pos,
                                   moe_stream_t stream);

/*
 * moe_ep_experts: the grouped SwiGLU experts of rank `rank` over its receive
 * buffer recv [recv_rows][d] (filled by every rank's moe_ep_dispatch), with
 * its local weights w1, w3 [n/world][d][ffn] and w2 [n/world][ffn][d] (bf16);
 * out [recv_rows][d] bf16 receives the expert output of every received row,
 * in the receive layout.  The workspace grows to recv_rows rows.
 */
MOE_API moe_status moe_ep_experts(moe_handle *h, int world, int rank, const int32_t *counts_all,
                                  const void *recv, int64_t recv_rows, const void *w1, const void *w3,
                                  const void *w2, void *out, moe_stream_t stream);

/*
 * moe_ep_combine: y[t] = sum_k topk_w[t][k] * out_{owner}[row_pos[t][k]],
 * fp32 in slot order, rounded to bf16; out_buffers: host array of `world`
 * device pointers, entry q = rank q's `out` of moe_ep_experts.  Pairs with
 * row_pos < 0 add nothing.
 *   Errors (all three): MOE_ERR_INVALID_ARG (world, rank, n not divisible,
 *   null / misaligned pointer, recv_rows outside [1, 2^31 - 1]);
 *   MOE_ERR_UNSUPPORTED (fp32 handle, capacity factor set); MOE_ERR_CUDA.
 */
MOE_API moe_status moe_ep_combine(moe_handle *h, int world, int64_t T, const int32_t *topk_idx,
                                  const float *topk_w, const int32_t *row_pos, const void *const *out_buffers,
                                  void *y, moe_stream_t stream);

/*
 * Buffers that other ranks' kernels read or write (the receive and output
 * buffers of expert parallelism): moe_ep_buffer_alloc allocates `bytes` of
 * device memory on the current device (cudaMalloc: the base of its own
 * allocation) and, when ipc_handle is not NULL, writes its 64-byte CUDA IPC
 * handle there for the other processes; moe_ep_buffer_open maps another
 * process's buffer from its handle (peer access enabled); moe_ep_buffer_close
 * releases one (opened = 1 for a mapped peer buffer, 0 for an own buffer).
 *   Errors: MOE_ERR_INVALID_ARG (null pointers, bytes < 1), MOE_ERR_ALLOC,
 *   MOE_ERR_CUDA.
 */
MOE_API moe_status moe_ep_buffer_alloc(int64_t bytes, void **ptr, uint8_t *ipc_handle);
MOE_API moe_status moe_ep_buffer_open(const uint8_t *ipc_handle, void **ptr);
MOE_API moe_status moe_ep_buffer_close(void *ptr, int opened);

/*
 * Debug view of the workspace written by the last forward call: name is "H"
 * (expert hidden layer, [rows][ffn], handle dtype) or "O" (per-row expert
 * outputs, [rows][d], handle dtype for bf16 handles, fp32 for fp32 handles);
 * after moe_forward_e4m3 also "X8" (E4M3 codes of the gathered x rows,
 * [rows][d] uint8), "XS" (their scales, [rows] fp32), "H8" (codes of H,
 * [rows][ffn] uint8) and "HS" ([rows] fp32).  Returns the device pointer and
 * the row capacity; rows are in dispatch order.
 *   Errors: MOE_ERR_INVALID_ARG (unknown name, null argument, no workspace yet).
 */
MOE_API moe_status moe_workspace_view(moe_handle *h, const char *name, void **ptr, int64_t *rows);

/*
 * Wait for `stream`, then report whether any kernel of this handle gave up a
 * bounded wait since the last call (MOE_ERR_TIMEOUT; the flag is cleared) or a
 * CUDA error is pending (MOE_ERR_CUDA).
 */
MOE_API moe_status moe_sync_status(moe_handle *h, moe_stream_t stream);

/*
 * Per-stage timing with CUDA events, for profiling.  After moe_trace_begin(h,
 * max_calls) each of the next max_calls moe_forward / moe_forward_with_routing
 * calls records events around its stages on its stream:
 *   stage 0 router, 1 dispatch (rank, scan, scatter), 2 gather (or the x-row
 *   quantisation of the 8- and 4-bit forms), 3 GEMM1 (w1/w3 + SwiGLU), 4 GEMM2
 *   (w2; with the H-row quantisation first in the 8- and 4-bit-activation
 *   forms), 5 combine
 * (stage 0 is 0 ms for moe_forward_with_routing).  moe_trace_end waits for the
 * recorded events, writes the summed milliseconds of each stage into
 * stage_ms[0 .. n_stages-1] (n_stages <= 6), the number of traced calls into
 * *calls, and stops tracing.  Calls beyond max_calls are not traced.
 *   Errors: MOE_ERR_INVALID_ARG (null handle or output, max_calls < 1 or
 *   > 100000, end without begin), MOE_ERR_CUDA.
 */
MOE_API moe_status moe_trace_begin(moe_handle *h, int max_calls);
MOE_API moe_status moe_trace_end(moe_handle *h, double *stage_ms, int n_stages, int *calls);

/*
 * Dispatch for callers that cannot allocate device memory.  The pages have no
 * counterpart: this is an interface convenience of this library.
 *
 * Same outputs as moe_dispatch (counts[n], offsets[n+1], row_token[T*K],
 * token_row[T][K], all caller-owned device int32, all required here), but no
 * handle and no cudaMalloc / cudaFree: the scratch lives in a fixed device
 * array inside the library (about 0.5 MB, held on every GPU that loads the
 * library until the process exits).  Meant for callers whose device memory
 * comes from a framework allocator or a fixed memory plan, and for callers
 * that cannot take cudaMalloc's implicit device-wide synchronisation.
 *   Limit: T * K <= 65,536 pairs, n <= 256; larger sizes return
 *   MOE_ERR_INVALID_ARG with a message naming the limit.
 *   Every call looks up the array's device address (cudaGetSymbolAddress)
 *   on the current device.  The first lookup on a device may load the
 *   library's module there, so make the first call on each device before any
 *   stream capture.
 *   Every call shares the array and it keeps the last call's contents (each
 *   call overwrites what it reads).  Calls that overlap on the GPU race on
 *   it: order them on one stream.
 *   Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA.
 */
MOE_API moe_status moe_dispatch_noalloc(int64_t T, int n, int K, const int32_t *topk_idx,
                                        int32_t *counts, int32_t *offsets, int32_t *row_token,
                                        int32_t *token_row, moe_stream_t stream);

/*
 * Self-test of failure detection (the pages have no counterpart).  Launches
 * one kernel whose bounded wait -- the same helper every pipelined kernel of
 * this library waits through -- is on a barrier nothing ever completes, with
 * a budget of budget_us microseconds.  The wait gives up, sets the handle's
 * status flag and the kernel returns normally; the next moe_sync_status then
 * returns MOE_ERR_TIMEOUT and clears the flag.  Nothing faults or hangs, and
 * the context stays usable.
 *   Errors: MOE_ERR_INVALID_ARG (null handle, budget_us outside [1, 10^6]),
 *   MOE_ERR_UNSUPPORTED, MOE_ERR_ALLOC, MOE_ERR_CUDA.
 */
MOE_API moe_status moe_selftest_timeout(moe_handle *h, int budget_us, moe_stream_t stream);

/* Number of CUDA kernels this handle has launched so far (all entry points). */
MOE_API moe_status moe_launch_count(moe_handle *h, int64_t *count);

/* Free the workspace and the handle.  NULL is allowed. */
MOE_API moe_status moe_destroy(moe_handle *h);

/* Message for the last failing call on this host thread ("" if none). */
MOE_API const char *moe_last_error(void);

/* Library version string. */
MOE_API const char *moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
