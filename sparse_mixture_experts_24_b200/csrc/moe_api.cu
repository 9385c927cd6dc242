// moe_api.cu -- the C ABI declared in include/moe.h: argument checking, the
// workspace, TMA tensor maps, and the launch sequence of the layer forward
//   router -> dispatch (rank, scan, scatter) -> gather -> GEMM1 -> GEMM2 -> combine
// all on the caller's stream with no host synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <new>
#include <vector>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

moe_status fail(moe_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

moe_status ok() {
    g_err[0] = '\0';
    return MOE_OK;
}

}  // namespace

namespace moe {
thread_local bool g_chain_started = false;
bool pdl_enabled() {
    static const bool on = [] {
        const char* e = getenv("MOE_PDL");
        return !(e && strcmp(e, "0") == 0);
    }();
    return on;
}
}  // namespace moe

namespace moe_api_detail {
// Lets other translation units of the library set the moe_last_error() text.
void set_last_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }
}  // namespace moe_api_detail

namespace {

moe_status cuda_fail(cudaError_t e, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// cuTensorMapEncodeTiled, fetched through the runtime so the library does not
// link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// bf16 row-major [rows][cols] operand read in box_rows x 64 (cols) boxes.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                 uint32_t box_rows = 128) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 weights [n][rows][cols] read in 64 (rows) x 64 (cols) boxes of one expert.
bool encode_weights(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t n) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {cols, rows, n};
    cuuint64_t strides[2] = {cols * 2, cols * rows * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 rows [rows][cols] as a 3-D map (64 columns, rows, 64-column chunk)
// read in boxes of 64 columns x box_rows rows x `chunks` chunks: one copy
// lands `chunks` row tiles of box_rows x 64, back to back.
bool encode_rows_chunked(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
                         uint32_t chunks) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, chunks};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 weights [n][rows][cols] as a 4-D map (64 columns, rows, 64-column
// chunk, expert) read in boxes of 64 columns x 64 rows x `chunks` chunks:
// one copy lands `chunks` 64-column chunks of 8 KB each, back to back.
bool encode_weights_wide(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t n,
                         uint32_t chunks) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[4] = {64, rows, cols / 64, n};
    cuuint64_t strides[3] = {cols * 2, 128, cols * rows * 2};
    cuuint32_t box[4] = {64, 64, chunks, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 codes, uint8: [rows][cols] (box_rows x 128) or weights [n][rows][cols]
// (128 x 128 boxes of one expert); out-of-range boxes read zeros.
bool encode_codes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t n,
                  uint32_t box_rows = 128) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {cols, rows, n};
    cuuint64_t strides[2] = {cols, cols * rows};
    cuuint32_t box[3] = {128, box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, n ? 3 : 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-bit weight codes [n][rows][cols/2] read in 64-byte x 64-row boxes, and
// their block scales [n][rows/16][cols] in 128 x 4 boxes; no swizzle (the
// kernel's converter warps read them).
bool encode_fp4_codes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t n) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {cols / 2, rows, n};
    cuuint64_t strides[2] = {cols / 2, cols / 2 * rows};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_fp4_scales(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t n) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[3] = {cols, rows / 16, n};
    cuuint64_t strides[2] = {cols, cols * (rows / 16)};
    cuuint32_t box[3] = {128, 4, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

struct moe_handle {
    int n, K, d, F;
    moe_dtype dtype;
    int device = -1;
    int num_sms = 0;
    int64_t T_cap = 0;  // tokens the workspace holds
    int64_t R_cap = 0;  // expert rows (Xp, H, O) the workspace holds
    void* ws = nullptr;
    size_t ws_bytes = 0;
    moe::DispatchBufs db{};
    float* logits = nullptr;
    void* xp = nullptr;
    void* h = nullptr;
    void* o = nullptr;
    int* status = nullptr;
    CUtensorMap tm_xp, tm_h, tm_w1, tm_w3, tm_w2;
    CUtensorMap tm_w1x, tm_w3x, tm_w2x;  // the same weights as 4-D maps (single-SM GEMMs)
    CUtensorMap tm_w2p;                  // w2 as a 4-D map of two-chunk boxes (CTA-pair GEMM2)
    const void* c_w1 = nullptr;
    const void* c_w3 = nullptr;
    const void* c_w2 = nullptr;
    // tensor-core router: W_g split parts and the maps over x and the parts
    uint16_t* wg_parts = nullptr;
    CUtensorMap tm_rx, tm_parts;
    const void* c_rx = nullptr;
    int64_t c_rx_T = -1;
    // expert parallelism: plan arrays (workspace), and tensor maps of the
    // receive buffer and the local experts' weights
    int32_t* ep_dst = nullptr;    // [n]
    int32_t* ep_loff = nullptr;   // [n+1]
    int32_t* ep_lmblk = nullptr;  // [n+1]
    CUtensorMap tm_erecv, tm_ew1, tm_ew3, tm_ew2;
    const void* c_erecv = nullptr;
    int64_t c_erecv_rows = -1;
    const void* c_ew[3] = {nullptr, nullptr, nullptr};
    int c_ew_nl = 0;
    // expert capacity factor (0: dropless) and load-balancing statistics scratch
    double capacity_factor = 0.0;
    bool gates_bf16 = false;  // moe_set_gate_rounding
    // kernels this handle has launched (for profiling and launch accounting)
    int64_t launches = 0;
    float* stats_partial = nullptr;
    int32_t* stats_counts = nullptr;
    // expert-choice routing: probabilities [n][T], row of (token, expert) [T][n]
    float* ec_probs = nullptr;
    int32_t* ec_rowmap = nullptr;
    // E4M3 experts: the workspace also holds x8 (in the Xp buffer), h8 and the
    // row scales once a call has asked for them
    bool want_e4m3 = false;
    bool has_e4m3 = false;
    uint8_t* x8 = nullptr;
    uint8_t* h8 = nullptr;
    float* xs = nullptr;
    float* hs = nullptr;
    CUtensorMap tm_x8, tm_h8, tm_q1, tm_q3, tm_q2;
    const void* c_q1 = nullptr;
    const void* c_q3 = nullptr;
    const void* c_q2 = nullptr;
    // 4-bit weights and activations: codes of the gathered x rows and of H,
    // their row scales and scale chunks (allocated once a call asks for them)
    bool want_w4a4 = false;
    bool has_w4a4 = false;
    uint8_t* xq4 = nullptr;
    uint8_t* hq4 = nullptr;
    uint8_t* xc4 = nullptr;
    uint8_t* hc4 = nullptr;
    float* xr4 = nullptr;
    float* hr4 = nullptr;
    CUtensorMap tm_xq4, tm_hq4, tm_wp4[2];
    CUtensorMap tm_xq4s, tm_hq4s;  // the same codes in 32-row boxes
    const void* c_wp4[2] = {nullptr, nullptr};
    int c_wp4_rows[2] = {0, 0};  // box rows the cached maps were encoded with
    // 4-bit weights decoded into tensor memory: Xp and H as 3-D maps whose
    // boxes hold 4 chunks of 32 rows ([0]) or 2 chunks of 128 rows ([1])
    CUtensorMap tm_xpw[2], tm_hw[2];
    // 4-bit experts: maps over the caller's codes and block scales
    CUtensorMap tm_f4[6];  // codes w1, scales w1, codes w3, scales w3, codes w2, scales w2
    const void* c_f4[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    // tracing: kTraceEvents events per traced call
    std::vector<cudaEvent_t> trace_ev;
    int trace_max = 0;
    int trace_calls = 0;
    bool tracing = false;

    size_t esize() const { return dtype == MOE_BF16 ? 2 : 4; }
    size_t osize() const { return dtype == MOE_BF16 ? 2 : 4; }
};

namespace {

constexpr int kTraceStages = 6;
constexpr int kTraceEvents = kTraceStages + 1;

// Event that closes `stage` of the current traced call (stage -1 = the start),
// or nullptr when this call is not traced.
cudaEvent_t trace_event(moe_handle* h, int stage) {
    if (!h->tracing || h->trace_calls >= h->trace_max) return nullptr;
    return h->trace_ev[static_cast<size_t>(h->trace_calls) * kTraceEvents + (stage + 1)];
}

void trace_mark(moe_handle* h, int stage, cudaStream_t st) {
    cudaEvent_t e = trace_event(h, stage);
    if (e) cudaEventRecord(e, st);
}

void trace_finish_call(moe_handle* h) {
    if (h->tracing && h->trace_calls < h->trace_max) ++h->trace_calls;
}

void trace_free(moe_handle* h) {
    for (cudaEvent_t e : h->trace_ev) cudaEventDestroy(e);
    h->trace_ev.clear();
    h->tracing = false;
    h->trace_max = h->trace_calls = 0;
}

moe_status check_device(moe_handle* h) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (h->device < 0) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        if (major != 10 || minor != 0)
            return fail(MOE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                        dev, major, minor);
        h->device = dev;
        h->num_sms = sms;
    } else if (dev != h->device) {
        return fail(MOE_ERR_INVALID_ARG, "handle belongs to device %d, current device is %d",
                    h->device, dev);
    }
    return MOE_OK;
}

// Workspace for T tokens and at least rows_min expert rows (T*K for
// token-choice calls, n*C for expert-choice calls).  Capacities only grow.
moe_status grow(moe_handle* h, int64_t T, int64_t rows_min = 0) {
    const int64_t R_need = std::max(T * h->K, rows_min);
    if (h->ws && T <= h->T_cap && R_need <= h->R_cap && (h->has_e4m3 || !h->want_e4m3) &&
        (h->has_w4a4 || !h->want_w4a4))
        return MOE_OK;
    T = std::max(T, h->T_cap);
    const int64_t R = std::max(std::max(R_need, h->R_cap), T * h->K);
    const int64_t nblk = (R + moe::kPairsPerBlock - 1) / moe::kPairsPerBlock;
    const size_t A = 256;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + (bytes ? bytes : 1), A);
        return o;
    };
    const size_t o_blockcounts = take(static_cast<size_t>(nblk) * h->n * 4);
    const size_t o_pair_rank = take(static_cast<size_t>(R) * 4);
    const size_t o_counts = take(static_cast<size_t>(h->n) * 4);
    const size_t o_offsets = take(static_cast<size_t>(h->n + 1) * 4);
    const size_t o_mblk = take(static_cast<size_t>(h->n + 1) * 4);
    const size_t o_row_token = take(static_cast<size_t>(R) * 4);
    const size_t o_token_row = take(static_cast<size_t>(R) * 4);
    const bool bf = h->dtype == MOE_BF16;
    const int npad = (h->n + 15) / 16 * 16;
    const size_t o_logits = take(static_cast<size_t>(moe::kRouterMaxSplits) * T * h->n * 4);
    const size_t o_stats_partial = take(static_cast<size_t>((T + 255) / 256) * h->n * 4);
    const size_t o_stats_counts = take(static_cast<size_t>(h->n) * 4);
    const size_t o_parts = take(bf ? static_cast<size_t>(3) * npad * h->d * 2 : 0);
    const size_t o_status = take(64);
    const size_t o_ep = take(static_cast<size_t>(3 * h->n + 2) * 4);
    const size_t o_ec_probs = take(static_cast<size_t>(T) * h->n * 4);
    const size_t o_ec_rowmap = take(static_cast<size_t>(T) * h->n * 4);
    const size_t o_xp = take(static_cast<size_t>(R) * h->d * h->esize());
    const size_t o_h = take(static_cast<size_t>(R) * h->F * h->esize());
    const size_t o_o = take(static_cast<size_t>(R) * h->d * h->osize());
    const bool e4 = h->want_e4m3;
    const size_t o_h8 = take(e4 ? static_cast<size_t>(R) * h->F : 0);
    const size_t o_xs = take(e4 ? static_cast<size_t>(R) * 4 : 0);
    const size_t o_hs = take(e4 ? static_cast<size_t>(R) * 4 : 0);
    const bool w4 = h->want_w4a4;
    const size_t tiles4 = static_cast<size_t>((R + 31) / 32 + h->n);  // 32-row tiles at most
    const size_t o_xq4 = take(w4 ? static_cast<size_t>(R) * (h->d / 2) : 0);
    const size_t o_hq4 = take(w4 ? static_cast<size_t>(R) * (h->F / 2) : 0);
    const size_t o_xc4 = take(w4 ? tiles4 * (h->d / 64) * 512 : 0);
    const size_t o_hc4 = take(w4 ? tiles4 * (h->F / 64) * 512 : 0);
    const size_t o_xr4 = take(w4 ? static_cast<size_t>(R) * 4 : 0);
    const size_t o_hr4 = take(w4 ? static_cast<size_t>(R) * 4 : 0);
    const size_t total = off;

    if (h->ws) {
        cudaFree(h->ws);
        h->ws = nullptr;
        h->T_cap = 0;
        h->R_cap = 0;
    }
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, total);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MOE_ERR_ALLOC, "cudaMalloc(%zu bytes) for the workspace failed: %s", total,
                    cudaGetErrorString(e));
    }
    e = cudaMemset(p, 0, total);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e, "cudaMemset(workspace)");
    }
    uint8_t* b = static_cast<uint8_t*>(p);
    h->ws = p;
    h->ws_bytes = total;
    h->T_cap = T;
    h->R_cap = R;
    h->ec_probs = reinterpret_cast<float*>(b + o_ec_probs);
    h->ec_rowmap = reinterpret_cast<int32_t*>(b + o_ec_rowmap);
    h->db.blockcounts = reinterpret_cast<int32_t*>(b + o_blockcounts);
    h->db.pair_rank = reinterpret_cast<int32_t*>(b + o_pair_rank);
    h->db.counts = reinterpret_cast<int32_t*>(b + o_counts);
    h->db.offsets = reinterpret_cast<int32_t*>(b + o_offsets);
    h->db.mblk_base = reinterpret_cast<int32_t*>(b + o_mblk);
    h->db.row_token = reinterpret_cast<int32_t*>(b + o_row_token);
    h->db.token_row = reinterpret_cast<int32_t*>(b + o_token_row);
    h->logits = reinterpret_cast<float*>(b + o_logits);
    h->wg_parts = reinterpret_cast<uint16_t*>(b + o_parts);
    h->stats_partial = reinterpret_cast<float*>(b + o_stats_partial);
    h->stats_counts = reinterpret_cast<int32_t*>(b + o_stats_counts);
    h->c_rx = nullptr;
    h->status = reinterpret_cast<int*>(b + o_status);
    h->ep_dst = reinterpret_cast<int32_t*>(b + o_ep);
    h->ep_loff = h->ep_dst + h->n;
    h->ep_lmblk = h->ep_loff + h->n + 1;
    h->c_erecv = nullptr;
    h->xp = b + o_xp;
    h->h = b + o_h;
    h->o = b + o_o;
    h->has_e4m3 = e4;
    h->x8 = e4 ? static_cast<uint8_t*>(h->xp) : nullptr;
    h->h8 = e4 ? b + o_h8 : nullptr;
    h->xs = e4 ? reinterpret_cast<float*>(b + o_xs) : nullptr;
    h->hs = e4 ? reinterpret_cast<float*>(b + o_hs) : nullptr;
    h->has_w4a4 = w4;
    h->xq4 = w4 ? b + o_xq4 : nullptr;
    h->hq4 = w4 ? b + o_hq4 : nullptr;
    h->xc4 = w4 ? b + o_xc4 : nullptr;
    h->hc4 = w4 ? b + o_hc4 : nullptr;
    h->xr4 = w4 ? reinterpret_cast<float*>(b + o_xr4) : nullptr;
    h->hr4 = w4 ? reinterpret_cast<float*>(b + o_hr4) : nullptr;
    // 4-bit codes: two per byte, so a row of d codes is d / 2 bytes wide
    if (w4 && (!encode_codes(&h->tm_xq4, h->xq4, h->d / 2, static_cast<uint64_t>(R), 0) ||
               !encode_codes(&h->tm_hq4, h->hq4, h->F / 2, static_cast<uint64_t>(R), 0) ||
               !encode_codes(&h->tm_xq4s, h->xq4, h->d / 2, static_cast<uint64_t>(R), 0, 32) ||
               !encode_codes(&h->tm_hq4s, h->hq4, h->F / 2, static_cast<uint64_t>(R), 0, 32)))
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the 4-bit workspace");
    if (e4 && (!encode_codes(&h->tm_x8, h->x8, h->d, static_cast<uint64_t>(R), 0) ||
               !encode_codes(&h->tm_h8, h->h8, h->F, static_cast<uint64_t>(R), 0)))
        return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the E4M3 workspace");
    if (h->dtype == MOE_BF16) {
        if (!encode_rows(&h->tm_xp, h->xp, h->d, static_cast<uint64_t>(R)) ||
            !encode_rows(&h->tm_h, h->h, h->F, static_cast<uint64_t>(R)) ||
            !encode_rows_chunked(&h->tm_xpw[0], h->xp, h->d, static_cast<uint64_t>(R), 32, 4) ||
            !encode_rows_chunked(&h->tm_hw[0], h->h, h->F, static_cast<uint64_t>(R), 32, 4) ||
            !encode_rows_chunked(&h->tm_xpw[1], h->xp, h->d, static_cast<uint64_t>(R), 128, 2) ||
            !encode_rows_chunked(&h->tm_hw[1], h->h, h->F, static_cast<uint64_t>(R), 128, 2) ||
            !encode_rows(&h->tm_parts, h->wg_parts, h->d, static_cast<uint64_t>(3 * npad),
                         static_cast<uint32_t>(npad)))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the workspace");
    }
    return MOE_OK;
}

moe_status check_common(moe_handle* h, int64_t T) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %lld < 0", static_cast<long long>(T));
    if (T > 0 && T * h->K > 2147483647LL)
        return fail(MOE_ERR_INVALID_ARG, "T * K = %lld exceeds 2^31 - 1",
                    static_cast<long long>(T * h->K));
    return MOE_OK;
}

#define REQUIRE_PTR(p)                                                                        \
    do {                                                                                      \
        if (!(p)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #p);                         \
        if (!aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p); \
    } while (0)

moe_status prepare(moe_handle* h, int64_t T, int64_t rows_min = 0) {
    moe_status s = check_device(h);
    if (s != MOE_OK) return s;
    return grow(h, T, rows_min);
}

// Router: the tensor-core path (bf16 x, enough tokens or many experts) or the
// CUDA-core kernels.
moe_status run_router(moe_handle* h, int64_t T, const void* x, const float* W_g, int32_t* topk_idx,
                      float* topk_w, cudaStream_t st) {
    cudaError_t e;
    if (h->dtype == MOE_BF16 && (T >= 512 || h->n > 32)) {
        if (x != h->c_rx || T != h->c_rx_T) {
            if (!encode_rows(&h->tm_rx, x, h->d, static_cast<uint64_t>(T)))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
            h->c_rx = x;
            h->c_rx_T = T;
        }
        e = moe::launch_router_tc(h->tm_rx, h->tm_parts, W_g, h->wg_parts, T, h->d, h->n, h->K,
                                  h->logits, topk_idx, topk_w, h->status, h->num_sms, st);
        h->launches += moe::router_tc_launches(h->K);
    } else {
        e = moe::launch_router(x, h->dtype == MOE_BF16, W_g, T, h->d, h->n, h->K, topk_idx, topk_w,
                               h->logits, h->num_sms, st);
        h->launches += h->n > 32 ? 2 : 1;
    }
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    if (h->gates_bf16) {
        e = moe::launch_gates_to_bf16(topk_w, T * h->K, h->num_sms, st);
        if (e != cudaSuccess) return cuda_fail(e, "gate rounding launch");
        h->launches += 1;
    }
    return MOE_OK;
}

// GEMM tiling: single-SM 128-row tiles (default) or CTA-pair 256-row tiles
// (MOE_GEMM_PATH=pair).  On the Mixtral prefill shapes the pair tiles halve
// the shared-memory operand traffic but measured no faster (tensor pipe ~80%
// busy either way), so the single-SM kernel stays the default.
bool use_pair_gemm(const moe_handle* h, int64_t T) {
    (void)T;
    if (h->dtype != MOE_BF16) return false;
    const char* env = getenv("MOE_GEMM_PATH");
    return env && strcmp(env, "pair") == 0;
}

// E4M3 GEMM tiling: the same switch (MOE_GEMM_PATH=pair selects CTA pairs).
bool use_pair_gemm_e4m3(const moe_handle* h, int64_t T) {
    const char* env = getenv("MOE_GEMM_PATH");
    if (env && strcmp(env, "single") == 0) return false;
    if (env && strcmp(env, "pair") == 0) return true;
    (void)h;
    (void)T;
    return false;
}

// Persistent GEMMs spread their tiles over the fewest CTAs that need no more
// rounds than the whole grid (every working CTA the same number of tiles)
// unless MOE_GRID_BALANCE=0.
int grid_balance() {
    const char* env = getenv("MOE_GRID_BALANCE");
    return (env && strcmp(env, "0") == 0) ? 0 : 1;
}

// Tile order of the single-SM GEMMs (gemm_tc.cu): bands of as many 128-row
// blocks of the A operand (rows of a_row_bytes) as fit in the band budget.
// The budget is 32 MB for GEMM1 (measured best on the skewed prefill, against
// 16, 40, 48 and 64 MB) and 40 MB for GEMM2 (against 24 and 32 MB: GEMM2 3.08
// against 3.13-3.19 ms there, 5.68 against 5.82 GB of DRAM traffic);
// MOE_GEMM1_BAND_KB / MOE_GEMM2_BAND_KB override them in kilobytes (0: no bands).
void gemm_tile_order(moe::TcGemmArgs& a, int64_t a_row_bytes, bool gemm2) {
    int64_t kb = gemm2 ? 40 * 1024 : 32 * 1024;
    if (const char* v = getenv(gemm2 ? "MOE_GEMM2_BAND_KB" : "MOE_GEMM1_BAND_KB")) kb = atoll(v);
    if (kb <= 0) {
        a.band_m = 0;
        return;
    }
    const int64_t b = (kb << 10) / (static_cast<int64_t>(moe::kTcBM) * a_row_bytes);
    a.band_m = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(b, 1 << 20)));
}

// Most (token, slot) pairs one expert takes in a call of T tokens:
// ceil(factor * T * K / n), or no limit when the factor is 0.
int capacity_for(const moe_handle* h, int64_t T) {
    if (!(h->capacity_factor > 0.0)) return moe::kNoCapacity;
    const double c = std::ceil(h->capacity_factor * static_cast<double>(T) * h->K / h->n);
    return c >= static_cast<double>(moe::kNoCapacity) ? moe::kNoCapacity : static_cast<int>(c);
}

// Gather the segment rows of x, then GEMM1 (w1/w3 + SwiGLU) and GEMM2 (w2)
// over R rows laid out by the dispatch arrays already on the device.
// bf16 GEMM1 on the single-SM tiles gathers its A rows from x itself (no
// gather kernel, no Xp) when the experts average at most 256 rows: there the
// GEMMs stream weights and the gather kernel's round trip through HBM is
// what the fused gather saves (decode 0.435 -> 0.424 ms, many_expert 0.317 ->
// 0.308 ms).  With more rows GEMM1 is bound by the tensor cores and the
// cp.async gather, two stages behind the tensor core, slowed it (prefill
// GEMM1 1.62 -> 1.99 ms), so the gather kernel stays.  MOE_GATHER=separate /
// fused forces either.
// Two 128-row blocks per single-SM tile (gemm_tc3.cu): three 64 KB stages in
// flight instead of four 48 KB ones cover half again as much copy latency per
// tensor cycle, but the two accumulators fill TMEM, so each tile's epilogue
// stalls the next tile's MMAs.  Both GEMMs take it when the experts average
// more than 256 rows (pairs of blocks are mostly full; below that GEMM1
// gathers its own rows and the GEMMs stream weights) and the GEMM's K is at
// least 4,096 (the epilogue is short against the tile).  Measured on the
// skewed prefill: GEMM2 3.06-3.12 -> 2.92-2.95 ms, GEMM1 6.11-6.15 -> 5.89-5.95
// ms (GEMM1 with eight epilogue warps and its TMEM loads pipelined; with four
// it was slower, 6.9-7.0 ms); prefill GEMM2 0.81 -> 0.75-0.79 ms.
// MOE_GEMM_PATH=dual puts both GEMMs on it for every batch;
// MOE_GEMM1_TILE / MOE_GEMM2_TILE = single|dual force one GEMM's choice.
bool use_dual_gemm() {
    const char* env = getenv("MOE_GEMM_PATH");
    return env && strcmp(env, "dual") == 0;
}

// E4M3 (fp8 = true) stays on the single-block kernel unless a variable asks:
// its main loop per tile is half as long, so the two-block kernel's epilogue,
// which does not overlap the next tile's MMAs, costs twice the share (prefill
// 1.37 -> 1.44 ms, skewed prefill 5.37-5.48 -> 5.60-5.70 ms measured).
bool use_dual_tile(bool gemm2, int64_t R, int n, int K, bool fp8 = false) {
    if (use_dual_gemm()) return true;
    const char* env = getenv(gemm2 ? "MOE_GEMM2_TILE" : "MOE_GEMM1_TILE");
    if (env && strcmp(env, "single") == 0) return false;
    if (env && strcmp(env, "dual") == 0) return true;
    return !fp8 && R > 256 * static_cast<int64_t>(n) && K >= 4096;
}

bool gather_in_gemm1(int64_t R, int n) {
    const char* env = getenv("MOE_GATHER");
    if (env && strcmp(env, "separate") == 0) return false;
    if (env && strcmp(env, "fused") == 0) return true;
    return R <= 256 * static_cast<int64_t>(n);
}

moe_status run_gemms(moe_handle* h, int64_t T, int64_t R, const void* x, const void* w1, const void* w3,
                     const void* w2, bool pair, cudaStream_t st) {
    const bool bf = h->dtype == MOE_BF16;
    const bool fused_gather = bf && !pair && gather_in_gemm1(R, h->n);
    const bool dual = bf && !pair && !fused_gather && use_dual_tile(false, R, h->n, h->d);
    const bool dual2 = bf && !pair && use_dual_tile(true, R, h->n, h->F);
    cudaError_t e;
    if (!fused_gather) {
        e = moe::launch_gather(x, h->db.row_token, R, T, static_cast<int64_t>(h->d) * h->esize(), h->xp,
                               h->num_sms, st);
        if (e != cudaSuccess) return cuda_fail(e, "gather launch");
        h->launches += 1;
    }
    trace_mark(h, 2, st);
    if (bf) {
        if (w1 != h->c_w1) {
            if (!encode_weights(&h->tm_w1, w1, h->F, h->d, h->n) ||
                !encode_weights_wide(&h->tm_w1x, w1, h->F, h->d, h->n, 2))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w1");
            h->c_w1 = w1;
        }
        if (w3 != h->c_w3) {
            if (!encode_weights(&h->tm_w3, w3, h->F, h->d, h->n) ||
                !encode_weights_wide(&h->tm_w3x, w3, h->F, h->d, h->n, 2))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w3");
            h->c_w3 = w3;
        }
        if (w2 != h->c_w2) {
            if (!encode_weights(&h->tm_w2, w2, h->d, h->F, h->n) ||
                !encode_weights_wide(&h->tm_w2x, w2, h->d, h->F, h->n, 4) ||
                !encode_weights_wide(&h->tm_w2p, w2, h->d, h->F, h->n, 2))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w2");
            h->c_w2 = w2;
        }
        moe::TcGemmArgs a1{};
        a1.offsets = h->db.offsets;
        a1.mblk_base = h->db.mblk_base;
        a1.n = h->n;
        a1.R = R;
        a1.k_blocks = h->d / 64;
        a1.n_tiles = (h->F + 127) / 128;
        a1.out_cols = h->F;
        a1.out = h->h;
        a1.status = h->status;
        a1.balanced = grid_balance();
        gemm_tile_order(a1, static_cast<int64_t>(h->d) * 2, false);
        if (fused_gather) {
            a1.x = static_cast<const uint16_t*>(x);
            a1.row_token = h->db.row_token;
            a1.x_rows = T;
            a1.x_cols = h->d;
            e = moe::launch_tc_gemm1_gather(h->tm_w1x, h->tm_w3x, a1, h->num_sms, st);
        } else if (pair) {
            e = moe::launch_tc_gemm1_pair(h->tm_xp, h->tm_w1x, h->tm_w3x, a1, h->num_sms, st);
        } else if (dual) {
            e = moe::launch_tc_gemm1_dual(h->tm_xp, h->tm_w1x, h->tm_w3x, a1, h->num_sms, st);
        } else {
            e = moe::launch_tc_gemm1(h->tm_xp, h->tm_w1x, h->tm_w3x, a1, h->num_sms, st);
        }
        if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
        h->launches += 1;
        trace_mark(h, 3, st);
        moe::TcGemmArgs a2 = a1;
        a2.k_blocks = h->F / 64;
        a2.n_tiles = (h->d + 255) / 256;
        a2.out_cols = h->d;
        a2.out = h->o;
        gemm_tile_order(a2, static_cast<int64_t>(h->F) * 2, true);
        e = pair ? moe::launch_tc_gemm2_pair(h->tm_h, h->tm_w2p, a2, h->num_sms, st)
                 : (dual2 ? moe::launch_tc_gemm2_dual(h->tm_h, h->tm_w2x, a2, h->num_sms, st)
                          : moe::launch_tc_gemm2(h->tm_h, h->tm_w2x, a2, h->num_sms, st));
        if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
        h->launches += 1;
        trace_mark(h, 4, st);
    } else {
        e = moe::launch_simt_gemm1(static_cast<const float*>(h->xp), static_cast<const float*>(w1),
                                   static_cast<const float*>(w3), static_cast<float*>(h->h),
                                   h->db.offsets, h->db.mblk_base, h->n, R, h->d, h->F, st);
        if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
        h->launches += 1;
        trace_mark(h, 3, st);
        e = moe::launch_simt_gemm2(static_cast<const float*>(h->h), static_cast<const float*>(w2),
                                   static_cast<float*>(h->o), h->db.offsets, h->db.mblk_base, h->n,
                                   R, h->d, h->F, st);
        if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
        h->launches += 1;
        trace_mark(h, 4, st);
    }
    return MOE_OK;
}

moe_status run_experts(moe_handle* h, int64_t T, const void* x, const int32_t* topk_idx,
                       const float* topk_w, const void* w1, const void* w3, const void* w2, void* y,
                       cudaStream_t st) {
    const bool bf = h->dtype == MOE_BF16;
    const bool pair = use_pair_gemm(h, T);
    const int64_t R = T * h->K;
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n,
                                         pair ? moe::kTcPairBM : (bf ? moe::kTcBM : moe::kSimtBM),
                                         h->db, st, capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    trace_mark(h, 1, st);
    moe_status s = run_gemms(h, T, R, x, w1, w3, w2, pair, st);
    if (s != MOE_OK) return s;
    e = moe::launch_combine(h->o, bf, h->db.token_row, topk_w, T, h->K, h->d, y, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return MOE_OK;
}

// The E4M3 expert path: dispatch, quantised gather of x (one scale per row),
// GEMM1 on E4M3 operands (bf16 H), H rows to E4M3 (one scale per row), GEMM2
// on E4M3 operands (bf16 O), combine.
moe_status run_experts_e4m3(moe_handle* h, int64_t T, const void* x, const int32_t* topk_idx,
                            const float* topk_w, const uint8_t* q1, const float* s1, const uint8_t* q3,
                            const float* s3, const uint8_t* q2, const float* s2, void* y, cudaStream_t st) {
    const int64_t R = T * h->K;
    const bool pair = use_pair_gemm_e4m3(h, T);
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n, pair ? moe::kTcPairBM : moe::kTcBM, h->db, st,
                                         capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    trace_mark(h, 1, st);
    const int32_t* used_rows = h->db.offsets + h->n;  // offsets[n]: rows the segments hold
    e = moe::launch_quantize_rows_e4m3(x, true, h->db.row_token, T, R, used_rows, h->d, h->x8, h->xs, h->num_sms,
                                       st);
    if (e != cudaSuccess) return cuda_fail(e, "activation quantisation launch");
    h->launches += 1;
    trace_mark(h, 2, st);
    if (q1 != h->c_q1) {
        if (!encode_codes(&h->tm_q1, q1, h->F, h->d, h->n))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w1 codes");
        h->c_q1 = q1;
    }
    if (q3 != h->c_q3) {
        if (!encode_codes(&h->tm_q3, q3, h->F, h->d, h->n))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w3 codes");
        h->c_q3 = q3;
    }
    if (q2 != h->c_q2) {
        if (!encode_codes(&h->tm_q2, q2, h->d, h->F, h->n))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for w2 codes");
        h->c_q2 = q2;
    }
    moe::TcGemmArgs a1{};
    a1.offsets = h->db.offsets;
    a1.mblk_base = h->db.mblk_base;
    a1.n = h->n;
    a1.R = R;
    a1.k_blocks = (h->d + 127) / 128;
    a1.n_tiles = (h->F + 127) / 128;
    a1.out_cols = h->F;
    a1.out = h->h;
    a1.status = h->status;
    a1.balanced = grid_balance();
    a1.row_scale = h->xs;
    a1.col_scale0 = s1;
    a1.col_scale1 = s3;
    gemm_tile_order(a1, h->d, false);
    const bool dual = !pair && use_dual_tile(false, R, h->n, h->d, true);
    const bool dual2 = !pair && use_dual_tile(true, R, h->n, h->F, true);
    e = pair   ? moe::launch_tc_gemm1_pair_e4m3(h->tm_x8, h->tm_q1, h->tm_q3, a1, h->num_sms, st)
        : dual ? moe::launch_tc_gemm1_dual_e4m3(h->tm_x8, h->tm_q1, h->tm_q3, a1, h->num_sms, st)
               : moe::launch_tc_gemm1_e4m3(h->tm_x8, h->tm_q1, h->tm_q3, a1, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
    trace_mark(h, 3, st);  // the GEMM1 stage is the GEMM1 kernel alone; the H rows go with GEMM2
    e = moe::launch_quantize_rows_e4m3(h->h, true, nullptr, R, R, used_rows, h->F, h->h8, h->hs, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "hidden-row quantisation launch");
    h->launches += 2;
    moe::TcGemmArgs a2 = a1;
    a2.k_blocks = (h->F + 127) / 128;
    a2.n_tiles = (h->d + 255) / 256;
    a2.out_cols = h->d;
    a2.out = h->o;
    a2.row_scale = h->hs;
    a2.col_scale0 = s2;
    a2.col_scale1 = nullptr;
    gemm_tile_order(a2, h->F, true);
    e = pair    ? moe::launch_tc_gemm2_pair_e4m3(h->tm_h8, h->tm_q2, a2, h->num_sms, st)
        : dual2 ? moe::launch_tc_gemm2_dual_e4m3(h->tm_h8, h->tm_q2, a2, h->num_sms, st)
                : moe::launch_tc_gemm2_e4m3(h->tm_h8, h->tm_q2, a2, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
    h->launches += 1;
    trace_mark(h, 4, st);
    e = moe::launch_combine(h->o, true, h->db.token_row, topk_w, T, h->K, h->d, y, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return MOE_OK;
}

// The 4-bit expert path: dispatch and gather as for bf16, then both GEMMs on
// the 4-bit weights (converted to bf16 tiles in shared memory), combine.
moe_status run_experts_fp4(moe_handle* h, int64_t T, const void* x, const float* topk_w, const uint8_t* const* cw,
                           const uint8_t* const* bs, const float* const* ts, void* y, const int32_t* topk_idx,
                           cudaStream_t st) {
    const int64_t R = T * h->K;
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n, moe::kTcBM, h->db, st, capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    trace_mark(h, 1, st);
    e = moe::launch_gather(x, h->db.row_token, R, T, static_cast<int64_t>(h->d) * 2, h->xp, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
    h->launches += 1;
    trace_mark(h, 2, st);
    // matrices: 0 = w1 [n][d][F], 1 = w3 [n][d][F], 2 = w2 [n][F][d]
    for (int m = 0; m < 3; ++m) {
        const uint64_t rows = m < 2 ? h->d : h->F, cols = m < 2 ? h->F : h->d;
        if (cw[m] != h->c_f4[2 * m]) {
            if (!encode_fp4_codes(&h->tm_f4[2 * m], cw[m], cols, rows, h->n))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for 4-bit codes");
            h->c_f4[2 * m] = cw[m];
        }
        if (bs[m] != h->c_f4[2 * m + 1]) {
            if (!encode_fp4_scales(&h->tm_f4[2 * m + 1], bs[m], cols, rows, h->n))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for 4-bit block scales");
            h->c_f4[2 * m + 1] = bs[m];
        }
    }
    moe::Fp4GemmArgs a1{};
    a1.balanced = 0;  // bound by its converter warps: every SM keeps working (measured 0.680 vs 0.688 ms)
    a1.offsets = h->db.offsets;
    a1.mblk_base = h->db.mblk_base;
    a1.n = h->n;
    a1.R = R;
    a1.k_blocks = h->d / 64;
    a1.n_tiles = (h->F + 127) / 128;
    a1.out_cols = h->F;
    a1.out = h->h;
    a1.status = h->status;
    a1.tscale0 = ts[0];
    a1.tscale1 = ts[1];
    e = moe::launch_fp4_gemm1(h->tm_xp, h->tm_f4[0], h->tm_f4[1], h->tm_f4[2], h->tm_f4[3], a1, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
    h->launches += 1;
    trace_mark(h, 3, st);
    moe::Fp4GemmArgs a2 = a1;
    a2.k_blocks = h->F / 64;
    a2.n_tiles = (h->d + 255) / 256;
    a2.out_cols = h->d;
    a2.out = h->o;
    a2.tscale0 = ts[2];
    a2.tscale1 = nullptr;
    e = moe::launch_fp4_gemm2(h->tm_h, h->tm_f4[4], h->tm_f4[5], a2, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
    h->launches += 1;
    trace_mark(h, 4, st);
    e = moe::launch_combine(h->o, true, h->db.token_row, topk_w, T, h->K, h->d, y, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return MOE_OK;
}

// The 4-bit weight-and-activation path: dispatch, x rows to 4 bits (with the
// tiles' scale chunks), GEMM1 on the block-scaled tensor cores (bf16 H), H rows
// to 4 bits, GEMM2, combine.
moe_status run_experts_w4a4(moe_handle* h, int64_t T, const void* x, const float* topk_w, const uint8_t* const* wp,
                            const uint8_t* const* wc, const float* const* ws, void* y, const int32_t* topk_idx,
                            cudaStream_t st) {
    const int64_t R = T * h->K;
    // 256-column tiles (one accumulator) by default: on the Mixtral decode
    // and prefill shapes and 128 experts of 2048 x 768 they measured faster
    // than 128-column tiles with two accumulators, which reload A for every
    // 64 hidden columns.  Row tiles of 32 when the experts average at most 32
    // rows: a quarter of the A bytes per stage, and a fifth stage in flight.
    bool wide = true;
    if (const char* v = getenv("MOE_W4A4_TILE")) {  // 128 or 256 forces a width
        if (atoi(v) == 128) wide = false;
        if (atoi(v) == 256) wide = true;
    }
    int tile_rows = R <= 32 * static_cast<int64_t>(h->n) ? 32 : 128;
    if (const char* v = getenv("MOE_W4A4_ROWS")) {  // 32 or 128 forces a height
        if (atoi(v) == 128) tile_rows = 128;
        if (atoi(v) == 32) tile_rows = 32;
    }
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n, tile_rows, h->db, st, capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    trace_mark(h, 1, st);
    e = moe::launch_w4a4_rows(static_cast<const uint16_t*>(x), h->db.row_token, T, R, h->d, h->db.offsets,
                              h->db.mblk_base, h->n, tile_rows, h->xq4, h->xc4, h->xr4, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "activation quantisation launch");
    h->launches += 1;
    trace_mark(h, 2, st);
    // wp[0]: the gate/up pair pack (2 ffn rows of d codes), wp[1]: w2 (d rows of ffn)
    const int bn = moe::w4a4_tile_cols(wide);
    for (int m = 0; m < 2; ++m) {
        // boxes of a whole tile's rows: the kernel brings them in one copy
        const uint64_t K = m == 0 ? h->d : h->F, N = m == 0 ? 2 * static_cast<uint64_t>(h->F) : h->d;
        if (wp[m] != h->c_wp4[m] || h->c_wp4_rows[m] != bn) {
            if (!encode_codes(&h->tm_wp4[m], wp[m], K / 2, N, h->n, static_cast<uint32_t>(bn)))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for packed 4-bit weights");
            h->c_wp4[m] = wp[m];
            h->c_wp4_rows[m] = bn;
        }
    }
    moe::W4a4GemmArgs a1{};
    a1.offsets = h->db.offsets;
    a1.mblk_base = h->db.mblk_base;
    a1.n = h->n;
    a1.R = R;
    a1.k_steps = h->d / 256;
    a1.n_tiles = 2 * h->F / bn;
    a1.out_cols = h->F;
    a1.n_rows_b = 2 * h->F;
    a1.out = h->h;
    a1.status = h->status;
    a1.balanced = grid_balance();
    a1.row_scale = h->xr4;
    a1.mscale0 = ws[0];
    a1.mscale1 = ws[1];
    a1.a_chunks = h->xc4;
    a1.b_chunks = wc[0];
    e = moe::launch_w4a4_gemm1(tile_rows == 32 ? h->tm_xq4s : h->tm_xq4, h->tm_wp4[0], a1, wide, tile_rows,
                               h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
    trace_mark(h, 3, st);  // the GEMM1 stage is the GEMM1 kernel alone; the H rows go with GEMM2
    e = moe::launch_w4a4_rows(static_cast<const uint16_t*>(h->h), nullptr, R, R, h->F, h->db.offsets,
                              h->db.mblk_base, h->n, tile_rows, h->hq4, h->hc4, h->hr4, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "hidden-row quantisation launch");
    h->launches += 2;
    moe::W4a4GemmArgs a2 = a1;
    a2.k_steps = h->F / 256;
    a2.n_tiles = h->d / bn;
    a2.out_cols = h->d;
    a2.n_rows_b = h->d;
    a2.out = h->o;
    a2.row_scale = h->hr4;
    a2.mscale0 = ws[2];
    a2.mscale1 = ws[2];
    a2.a_chunks = h->hc4;
    a2.b_chunks = wc[1];
    e = moe::launch_w4a4_gemm2(tile_rows == 32 ? h->tm_hq4s : h->tm_hq4, h->tm_wp4[1], a2, wide, tile_rows,
                               h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
    h->launches += 1;
    trace_mark(h, 4, st);
    e = moe::launch_combine(h->o, true, h->db.token_row, topk_w, T, h->K, h->d, y, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return MOE_OK;
}

// 4-bit weights with bf16 activations, decoded into tensor memory: dispatch
// (token blocks of 32 rows when the experts average at most 32 rows, else
// 128), gather, GEMM1 over the gate/up pair pack, GEMM2, combine.
moe_status run_experts_w4a16(moe_handle* h, int64_t T, const void* x, const float* topk_w,
                             const uint8_t* const* wp, const float* const* ws, void* y, const int32_t* topk_idx,
                             cudaStream_t st) {
    const int64_t R = T * h->K;
    int tile_rows = moe::w4a16_tile_rows(R, h->n);
    if (const char* v = getenv("MOE_W4A16_ROWS")) {  // 32 or 128 forces the token block
        if (atoi(v) == 32) tile_rows = 32;
        if (atoi(v) == 128) tile_rows = 128;
    }
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n, tile_rows, h->db, st, capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    trace_mark(h, 1, st);
    e = moe::launch_gather(x, h->db.row_token, R, T, static_cast<int64_t>(h->d) * 2, h->xp, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
    h->launches += 1;
    trace_mark(h, 2, st);
    moe::W4a16GemmArgs a1{};
    a1.offsets = h->db.offsets;
    a1.mblk_base = h->db.mblk_base;
    a1.n = h->n;
    a1.R = R;
    a1.k_blocks = h->d / 64;
    a1.n_tiles = h->F / 64;
    a1.out_cols = h->F;
    a1.out = h->h;
    a1.status = h->status;
    a1.wpack = wp[0];
    a1.mscale0 = ws[0];
    a1.mscale1 = ws[1];
    a1.balanced = grid_balance();
    e = moe::launch_w4a16_gemm1(h->tm_xpw[tile_rows == 32 ? 0 : 1], a1, tile_rows, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
    h->launches += 1;
    trace_mark(h, 3, st);
    moe::W4a16GemmArgs a2 = a1;
    a2.k_blocks = h->F / 64;
    a2.n_tiles = h->d / 128;
    a2.out_cols = h->d;
    a2.out = h->o;
    a2.wpack = wp[1];
    a2.mscale0 = ws[2];
    a2.mscale1 = ws[2];
    e = moe::launch_w4a16_gemm2(h->tm_hw[tile_rows == 32 ? 0 : 1], a2, tile_rows, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
    h->launches += 1;
    trace_mark(h, 4, st);
    e = moe::launch_combine(h->o, true, h->db.token_row, topk_w, T, h->K, h->d, y, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return MOE_OK;
}

// Router logits into h->logits (tensor cores for bf16, CUDA cores for fp32);
// returns the number of split partials.
moe_status run_logits(moe_handle* h, int64_t T, const void* x, const float* W_g, cudaStream_t st,
                      int* splits) {
    cudaError_t e;
    *splits = 1;
    if (h->dtype == MOE_BF16) {
        if (x != h->c_rx || T != h->c_rx_T) {
            if (!encode_rows(&h->tm_rx, x, h->d, static_cast<uint64_t>(T)))
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
            h->c_rx = x;
            h->c_rx_T = T;
        }
        e = moe::launch_router_logits_tc(h->tm_rx, h->tm_parts, W_g, h->wg_parts, T, h->d, h->n, h->logits,
                                         h->status, h->num_sms, st, splits);
        h->launches += 2;
    } else {
        e = moe::launch_router_logits_simt(x, false, W_g, T, h->d, h->n, h->logits, st);
        h->launches += 1;
    }
    if (e != cudaSuccess) return cuda_fail(e, "router logits launch");
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// Expert parallelism
moe_status ep_check(moe_handle* h, int world, int rank) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (world < 1 || world > moe::kMaxEpRanks)
        return fail(MOE_ERR_INVALID_ARG, "world = %d outside [1, %d]", world, moe::kMaxEpRanks);
    if (rank < 0 || rank >= world) return fail(MOE_ERR_INVALID_ARG, "rank = %d outside [0, %d)", rank, world);
    if (h->n % world != 0)
        return fail(MOE_ERR_INVALID_ARG, "n = %d experts do not split evenly over %d ranks", h->n, world);
    if (h->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "expert parallelism needs a MOE_BF16 handle");
    if (h->capacity_factor > 0.0)
        return fail(MOE_ERR_UNSUPPORTED, "expert parallelism is dropless: the capacity factor must be 0");
    return MOE_OK;
}

moe_status ep_peers(int world, void* const* ptrs, const char* name, moe::EpPeers* out) {
    if (!ptrs) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
    *out = moe::EpPeers{};
    for (int q = 0; q < world; ++q) {
        if (!ptrs[q]) return fail(MOE_ERR_INVALID_ARG, "%s[%d] is NULL", name, q);
        if (!aligned16(ptrs[q])) return fail(MOE_ERR_INVALID_ARG, "%s[%d] is not 16-byte aligned", name, q);
        out->ptr[q] = ptrs[q];
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_create(int n, int K, int d, int ffn, moe_dtype dtype, moe_handle** out) {
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (n < 1 || n > 256) return fail(MOE_ERR_INVALID_ARG, "n = %d outside [1, 256]", n);
    if (K < 1 || K > n) return fail(MOE_ERR_INVALID_ARG, "K = %d outside [1, n = %d]", K, n);
    if (d < 64 || d > 65536 || d % 64 != 0)
        return fail(MOE_ERR_INVALID_ARG, "d = %d is not a multiple of 64 in [64, 65536]", d);
    if (ffn < 64 || ffn > 65536 || ffn % 64 != 0)
        return fail(MOE_ERR_INVALID_ARG, "ffn = %d is not a multiple of 64 in [64, 65536]", ffn);
    if (dtype != MOE_F32 && dtype != MOE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "dtype = %d is not MOE_F32 or MOE_BF16", static_cast<int>(dtype));
    moe_handle* h = new (std::nothrow) moe_handle();
    if (!h) return fail(MOE_ERR_ALLOC, "out of host memory");
    h->n = n;
    h->K = K;
    h->d = d;
    h->F = ffn;
    h->dtype = dtype;
    *out = h;
    return ok();
}

moe_status moe_reserve(moe_handle* h, int64_t T_max) {
    moe_status s = check_common(h, T_max);
    if (s != MOE_OK) return s;
    if (T_max == 0) return ok();
    s = prepare(h, T_max);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_route(moe_handle* h, int64_t T, const void* x, const float* W_g, int32_t* topk_idx,
                     float* topk_w, moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_forward(moe_handle* h, int64_t T, const void* x, const float* W_g, const void* w1,
                       const void* w3, const void* w2, void* y, int32_t* topk_idx, float* topk_w,
                       moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w1);
    REQUIRE_PTR(w3);
    REQUIRE_PTR(w2);
    REQUIRE_PTR(y);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    if (s != MOE_OK) return s;
    trace_mark(h, 0, st);
    s = run_experts(h, T, x, topk_idx, topk_w, w1, w3, w2, y, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_forward_with_routing(moe_handle* h, int64_t T, const void* x,
                                    const int32_t* topk_idx, const float* topk_w, const void* w1,
                                    const void* w3, const void* w2, void* y, moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(w1);
    REQUIRE_PTR(w3);
    REQUIRE_PTR(w2);
    REQUIRE_PTR(y);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    trace_mark(h, 0, st);
    s = run_experts(h, T, x, topk_idx, topk_w, w1, w3, w2, y, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_dispatch(moe_handle* h, int64_t T, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* row_token, int32_t* token_row,
                        moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    REQUIRE_PTR(topk_idx);
    if (T == 0) return ok();
    if (counts && !aligned16(counts)) return fail(MOE_ERR_INVALID_ARG, "counts is not 16-byte aligned");
    if (offsets && !aligned16(offsets)) return fail(MOE_ERR_INVALID_ARG, "offsets is not 16-byte aligned");
    if (row_token && !aligned16(row_token))
        return fail(MOE_ERR_INVALID_ARG, "row_token is not 16-byte aligned");
    if (token_row && !aligned16(token_row))
        return fail(MOE_ERR_INVALID_ARG, "token_row is not 16-byte aligned");
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    const int64_t R = T * h->K;
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n,
                                         h->dtype == MOE_BF16 ? moe::kTcBM : moe::kSimtBM, h->db, st,
                                         capacity_for(h, T));
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    struct {
        void* dst;
        const void* src;
        size_t bytes;
    } cp[4] = {{counts, h->db.counts, static_cast<size_t>(h->n) * 4},
               {offsets, h->db.offsets, static_cast<size_t>(h->n + 1) * 4},
               {row_token, h->db.row_token, static_cast<size_t>(R) * 4},
               {token_row, h->db.token_row, static_cast<size_t>(R) * 4}};
    for (auto& c : cp) {
        if (!c.dst) continue;
        e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(dispatch output)");
    }
    return ok();
}

moe_status moe_forward_expert_choice(moe_handle* h, int64_t T, int64_t capacity, const void* x,
                                     const float* W_g, const void* w1, const void* w3, const void* w2,
                                     void* y, int32_t* sel_token, float* sel_gate, moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (T == 0) return ok();
    if (capacity < 1 || capacity > T)
        return fail(MOE_ERR_INVALID_ARG, "capacity = %lld outside [1, T = %lld]",
                    static_cast<long long>(capacity), static_cast<long long>(T));
    if (capacity * h->n > 2147483647LL)
        return fail(MOE_ERR_INVALID_ARG, "capacity * n exceeds 2^31 - 1");
    if (T > 2147483647LL) return fail(MOE_ERR_INVALID_ARG, "T exceeds 2^31 - 1");
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w1);
    REQUIRE_PTR(w3);
    REQUIRE_PTR(w2);
    REQUIRE_PTR(y);
    REQUIRE_PTR(sel_token);
    REQUIRE_PTR(sel_gate);
    const int64_t R = capacity * h->n;
    s = prepare(h, T, R);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    int splits = 1;
    s = run_logits(h, T, x, W_g, st, &splits);
    if (s != MOE_OK) return s;
    const bool pair = use_pair_gemm(h, T);
    const int bm = pair ? moe::kTcPairBM : (h->dtype == MOE_BF16 ? moe::kTcBM : moe::kSimtBM);
    cudaError_t e = moe::launch_ec_route(h->logits, splits, T, h->n, static_cast<int>(capacity), bm,
                                         h->ec_probs, h->ec_rowmap, sel_token, sel_gate, h->db.row_token,
                                         h->db.counts, h->db.offsets, h->db.mblk_base, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-choice routing launch");
    h->launches += 2;
    trace_mark(h, 0, st);
    trace_mark(h, 1, st);
    s = run_gemms(h, T, R, x, w1, w3, w2, pair, st);
    if (s != MOE_OK) return s;
    e = moe::launch_ec_combine(h->o, h->dtype == MOE_BF16, h->ec_rowmap, sel_gate, T, h->n, h->d, y,
                               h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-choice combine launch");
    h->launches += 1;
    trace_mark(h, 5, st);
    trace_finish_call(h);
    return ok();
}

moe_status moe_quantize_weights_e4m3(int n, int rows, int cols, const void* w, moe_dtype dtype, uint8_t* codes,
                                     float* scales, moe_stream_t stream) {
    if (n < 1 || n > 65535) return fail(MOE_ERR_INVALID_ARG, "n = %d outside [1, 65535]", n);
    if (rows < 1) return fail(MOE_ERR_INVALID_ARG, "rows = %d < 1", rows);
    if (cols < 16 || cols % 16 != 0)
        return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a positive multiple of 16", cols);
    if (dtype != MOE_F32 && dtype != MOE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "dtype = %d is not MOE_F32 or MOE_BF16", static_cast<int>(dtype));
    if (static_cast<int64_t>(n) * rows * cols > (static_cast<int64_t>(1) << 40))
        return fail(MOE_ERR_INVALID_ARG, "n * rows * cols exceeds 2^40");
    REQUIRE_PTR(w);
    REQUIRE_PTR(codes);
    REQUIRE_PTR(scales);
    int dev = 0, sms = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10) return fail(MOE_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
    e = moe::launch_quantize_weights_e4m3(w, dtype == MOE_BF16, n, rows, cols, codes, scales, sms,
                                          reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "weight quantisation launch");
    return ok();
}

moe_status moe_forward_e4m3(moe_handle* h, int64_t T, const void* x, const float* W_g, const uint8_t* w1_q,
                            const float* w1_s, const uint8_t* w3_q, const float* w3_s, const uint8_t* w2_q,
                            const float* w2_s, void* y, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (h->dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "the E4M3 expert path needs a MOE_BF16 handle");
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w1_q);
    REQUIRE_PTR(w1_s);
    REQUIRE_PTR(w3_q);
    REQUIRE_PTR(w3_s);
    REQUIRE_PTR(w2_q);
    REQUIRE_PTR(w2_s);
    REQUIRE_PTR(y);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    h->want_e4m3 = true;
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    if (s != MOE_OK) return s;
    trace_mark(h, 0, st);
    s = run_experts_e4m3(h, T, x, topk_idx, topk_w, w1_q, w1_s, w3_q, w3_s, w2_q, w2_s, y, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_quantize_weights_fp4(int n, int rows, int cols, const void* w, moe_dtype dtype, uint8_t* codes,
                                    uint8_t* block_scales, float* matrix_scales, moe_stream_t stream) {
    if (n < 1 || n > 65535) return fail(MOE_ERR_INVALID_ARG, "n = %d outside [1, 65535]", n);
    if (rows < 16 || rows % 16 != 0)
        return fail(MOE_ERR_INVALID_ARG, "rows = %d is not a positive multiple of 16", rows);
    if (cols < 32 || cols % 32 != 0)
        return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a positive multiple of 32", cols);
    if (dtype != MOE_F32 && dtype != MOE_BF16)
        return fail(MOE_ERR_INVALID_ARG, "dtype = %d is not MOE_F32 or MOE_BF16", static_cast<int>(dtype));
    if (static_cast<int64_t>(rows) / 16 * (cols / 2) > 2147483647LL / 256)
        return fail(MOE_ERR_INVALID_ARG, "rows * cols too large");
    REQUIRE_PTR(w);
    REQUIRE_PTR(codes);
    REQUIRE_PTR(block_scales);
    REQUIRE_PTR(matrix_scales);
    int dev = 0, sms = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10) return fail(MOE_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
    e = moe::launch_quantize_weights_fp4(w, dtype == MOE_BF16, n, rows, cols, codes, block_scales, matrix_scales,
                                         sms, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "4-bit weight quantisation launch");
    return ok();
}

moe_status moe_forward_fp4(moe_handle* h, int64_t T, const void* x, const float* W_g, const uint8_t* w1_codes,
                           const uint8_t* w1_bscale, const float* w1_tscale, const uint8_t* w3_codes,
                           const uint8_t* w3_bscale, const float* w3_tscale, const uint8_t* w2_codes,
                           const uint8_t* w2_bscale, const float* w2_tscale, void* y, int32_t* topk_idx,
                           float* topk_w, moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (h->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "the 4-bit expert path needs a MOE_BF16 handle");
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w1_codes);
    REQUIRE_PTR(w1_bscale);
    REQUIRE_PTR(w1_tscale);
    REQUIRE_PTR(w3_codes);
    REQUIRE_PTR(w3_bscale);
    REQUIRE_PTR(w3_tscale);
    REQUIRE_PTR(w2_codes);
    REQUIRE_PTR(w2_bscale);
    REQUIRE_PTR(w2_tscale);
    REQUIRE_PTR(y);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    if (s != MOE_OK) return s;
    trace_mark(h, 0, st);
    const uint8_t* cw[3] = {w1_codes, w3_codes, w2_codes};
    const uint8_t* bs[3] = {w1_bscale, w3_bscale, w2_bscale};
    const float* ts[3] = {w1_tscale, w3_tscale, w2_tscale};
    s = run_experts_fp4(h, T, x, topk_w, cw, bs, ts, y, topk_idx, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_pack_weights_w4a4(int n, int rows, int cols, const uint8_t* codes, const uint8_t* block_scales,
                                  const uint8_t* pair_codes, const uint8_t* pair_block_scales, uint8_t* packed_codes,
                                  uint8_t* scale_chunks, moe_stream_t stream) {
    if (n < 1 || n > 65535) return fail(MOE_ERR_INVALID_ARG, "n = %d outside [1, 65535]", n);
    if (rows < 64 || rows % 64 != 0 || rows > 1048576)
        return fail(MOE_ERR_INVALID_ARG, "rows = %d is not a multiple of 64 in [64, 1048576]", rows);
    if (pair_codes) {
        if (cols < 64 || cols % 64 != 0 || cols > 1048576)
            return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a multiple of 64 in [64, 1048576]", cols);
    } else if (cols < 128 || cols % 128 != 0 || cols > 1048576) {
        return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a multiple of 128 in [128, 1048576]", cols);
    }
    if ((pair_codes == nullptr) != (pair_block_scales == nullptr))
        return fail(MOE_ERR_INVALID_ARG, "pair_codes and pair_block_scales must both be given or both be null");
    REQUIRE_PTR(codes);
    REQUIRE_PTR(block_scales);
    REQUIRE_PTR(packed_codes);
    REQUIRE_PTR(scale_chunks);
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return fail(MOE_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
    e = moe::launch_w4a4_pack(codes, block_scales, pair_codes, pair_block_scales, n, rows, cols, packed_codes,
                              scale_chunks, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "4-bit weight packing launch");
    return ok();
}

moe_status moe_forward_w4a4(moe_handle* h, int64_t T, const void* x, const float* W_g, const uint8_t* w13_packed,
                            const uint8_t* w13_chunks, const float* w1_matrix_scales,
                            const float* w3_matrix_scales, const uint8_t* w2_packed, const uint8_t* w2_chunks,
                            const float* w2_matrix_scales, void* y, int32_t* topk_idx, float* topk_w,
                            moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (h->dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "the 4-bit weight-and-activation path needs a MOE_BF16 handle");
    if (h->d % 256 != 0 || h->F % 256 != 0)
        return fail(MOE_ERR_UNSUPPORTED, "the 4-bit weight-and-activation path needs d and ffn multiples of 256");
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w13_packed);
    REQUIRE_PTR(w13_chunks);
    REQUIRE_PTR(w1_matrix_scales);
    REQUIRE_PTR(w3_matrix_scales);
    REQUIRE_PTR(w2_packed);
    REQUIRE_PTR(w2_chunks);
    REQUIRE_PTR(w2_matrix_scales);
    REQUIRE_PTR(y);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    h->want_w4a4 = true;
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    if (s != MOE_OK) return s;
    trace_mark(h, 0, st);
    const uint8_t* wp[2] = {w13_packed, w2_packed};
    const uint8_t* wc[2] = {w13_chunks, w2_chunks};
    const float* ws[3] = {w1_matrix_scales, w3_matrix_scales, w2_matrix_scales};
    s = run_experts_w4a4(h, T, x, topk_w, wp, wc, ws, y, topk_idx, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_pack_weights_w4a16(int n, int rows, int cols, const uint8_t* codes, const uint8_t* block_scales,
                                   const uint8_t* pair_codes, const uint8_t* pair_block_scales, uint8_t* packed,
                                   moe_stream_t stream) {
    if (n < 1 || n > 65535) return fail(MOE_ERR_INVALID_ARG, "n = %d outside [1, 65535]", n);
    if (rows < 64 || rows % 64 != 0 || rows > 1048576)
        return fail(MOE_ERR_INVALID_ARG, "rows = %d is not a multiple of 64 in [64, 1048576]", rows);
    if (pair_codes) {
        if (cols < 64 || cols % 64 != 0 || cols > 1048576)
            return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a multiple of 64 in [64, 1048576]", cols);
    } else if (cols < 128 || cols % 128 != 0 || cols > 1048576) {
        return fail(MOE_ERR_INVALID_ARG, "cols = %d is not a multiple of 128 in [128, 1048576]", cols);
    }
    if ((pair_codes == nullptr) != (pair_block_scales == nullptr))
        return fail(MOE_ERR_INVALID_ARG, "pair_codes and pair_block_scales must both be given or both be null");
    if (static_cast<int64_t>(pair_codes ? 2 * cols : cols) * (rows / 64) > 2147483647LL / 256)
        return fail(MOE_ERR_INVALID_ARG, "rows * cols too large");
    REQUIRE_PTR(codes);
    REQUIRE_PTR(block_scales);
    REQUIRE_PTR(packed);
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) return fail(MOE_ERR_UNSUPPORTED, "device %d is not sm_100", dev);
    e = moe::launch_w4a16_pack(codes, block_scales, pair_codes, pair_block_scales, n, rows, cols, packed,
                               reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "4-bit weight packing launch");
    return ok();
}

moe_status moe_forward_w4a16(moe_handle* h, int64_t T, const void* x, const float* W_g, const uint8_t* w13_packed,
                             const float* w1_matrix_scales, const float* w3_matrix_scales, const uint8_t* w2_packed,
                             const float* w2_matrix_scales, void* y, int32_t* topk_idx, float* topk_w,
                             moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (h->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "the 4-bit weight path needs a MOE_BF16 handle");
    if (h->d % 128 != 0)
        return fail(MOE_ERR_UNSUPPORTED, "the 4-bit weight path needs d a multiple of 128 (d = %d)", h->d);
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(w13_packed);
    REQUIRE_PTR(w1_matrix_scales);
    REQUIRE_PTR(w3_matrix_scales);
    REQUIRE_PTR(w2_packed);
    REQUIRE_PTR(w2_matrix_scales);
    REQUIRE_PTR(y);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    trace_mark(h, -1, st);
    s = run_router(h, T, x, W_g, topk_idx, topk_w, st);
    if (s != MOE_OK) return s;
    trace_mark(h, 0, st);
    const uint8_t* wp[2] = {w13_packed, w2_packed};
    const float* ws[3] = {w1_matrix_scales, w3_matrix_scales, w2_matrix_scales};
    s = run_experts_w4a16(h, T, x, topk_w, wp, ws, y, topk_idx, st);
    return s == MOE_OK ? ok() : s;
}

moe_status moe_ep_dispatch(moe_handle* h, int world, int rank, int64_t T, const void* x, const int32_t* topk_idx,
                           const int32_t* counts_all, void* const* recv_buffers, int64_t recv_rows,
                           int32_t* row_pos, moe_stream_t stream) {
    moe_status s = ep_check(h, world, rank);
    if (s != MOE_OK) return s;
    s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (recv_rows < 1 || recv_rows > 2147483647LL)
        return fail(MOE_ERR_INVALID_ARG, "recv_rows = %lld outside [1, 2^31 - 1]", static_cast<long long>(recv_rows));
    moe::EpPeers peers;
    s = ep_peers(world, recv_buffers, "recv_buffers", &peers);
    if (s != MOE_OK) return s;
    REQUIRE_PTR(counts_all);
    if (T == 0) return ok();
    REQUIRE_PTR(x);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(row_pos);
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    const int64_t R = T * h->K;
    cudaError_t e = moe::launch_dispatch(topk_idx, T, h->K, h->n, moe::kTcBM, h->db, st, moe::kNoCapacity);
    if (e != cudaSuccess) return cuda_fail(e, "dispatch launch");
    h->launches += moe::dispatch_kernel_count(R);
    e = moe::launch_ep_plan(counts_all, world, h->n, rank, h->db.counts, recv_rows, h->ep_dst, h->ep_loff,
                            h->ep_lmblk, h->status, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-parallel plan launch");
    e = moe::launch_ep_scatter(x, topk_idx, h->db.token_row, h->db.offsets, h->ep_dst, T, h->K, h->n,
                               h->n / world, peers, recv_rows, h->d, row_pos, h->status, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-parallel scatter launch");
    h->launches += 2;
    return ok();
}

moe_status moe_ep_experts(moe_handle* h, int world, int rank, const int32_t* counts_all, const void* recv,
                          int64_t recv_rows, const void* w1, const void* w3, const void* w2, void* out,
                          moe_stream_t stream) {
    moe_status s = ep_check(h, world, rank);
    if (s != MOE_OK) return s;
    if (recv_rows < 1 || recv_rows > 2147483647LL)
        return fail(MOE_ERR_INVALID_ARG, "recv_rows = %lld outside [1, 2^31 - 1]", static_cast<long long>(recv_rows));
    REQUIRE_PTR(counts_all);
    REQUIRE_PTR(recv);
    REQUIRE_PTR(w1);
    REQUIRE_PTR(w3);
    REQUIRE_PTR(w2);
    REQUIRE_PTR(out);
    s = prepare(h, 0, recv_rows);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    const int nl = h->n / world;
    if (recv != h->c_erecv || recv_rows != h->c_erecv_rows) {
        if (!encode_rows(&h->tm_erecv, recv, h->d, static_cast<uint64_t>(recv_rows)))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the receive buffer");
        h->c_erecv = recv;
        h->c_erecv_rows = recv_rows;
    }
    const void* w[3] = {w1, w3, w2};
    CUtensorMap* tm[3] = {&h->tm_ew1, &h->tm_ew3, &h->tm_ew2};
    for (int m = 0; m < 3; ++m) {
        if (w[m] == h->c_ew[m] && nl == h->c_ew_nl) continue;
        const bool down = m == 2;
        if (!encode_weights_wide(tm[m], w[m], down ? h->d : h->F, down ? h->F : h->d, static_cast<uint64_t>(nl),
                                 down ? 4 : 2))
            return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed for the local expert weights");
        h->c_ew[m] = w[m];
    }
    h->c_ew_nl = nl;
    cudaError_t e = moe::launch_ep_plan(counts_all, world, h->n, rank, nullptr, recv_rows, h->ep_dst, h->ep_loff,
                                        h->ep_lmblk, h->status, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-parallel plan launch");
    moe::TcGemmArgs a1{};
    a1.offsets = h->ep_loff;
    a1.mblk_base = h->ep_lmblk;
    a1.n = nl;
    a1.R = recv_rows;
    a1.k_blocks = h->d / 64;
    a1.n_tiles = (h->F + 127) / 128;
    a1.out_cols = h->F;
    a1.out = h->h;
    a1.status = h->status;
    a1.balanced = grid_balance();
    gemm_tile_order(a1, static_cast<int64_t>(h->d) * 2, false);
    e = moe::launch_tc_gemm1(h->tm_erecv, h->tm_ew1, h->tm_ew3, a1, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM1 launch");
    moe::TcGemmArgs a2 = a1;
    a2.k_blocks = h->F / 64;
    a2.n_tiles = (h->d + 255) / 256;
    a2.out_cols = h->d;
    a2.out = out;
    gemm_tile_order(a2, static_cast<int64_t>(h->F) * 2, true);
    e = moe::launch_tc_gemm2(h->tm_h, h->tm_ew2, a2, h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "GEMM2 launch");
    h->launches += 3;
    return ok();
}

moe_status moe_ep_combine(moe_handle* h, int world, int64_t T, const int32_t* topk_idx, const float* topk_w,
                          const int32_t* row_pos, const void* const* out_buffers, void* y, moe_stream_t stream) {
    moe_status s = ep_check(h, world, 0);
    if (s != MOE_OK) return s;
    s = check_common(h, T);
    if (s != MOE_OK) return s;
    moe::EpPeers peers;
    s = ep_peers(world, const_cast<void* const*>(out_buffers), "out_buffers", &peers);
    if (s != MOE_OK) return s;
    if (T == 0) return ok();
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(row_pos);
    REQUIRE_PTR(y);
    s = check_device(h);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    cudaError_t e = moe::launch_ep_combine(topk_idx, topk_w, row_pos, T, h->K, h->n, h->n / world, peers, h->d, y,
                                           h->num_sms, st);
    if (e != cudaSuccess) return cuda_fail(e, "expert-parallel combine launch");
    h->launches += 1;
    return ok();
}

moe_status moe_ep_buffer_alloc(int64_t bytes, void** ptr, uint8_t* ipc_handle) {
    if (!ptr) return fail(MOE_ERR_INVALID_ARG, "ptr is NULL");
    *ptr = nullptr;
    if (bytes < 1) return fail(MOE_ERR_INVALID_ARG, "bytes = %lld < 1", static_cast<long long>(bytes));
    void* p = nullptr;
    cudaError_t e = cudaMalloc(&p, static_cast<size_t>(bytes));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(MOE_ERR_ALLOC, "cudaMalloc(%lld bytes) failed: %s", static_cast<long long>(bytes),
                    cudaGetErrorString(e));
    }
    if (ipc_handle) {
        cudaIpcMemHandle_t hd;
        e = cudaIpcGetMemHandle(&hd, p);
        if (e != cudaSuccess) {
            cudaFree(p);
            return cuda_fail(e, "cudaIpcGetMemHandle");
        }
        static_assert(sizeof hd == 64, "CUDA IPC handles are 64 bytes");
        memcpy(ipc_handle, &hd, sizeof hd);
    }
    *ptr = p;
    return ok();
}

moe_status moe_ep_buffer_open(const uint8_t* ipc_handle, void** ptr) {
    if (!ipc_handle || !ptr) return fail(MOE_ERR_INVALID_ARG, "ipc_handle or ptr is NULL");
    *ptr = nullptr;
    cudaIpcMemHandle_t hd;
    memcpy(&hd, ipc_handle, sizeof hd);
    void* p = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&p, hd, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
    *ptr = p;
    return ok();
}

moe_status moe_ep_buffer_close(void* ptr, int opened) {
    if (!ptr) return ok();
    cudaError_t e = opened ? cudaIpcCloseMemHandle(ptr) : cudaFree(ptr);
    if (e != cudaSuccess) return cuda_fail(e, opened ? "cudaIpcCloseMemHandle" : "cudaFree");
    return ok();
}

moe_status moe_set_gate_rounding(moe_handle* h, int bf16) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (bf16 != 0 && bf16 != 1) return fail(MOE_ERR_INVALID_ARG, "bf16 = %d is neither 0 nor 1", bf16);
    h->gates_bf16 = bf16 == 1;
    return ok();
}

moe_status moe_set_capacity_factor(moe_handle* h, double factor) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (!(factor >= 0.0) || !std::isfinite(factor))
        return fail(MOE_ERR_INVALID_ARG, "capacity factor must be finite and >= 0 (0 = no capacity)");
    h->capacity_factor = factor;
    return ok();
}

moe_status moe_router_stats(moe_handle* h, int64_t T, const void* x, const float* W_g,
                            const int32_t* topk_idx, float alpha, float* f, float* P, float* aux,
                            moe_stream_t stream) {
    moe_status s = check_common(h, T);
    if (s != MOE_OK) return s;
    if (T == 0) return fail(MOE_ERR_INVALID_ARG, "T = 0: the statistics are averages over tokens");
    REQUIRE_PTR(x);
    REQUIRE_PTR(W_g);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(f);
    REQUIRE_PTR(P);
    REQUIRE_PTR(aux);
    if (!std::isfinite(alpha)) return fail(MOE_ERR_INVALID_ARG, "alpha is not finite");
    s = prepare(h, T);
    if (s != MOE_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    int splits = 1;
    s = run_logits(h, T, x, W_g, st, &splits);
    if (s != MOE_OK) return s;
    cudaError_t e;
    e = moe::launch_router_stats(h->logits, splits, T, h->n, h->K, topk_idx, alpha, h->stats_partial,
                                 h->stats_counts, f, P, aux, st);
    if (e != cudaSuccess) return cuda_fail(e, "router statistics launch");
    h->launches += 2;
    return ok();
}

moe_status moe_workspace_view(moe_handle* h, const char* name, void** ptr, int64_t* rows) {
    if (!h || !name || !ptr || !rows) return fail(MOE_ERR_INVALID_ARG, "null argument");
    if (!h->ws) return fail(MOE_ERR_INVALID_ARG, "no workspace allocated yet");
    if (strcmp(name, "H") == 0)
        *ptr = h->h;
    else if (strcmp(name, "O") == 0)
        *ptr = h->o;
    else if (strcmp(name, "X8") == 0 || strcmp(name, "H8") == 0 || strcmp(name, "XS") == 0 ||
             strcmp(name, "HS") == 0) {
        if (!h->has_e4m3) return fail(MOE_ERR_INVALID_ARG, "no E4M3 workspace yet (no moe_forward_e4m3 call)");
        *ptr = name[0] == 'X' ? (name[1] == '8' ? static_cast<void*>(h->x8) : static_cast<void*>(h->xs))
                              : (name[1] == '8' ? static_cast<void*>(h->h8) : static_cast<void*>(h->hs));
    } else
        return fail(MOE_ERR_INVALID_ARG, "unknown workspace buffer '%s' (H, O, X8, XS, H8, HS)", name);
    *rows = h->R_cap;
    return ok();
}

moe_status moe_sync_status(moe_handle* h, moe_stream_t stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pending CUDA error");
    if (!h->status) return ok();
    int st = 0;
    e = cudaMemcpy(&st, h->status, sizeof st, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
    if (st != 0) {
        cudaMemset(h->status, 0, sizeof st);
        if (st == moe::kStatusEpPlan)
            return fail(MOE_ERR_INVALID_ARG,
                        "expert-parallel plan rejected: counts_all disagrees with this rank's routing or holds a "
                        "negative count, or a receive buffer has too few rows (status bits 0x%x)",
                        st);
        return fail(MOE_ERR_TIMEOUT, "a kernel gave up a bounded wait (status bits 0x%x)", st);
    }
    return ok();
}

moe_status moe_trace_begin(moe_handle* h, int max_calls) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (max_calls < 1 || max_calls > 100000)
        return fail(MOE_ERR_INVALID_ARG, "max_calls = %d outside [1, 100000]", max_calls);
    trace_free(h);
    h->trace_ev.resize(static_cast<size_t>(max_calls) * kTraceEvents, nullptr);
    for (auto& ev : h->trace_ev) {
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) {
            ev = nullptr;
            trace_free(h);
            return cuda_fail(e, "cudaEventCreate");
        }
    }
    h->trace_max = max_calls;
    h->trace_calls = 0;
    h->tracing = true;
    return ok();
}

moe_status moe_trace_end(moe_handle* h, double* stage_ms, int n_stages, int* calls) {
    if (!h || !stage_ms || !calls) return fail(MOE_ERR_INVALID_ARG, "null argument");
    if (!h->tracing) return fail(MOE_ERR_INVALID_ARG, "moe_trace_end without moe_trace_begin");
    if (n_stages < 1 || n_stages > kTraceStages)
        return fail(MOE_ERR_INVALID_ARG, "n_stages = %d outside [1, %d]", n_stages, kTraceStages);
    for (int s = 0; s < n_stages; ++s) stage_ms[s] = 0.0;
    for (int c = 0; c < h->trace_calls; ++c) {
        cudaEvent_t* ev = &h->trace_ev[static_cast<size_t>(c) * kTraceEvents];
        cudaError_t e = cudaEventSynchronize(ev[kTraceEvents - 1]);
        if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
        for (int s = 0; s < n_stages; ++s) {
            float ms = 0.f;
            e = cudaEventElapsedTime(&ms, ev[s], ev[s + 1]);
            if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
            stage_ms[s] += ms;
        }
    }
    *calls = h->trace_calls;
    trace_free(h);
    return ok();
}

moe_status moe_selftest_timeout(moe_handle* h, int budget_us, moe_stream_t stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "null handle");
    if (budget_us < 1 || budget_us > 1000000)
        return fail(MOE_ERR_INVALID_ARG, "budget_us = %d outside [1, 1000000]", budget_us);
    moe_status s = prepare(h, 1);
    if (s != MOE_OK) return s;
    int clk_khz = 0;
    cudaDeviceGetAttribute(&clk_khz, cudaDevAttrClockRate, h->device);
    if (clk_khz <= 0) clk_khz = 2000000;
    const long long budget = static_cast<long long>(budget_us) * clk_khz / 1000;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    moe::chain_begin();
    cudaError_t e = moe::launch_bounded_wait_probe(h->status, budget, st);
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    h->launches += 1;
    return ok();
}

moe_status moe_launch_count(moe_handle* h, int64_t* count) {
    if (!h || !count) return fail(MOE_ERR_INVALID_ARG, "null argument");
    *count = h->launches;
    return ok();
}

moe_status moe_destroy(moe_handle* h) {
    if (!h) return ok();
    trace_free(h);
    if (h->ws) cudaFree(h->ws);
    delete h;
    return ok();
}

const char* moe_last_error(void) { return g_err; }

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

}  // extern "C"
