// dispatch_noalloc.cu -- moe_dispatch_noalloc: the dispatch (per-expert
// segments of the (token, slot) pairs) for callers that must not allocate
// device memory.
//
// Who needs it: a caller whose device memory is owned by someone else (a
// framework's caching allocator or a fixed memory plan that every buffer must
// come from), or a caller that cannot afford cudaMalloc's implicit
// device-wide synchronisation in the middle of its work.  The regular entry
// points keep their scratch in a per-handle workspace that they cudaMalloc on
// first use; this one keeps it in a fixed array compiled into the library.
//
// The scratch (per-block expert counts, in-block ranks and the M-block prefix)
// lives in g_noalloc_scratch below: a file-scope device array that every GPU
// which loads the library holds until the process exits.  It bounds the call
// to kNoAllocMaxPairs = 65,536 (token, slot) pairs, i.e. T * K <= 65,536.
// All calls share it and it keeps the previous call's contents; the kernels
// overwrite every entry they read before reading it, so nothing needs
// clearing, but two calls that overlap on the GPU (different streams without
// ordering, or different host threads) race on it.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

constexpr int64_t kNoAllocMaxPairs = 65536;
constexpr int kNoAllocMaxBlocks =
    static_cast<int>((kNoAllocMaxPairs + moe::kPairsPerBlock - 1) / moe::kPairsPerBlock);
constexpr int kNoAllocMaxExperts = 256;
// int32 words: blockcounts [max blocks][max experts], pair_rank [max pairs],
// M-block prefix [max experts + 1] (rounded up to 512 words).
constexpr size_t kBlockcountsWords = static_cast<size_t>(kNoAllocMaxBlocks) * kNoAllocMaxExperts;
constexpr size_t kPairRankWords = static_cast<size_t>(kNoAllocMaxPairs);
constexpr size_t kMblkWords = 512;
constexpr size_t kScratchWords = kBlockcountsWords + kPairRankWords + kMblkWords;

static __device__ __align__(256) int32_t g_noalloc_scratch[kScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_device_checked[kMaxDevices] = {};

thread_local char g_msg[256];

}  // namespace

// Defined in moe_api.cu: records the message returned by moe_last_error().
namespace moe_api_detail {
void set_last_error(const char* msg);
}

namespace {

moe_status set_error(moe_status s, const char* msg) {
    moe_api_detail::set_last_error(msg);
    return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device, looked up with
// cudaGetSymbolAddress on every call (with that device current).  The lookup
// allocates nothing once the library's module is loaded on the device, and
// doing it each time keeps the address right after a device reset reloads
// the module.  Only the device check is cached.
moe_status scratch_for_current_device(int32_t** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        snprintf(g_msg, sizeof g_msg, "cudaGetDevice: %s", cudaGetErrorString(e));
        return set_error(MOE_ERR_CUDA, g_msg);
    }
    if (dev < 0 || dev >= kMaxDevices) return set_error(MOE_ERR_UNSUPPORTED, "device index out of range");
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_device_checked[dev]) {
            int major = 0, minor = 0;
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
            if (major != 10 || minor != 0) {
                snprintf(g_msg, sizeof g_msg, "device %d is sm_%d%d; this library is built for sm_100a",
                         dev, major, minor);
                return set_error(MOE_ERR_UNSUPPORTED, g_msg);
            }
            g_device_checked[dev] = true;
        }
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
        snprintf(g_msg, sizeof g_msg, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
        return set_error(MOE_ERR_CUDA, g_msg);
    }
    *out = static_cast<int32_t*>(p);
    return MOE_OK;
}

}  // namespace

extern "C" MOE_API moe_status moe_dispatch_noalloc(int64_t T, int n, int K, const int32_t* topk_idx,
                                                   int32_t* counts, int32_t* offsets,
                                                   int32_t* row_token, int32_t* token_row,
                                                   moe_stream_t stream) {
    if (n < 1 || n > kNoAllocMaxExperts) return set_error(MOE_ERR_INVALID_ARG, "n outside [1, 256]");
    if (K < 1 || K > n) return set_error(MOE_ERR_INVALID_ARG, "K outside [1, n]");
    if (T < 0) return set_error(MOE_ERR_INVALID_ARG, "T < 0");
    // T > max / K, not T * K > max: the product of a huge T would overflow
    if (T > kNoAllocMaxPairs / K) {
        snprintf(g_msg, sizeof g_msg,
                 "T = %lld with K = %d exceeds the %lld (token, slot) pairs moe_dispatch_noalloc's "
                 "fixed scratch holds; use moe_dispatch",
                 static_cast<long long>(T), K, static_cast<long long>(kNoAllocMaxPairs));
        return set_error(MOE_ERR_INVALID_ARG, g_msg);
    }
    if (T == 0) return set_error(MOE_OK, "");
    const void* ptrs[5] = {topk_idx, counts, offsets, row_token, token_row};
    const char* names[5] = {"topk_idx", "counts", "offsets", "row_token", "token_row"};
    for (int i = 0; i < 5; ++i) {
        if (!ptrs[i]) {
            snprintf(g_msg, sizeof g_msg, "%s is NULL", names[i]);
            return set_error(MOE_ERR_INVALID_ARG, g_msg);
        }
        if (!aligned16(ptrs[i])) {
            snprintf(g_msg, sizeof g_msg, "%s is not 16-byte aligned", names[i]);
            return set_error(MOE_ERR_INVALID_ARG, g_msg);
        }
    }
    int32_t* scratch = nullptr;
    moe_status s = scratch_for_current_device(&scratch);
    if (s != MOE_OK) return s;
    moe::DispatchBufs b{};
    b.blockcounts = scratch;
    b.pair_rank = scratch + kBlockcountsWords;
    b.mblk_base = scratch + kBlockcountsWords + kPairRankWords;
    b.counts = counts;
    b.offsets = offsets;
    b.row_token = row_token;
    b.token_row = token_row;
    moe::chain_begin();
    cudaError_t e = moe::launch_dispatch(topk_idx, T, K, n, moe::kTcBM, b,
                                         reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        snprintf(g_msg, sizeof g_msg, "dispatch launch: %s", cudaGetErrorString(e));
        return set_error(MOE_ERR_CUDA, g_msg);
    }
    return set_error(MOE_OK, "");
}
