// topk.cuh -- one warp selects the top K of one token's logits and writes the
// softmax over the kept K ("Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists", Part 3, Steps 2-3; the layer equation of "Mixtral of Experts"
// section 2.1).  Shared by router_topk_kernel and the fused tensor-core router
// so that both select and normalise with the same arithmetic.
#pragma once

#include "common.cuh"

namespace moe {

// Order key of a logit: an unsigned integer with the same order as the
// value (sign bit set for non-negative values, all bits inverted for negative
// ones); -0 is folded into +0 first so that the two zeros tie like the
// comparison of their values.  Every finite or infinite value maps above 0, so
// 0 means "no candidate".
__device__ __forceinline__ uint32_t topk_ord(float v) {
    const uint32_t b = __float_as_uint(v + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float topk_ord_value(uint32_t ord) {
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}

// v[i] holds the logit of expert lane + 32 i, i < NS (NaN already mapped to
// -inf).  Order: descending logit, equal logits keep the lower expert index
// first.  Gates: ex_k = exp(L_k - L_0), w_k = ex_k * (1 / sum_j ex_j), the
// sum taken in k order.  Writes idx_out[0..K) and w_out[0..K).
template <int NS>
__device__ __forceinline__ void warp_topk_softmax(const float (&v)[NS], int n, int K, int lane,
                                                  int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
    uint32_t taken = 0;  // bit i: slot i of this lane already chosen
    float m = 0.f, s = 0.f;
    int my_idx = 0;      // selection `lane` (K <= 32)
    float my_ex = 0.f;
    for (int k = 0; k < K; ++k) {
        // this lane's best untaken slot (slots ascend in expert index, so the
        // strict '>' keeps the lower index on equal keys), then the warp's
        // largest key and, among the lanes holding it, the lowest index
        uint32_t best = 0;
        int best_e = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int e = lane + 32 * i;
            const uint32_t key = (e < n && !((taken >> i) & 1u)) ? topk_ord(v[i]) : 0u;
            if (key > best) {
                best = key;
                best_e = e;
            }
        }
        const uint32_t top = __reduce_max_sync(0xffffffffu, best);
        const int bi = static_cast<int>(
            __reduce_min_sync(0xffffffffu, best == top ? static_cast<uint32_t>(best_e) : 0x7FFFFFFFu));
        const float bv = topk_ord_value(top);
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (k == 0) m = bv;
        const float ex = expf(bv - m);
        s += ex;
        if (K <= 32) {
            if (lane == k) {
                my_idx = bi;
                my_ex = ex;
            }
        } else if (lane == 0) {
            idx_out[k] = bi;
            w_out[k] = ex;
        }
    }
    const float inv = 1.f / s;
    if (K <= 32) {
        if (lane < K) {
            idx_out[lane] = my_idx;
            w_out[lane] = my_ex * inv;
        }
    } else if (lane == 0) {
        for (int k = 0; k < K; ++k) w_out[k] *= inv;
    }
}

}  // namespace moe
