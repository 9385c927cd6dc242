// topk.cuh -- one warp selects the top K of one token's logits and writes the
// softmax over the kept K ("Mixture of Experts: Why Mixtral Only Wakes Up Two
// Specialists", Part 3, Steps 2-3; the layer equation of "Mixtral of Experts"
// section 2.1).  Shared by router_topk_kernel and the fused tensor-core router
// so that both select and normalise with the same arithmetic.
#pragma once

#include "common.cuh"

namespace moe {

// Candidate key: larger key = larger logit, equal logits -> lower expert
// index (the low word holds the inverted index).  The float is mapped to an
// unsigned integer with the same order (sign bit set for non-negative values,
// all bits inverted for negative ones); -0 is folded into +0 first so that
// the two zeros tie like the comparison of their values.  0 = no candidate.
__device__ __forceinline__ uint64_t topk_key(float v, int e) {
    const uint32_t b = __float_as_uint(v + 0.0f);
    const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return (static_cast<uint64_t>(ord) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float topk_key_value(uint64_t key) {
    const uint32_t ord = static_cast<uint32_t>(key >> 32);
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
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int e = lane + 32 * i;
            const uint64_t key = (e < n && !((taken >> i) & 1u)) ? topk_key(v[i], e) : 0ull;
            best = key > best ? key : best;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
            best = other > best ? other : best;
        }
        const int bi = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(best));
        const float bv = topk_key_value(best);
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
