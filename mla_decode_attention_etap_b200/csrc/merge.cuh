#pragma once
// Log-sum-exp merge of split-KV partial results (the split-KV combine step of the ETAP
// decode; FlashAttention-style split merge).  Shared by the stand-alone combine kernel and by
// the decode kernel's in-kernel merge, so that both produce bit-identical outputs.

#include <cstdint>

namespace mla {

// Merged LSE of one output column over its nsplit partial LSEs l(0..nsplit-1):
// lse = mx + ln(sum_s exp(l_s - mx)); -inf when every split is empty.
template <class L>
__device__ __forceinline__ float merged_lse(L l, int nsplit) {
    float mx = -INFINITY;
#pragma unroll 8
    for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, l(s));
    if (mx == -INFINITY) return -INFINITY;
    float sum = 0.f;
#pragma unroll 8
    for (int s = 0; s < nsplit; ++s) sum += expf(l(s) - mx);
    return mx + logf(sum);
}

// Weight of a split with partial LSE l_s in the merged output: exp(l_s - lse).
__device__ __forceinline__ float merge_weight(float l_s, float lse) { return expf(l_s - lse); }

}  // namespace mla
