// Top-K selection of one token by one warp ("Kimi K3 fine-grained MoE under
// high concurrency", FineGrainedMoERouter: softmax, top-k, renormalise;
// "Kimi K3 专家路由不均衡诊断" §四: scores Softmax(Logits + B)). Lane j holds
// the scores s = l + B of experts j, j+32, ...; K rounds of a warp arg-max
// by shuffles pick the experts in the order (score descending, expert index
// ascending), so ties go to the lower index and -0.0 == +0.0. The weights are
// w_k = exp(s_k - s_0) / sum_{j<K} exp(s_j - s_0), summed in slot order (the
// full softmax denominator cancels in the renormalisation).
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ bool better(float sa, int ea, float sb, int eb) {
  return sa > sb || (sa == sb && ea < eb);
}

// s[j]: score of expert lane + 32 j (-inf past E). Writes idx_out[0..K) and
// w_out[0..K) from lanes 0..K-1.
template <int NJ>
__device__ __forceinline__ void select_topk_warp(const float (&s)[NJ], int E, int K,
                                                 int32_t* __restrict__ idx_out,
                                                 float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;
  float my_s = -INFINITY;   // score of slot `lane` (lane < K)
  int my_e = 0;
  for (int k = 0; k < K; ++k) {
    float bs = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u) && better(s[j], e, bs, be)) {
        bs = s[j];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (better(os, oe, bs, be)) {
        bs = os;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == k) {
      my_s = bs;
      my_e = be;
    }
  }
  // w_k = exp(s_k - s_0) / sum_{j<K} exp(s_j - s_0), summed in slot order.
  const float s0 = __shfl_sync(0xffffffffu, my_s, 0);
  const float z = (lane < K) ? expf(my_s - s0) : 0.f;
  float den = 0.f;
  for (int j = 0; j < K; ++j) den += __shfl_sync(0xffffffffu, z, j);
  if (lane < K) {
    idx_out[lane] = my_e;
    w_out[lane] = z / den;
  }
}


}  // namespace moe
