// Top-K selection of one token by one warp ("Kimi K3 fine-grained MoE under
// high concurrency", FineGrainedMoERouter: softmax, top-k, renormalise;
// "Kimi K3 专家路由不均衡诊断" §四: scores Softmax(Logits + B)). Lane j holds
// the scores s = l + B of experts j, j+32, ...; K rounds of a warp arg-max
// (warp reductions over order-preserving keys) pick the experts in the order
// (score descending, expert index ascending), so ties go to the lower index
// and -0.0 == +0.0. The weights are
// w_k = exp(s_k - s_0) / sum_{j<K} exp(s_j - s_0), summed in slot order (the
// full softmax denominator cancels in the renormalisation).
#pragma once

#include "common.cuh"

namespace moe {

// Order-preserving 32-bit key of an fp32 score: a > b as floats iff
// key(a) > key(b); -0.0 and +0.0 get the same key (they tie). NaN scores are
// not supported.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if (u == 0x80000000u) u = 0u;   // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// s[j]: score of expert lane + 32 j (-inf past E). Writes idx_out[0..K) and
// w_out[0..K) from lanes 0..K-1. Each of the K rounds takes the best
// untaken score of every lane (its lowest expert on ties), the warp's
// largest key with one reduction, and the lowest expert index among the
// lanes that hold it with a second one.
template <int NJ>
__device__ __forceinline__ void select_topk_warp(const float (&s)[NJ], int E, int K,
                                                 int32_t* __restrict__ idx_out,
                                                 float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) key[j] = (lane + 32 * j < E) ? score_key(s[j]) : 0u;
  uint32_t taken = 0;
  float my_s = -INFINITY;   // score of slot `lane` (lane < K)
  int my_e = 0;
  for (int k = 0; k < K; ++k) {
    uint32_t bk = 0u;       // below the key of any score, -inf included
    float bs = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (!((taken >> j) & 1u) && key[j] > bk) {   // ascending e: the first of equals stays
        bk = key[j];
        bs = s[j];
        be = lane + 32 * j;
      }
    }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const int e = __reduce_min_sync(0xffffffffu, (bk == m) ? be : 0x7fffffff);
    const float sc = __shfl_sync(0xffffffffu, bs, e & 31);
    if ((e & 31) == lane) taken |= 1u << (e >> 5);
    if (lane == k) {
      my_s = sc;
      my_e = e;
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
