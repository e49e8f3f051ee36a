// Router: gate logits and the top-K selection with renormalised weights.
//
// Gate: l = x W_r^T, a bias-free Linear(H, E) ("Kimi K3 fine-grained MoE
// under high concurrency", FineGrainedMoERouter; "MoE architecture in
// production" §2.3). Selection: scores Softmax(l + B) with the dynamic
// expert bias B ("Kimi K3 专家路由不均衡诊断" §四), the top K of them, and
// the K weights divided by their sum (same router code). The decision is
// taken on the fp32 values s = l + B: softmax is strictly increasing, so the
// chosen set is the same, and ties stay exact ties (lower expert index wins).
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"
#include "select.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Gate logits on CUDA cores: one warp per expert row, 8 experts x 8 tokens
// per CTA. W_r rows are read once per token block; x rows come from L2.
// ---------------------------------------------------------------------------
template <typename TIn>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  using T = float4;
  __device__ static void unpack(const T& v, float* f) { f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w; }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  using T = uint4;
  __device__ static void unpack(const T& v, float* f) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 q = __bfloat1622float2(p[i]);
      f[2 * i] = q.x;
      f[2 * i + 1] = q.y;
    }
  }
};

constexpr int kGateTok = 8;   // tokens per CTA
constexpr int kGateExp = 8;   // experts per CTA (one per warp)

template <typename TIn>
__global__ void __launch_bounds__(256) gate_logits_simt(const TIn* __restrict__ x,
                                                        const TIn* __restrict__ wr,
                                                        float* __restrict__ logits, int T,
                                                        int H, int E) {
  pdl_wait();
  pdl_trigger();
  using V = Vec<TIn>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * kGateExp + warp;
  const int t0 = blockIdx.y * kGateTok;
  if (e >= E) return;
  float acc[kGateTok];
#pragma unroll
  for (int i = 0; i < kGateTok; ++i) acc[i] = 0.f;
  const TIn* wrow = wr + (size_t)e * H;
  for (int h = lane * V::N; h < H; h += 32 * V::N) {
    float wv[V::N], xv[V::N];
    V::unpack(*reinterpret_cast<const typename V::T*>(wrow + h), wv);
#pragma unroll
    for (int i = 0; i < kGateTok; ++i) {
      const int t = t0 + i;
      if (t < T) {
        V::unpack(*reinterpret_cast<const typename V::T*>(x + (size_t)t * H + h), xv);
#pragma unroll
        for (int j = 0; j < V::N; ++j) acc[i] = fmaf(xv[j], wv[j], acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kGateTok; ++i) {
    float v = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    acc[i] = v;
  }
  if (lane < kGateTok && t0 + lane < T) {
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < kGateTok; ++i)
      if (i == lane) v = acc[i];
    logits[(size_t)(t0 + lane) * E + e] = v;
  }
}

// ---------------------------------------------------------------------------
// Top-K selection kernel: one warp per token (the selection itself is in
// select.cuh).
// ---------------------------------------------------------------------------
// lrow: the token's logits, given as n_parts partial sums part_stride apart
// (reduction splits of the gate GEMM), added in split order; the total is
// written to logits_out when it is non-null. grow (nullable): the token's
// Gumbel noise for noisy routing ("MoE architecture in production" §2.3),
// added in fp32 after the bias: s = (l + B) + g.
template <int NJ>
__device__ __forceinline__ void select_row(const float* __restrict__ lrow, int n_parts,
                                           size_t part_stride, const float* __restrict__ bias,
                                           const float* __restrict__ grow, int E, int K,
                                           int32_t* __restrict__ idx_out,
                                           float* __restrict__ w_out,
                                           float* __restrict__ logits_out) {
  const int lane = threadIdx.x & 31;
  // Sum of the n_parts partial logits (reduction splits of the gate GEMM)
  // in split order. The loads of kPB parts for all NJ slots are issued
  // before any add, so the partial sums cost one round trip per kPB parts
  // (the router uses at most 16 splits).
  constexpr int kPB = (NJ >= 16) ? 4 : (NJ >= 8 ? 8 : 16);
  float l[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    l[j] = (e < E) ? lrow[e] : 0.f;
  }
  for (int p0 = 1; p0 < n_parts; p0 += kPB) {
    float v[kPB][NJ];
#pragma unroll
    for (int q = 0; q < kPB; ++q)
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = lane + 32 * j;
        v[q][j] = (p0 + q < n_parts && e < E) ? lrow[(p0 + q) * part_stride + e] : 0.f;
      }
#pragma unroll
    for (int q = 0; q < kPB; ++q)
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        if (p0 + q < n_parts) l[j] = __fadd_rn(l[j], v[q][j]);
  }
  float s[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    if (e < E) {
      if (logits_out) logits_out[e] = l[j];
      const float b = bias ? bias[e] : 0.f;
      s[j] = __fadd_rn(l[j], b);
      if (grow) s[j] = __fadd_rn(s[j], grow[e]);   // Gumbel noise, after the bias
    } else {
      s[j] = -INFINITY;
    }
  }
  select_topk_warp<NJ>(s, E, K, idx_out, w_out);
}

template <int NJ>
__global__ void __launch_bounds__(256) topk_select_kernel(const float* __restrict__ logits,
                                                          int n_parts, size_t part_stride,
                                                          const float* __restrict__ bias,
                                                          const float* __restrict__ noise, int T,
                                                          int E, int K,
                                                          int32_t* __restrict__ idx,
                                                          float* __restrict__ w,
                                                          float* __restrict__ logits_out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  select_row<NJ>(logits + (size_t)t * E, n_parts, part_stride, bias,
                 noise ? noise + (size_t)t * E : nullptr, E, K, idx + (size_t)t * K,
                 w + (size_t)t * K, logits_out ? logits_out + (size_t)t * E : nullptr);
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
cudaError_t launch_gate_logits(const moe_layer_desc& d, const void* x, const void* wr,
                               float* logits, cudaStream_t st) {
  if (d.T == 0) return cudaSuccess;
  dim3 grid((d.E + kGateExp - 1) / kGateExp, (d.T + kGateTok - 1) / kGateTok);
  if (d.dtype == MOE_BF16)
    return launch_pdl(gate_logits_simt<__nv_bfloat16>, grid, dim3(256), 0, st,
                      (const __nv_bfloat16*)x, (const __nv_bfloat16*)wr, logits, d.T, d.H, d.E);
  return launch_pdl(gate_logits_simt<float>, grid, dim3(256), 0, st, (const float*)x,
                    (const float*)wr, logits, d.T, d.H, d.E);
}

// Gate GEMM of bf16 layers on the tensor cores: W_r is operand A (expert
// rows, one or more 128-row blocks; rows past E are zero-filled by TMA and
// their outputs are not stored), x is operand B (token rows). With several
// reduction splits each split writes its own fp32 partial [T, E]; the
// selection kernel adds them in split order.
cudaError_t launch_gate_logits_tc(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                  const void* x, const void* wr, float* parts, int num_sms,
                                  cudaStream_t st) {
  if (d.T == 0) return cudaSuccess;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
  TcProblem p{};
  p.act = x;
  p.act_rows = (uint64_t)d.T;
  p.w = wr;
  p.w_rows = (uint64_t)d.E;
  p.m_rows = d.E;
  p.kd = d.H;
  p.out = parts;
  p.ld = d.E;
  p.out_f32 = true;
  p.splits = L.sp.router;
  p.split_stride = (long long)d.T * d.E;
  p.m_valid = d.E;
  DenseTiling dense;
  dense.rows = d.T;
  dense.m_tiles = (d.E + 127) / 128;
  dense.tiles = ((d.T + kTcRows - 1) / kTcRows) * dense.m_tiles * L.sp.router;
  return launch_grouped_gemm_tc(p, TcProblem{}, d.E, false, nullptr, nullptr, &dense,
                                /*pair=*/false, &hdr->status, num_sms, st);
}

cudaError_t launch_topk_select(const moe_layer_desc& d, const float* logits, int n_parts,
                               size_t part_stride, const float* bias, const float* noise,
                               int32_t* idx, float* w, float* logits_out, cudaStream_t st) {
  if (d.T == 0) return cudaSuccess;
  const int nj = (d.E + 31) / 32;
  dim3 grid((d.T + 7) / 8);
#define MOE_TOPK_CASE(NJ)                                                                    \
  case NJ:                                                                                   \
    return launch_pdl(topk_select_kernel<NJ>, grid, dim3(256), 0, st, logits, n_parts,       \
                      part_stride, bias, noise, d.T, d.E, d.K, idx, w, logits_out);
  switch (nj) {
    MOE_TOPK_CASE(1) MOE_TOPK_CASE(2) MOE_TOPK_CASE(3) MOE_TOPK_CASE(4)
    MOE_TOPK_CASE(5) MOE_TOPK_CASE(6) MOE_TOPK_CASE(7) MOE_TOPK_CASE(8)
    MOE_TOPK_CASE(9) MOE_TOPK_CASE(10) MOE_TOPK_CASE(11) MOE_TOPK_CASE(12)
    MOE_TOPK_CASE(13) MOE_TOPK_CASE(14) MOE_TOPK_CASE(15) MOE_TOPK_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef MOE_TOPK_CASE
  return cudaGetLastError();
}

}  // namespace moe
