// Combine and load statistics.
//
// Combine: y[t] = sum_{k<K} w[t,k] * y_rows[inv[t*K+k]] (+ y_shared[t]),
// fp32 in that order, one rounding to the layer dtype ("Kimi K3 fine-grained
// MoE under high concurrency", section "物理通信拓扑", combine phase; "MoE
// architecture in production" §3.1, results scattered back to the original
// token order). No residual is added.
//
// Statistics ("Kimi K3 专家路由不均衡诊断" §三, analyze_batch_routing and
// compute_gini_coefficient): capacity floor(T*K*cf/E), max / min load, skew
// max/(min + 1e-5), overflow past capacity (counted, never dropped: §五),
// its rate over T*K, stragglers (count > capacity) and the Gini coefficient
// (2*sum_i i*c_(i) - (n+1)*S) / (n*S) with exact integers and one fp64
// division. sum_i i*c_(i) over the ascending order equals sum_j rank_j*c_j
// with rank_j = 1 + #{i: c_i < c_j} + #{i < j: c_i == c_j}; equal counts
// may swap ranks without changing the sum, so no sort is needed.
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

template <typename T>
struct CVec;
template <>
struct CVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const void* p, float* f) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 q = __bfloat1622float2(h[i]);
      f[2 * i] = q.x;
      f[2 * i + 1] = q.y;
    }
  }
  __device__ static void store(void* p, const float* f) {
    uint4 v;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = v;
  }
};
template <>
struct CVec<float> {
  static constexpr int N = 4;
  __device__ static void load(const void* p, float* f) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  }
  __device__ static void store(void* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

// Expert outputs are fp32; each thread sums V::N consecutive columns of one
// token and rounds once to the layer dtype T.
// Sum of n_parts partial rows (reduction splits of the second expert GEMM),
// added in split order.
template <int N>
__device__ __forceinline__ void load_parts(const float* src, int n_parts, size_t stride,
                                           float* v) {
  CVec<float>::load(src, v);
  for (int p0 = 1; p0 < n_parts; p0 += 4) {   // 4 independent loads, then in-order adds
    float u[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (p0 + q < n_parts) CVec<float>::load(src + (p0 + q) * stride, u[q]);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (p0 + q < n_parts)
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __fadd_rn(v[i], u[q][i]);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_rows,
                                                      int rows_parts, size_t rows_stride,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ y_shared,
                                                      int shared_parts, size_t shared_stride,
                                                      T* __restrict__ y, int T_, int H, int K) {
  pdl_wait();
  pdl_trigger();
  using V = CVec<T>;
  using F = CVec<float>;
  const int t = blockIdx.x;
  const int h = (blockIdx.y * blockDim.x + threadIdx.x) * V::N;
  if (t >= T_ || h >= H) return;
  float acc[V::N];
#pragma unroll
  for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
  const unsigned TK = (unsigned)T_ * (unsigned)K;
  for (int k = 0; k < K; ++k) {
    const int row = inv[(size_t)t * K + k];
    // a copy the dispatch could not place (inv = -1, reported in the
    // workspace status) contributes nothing
    if ((unsigned)row >= TK) continue;
    const float wk = w[(size_t)t * K + k];
    const float* src = y_rows + (size_t)row * H + h;
#pragma unroll
    for (int q = 0; q < V::N; q += F::N) {
      float v[F::N];
      load_parts<F::N>(src + q, rows_parts, rows_stride, v);
#pragma unroll
      for (int i = 0; i < F::N; ++i) acc[q + i] = fmaf(wk, v[i], acc[q + i]);
    }
  }
  if (y_shared) {
    const float* src = y_shared + (size_t)t * H + h;
#pragma unroll
    for (int q = 0; q < V::N; q += F::N) {
      float v[F::N];
      load_parts<F::N>(src + q, shared_parts, shared_stride, v);
#pragma unroll
      for (int i = 0; i < F::N; ++i) acc[q + i] += v[i];
    }
  }
  V::store(y + (size_t)t * H + h, acc);
}

cudaError_t launch_combine(const moe_layer_desc& d, const void* y_rows, const float* w,
                           const int32_t* inv, const void* y_shared, void* y, cudaStream_t st,
                           int rows_parts, int shared_parts) {
  if (d.T == 0) return cudaSuccess;
  const int vec = (d.dtype == MOE_BF16) ? 8 : 4;
  const int threads = 128;
  dim3 grid(d.T, (d.H / vec + threads - 1) / threads);
  const size_t rows_stride = (size_t)d.T * d.K * d.H, shared_stride = (size_t)d.T * d.H;
  if (d.dtype == MOE_BF16)
    return launch_pdl(combine_kernel<__nv_bfloat16>, grid, dim3(threads), 0, st,
                      (const float*)y_rows, rows_parts, rows_stride, w, inv,
                      (const float*)y_shared, shared_parts, shared_stride, (__nv_bfloat16*)y,
                      d.T, d.H, d.K);
  return launch_pdl(combine_kernel<float>, grid, dim3(threads), 0, st, (const float*)y_rows,
                    rows_parts, rows_stride, w, inv, (const float*)y_shared, shared_parts,
                    shared_stride, (float*)y, d.T, d.H, d.K);
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(512) expert_stats_kernel(const int32_t* __restrict__ counts,
                                                           int E, long long TK, int capacity,
                                                           uint8_t* __restrict__ mask,
                                                           moe_stats* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  __shared__ int c[kMaxE];
  __shared__ long long red[6][16];
  const int j = threadIdx.x;
  for (int i = j; i < E; i += blockDim.x) c[i] = counts[i];
  __syncthreads();
  long long v_max = LLONG_MIN, v_min = LLONG_MAX, v_over = 0, v_strag = 0, v_sum = 0, v_rank = 0;
  for (int i = j; i < E; i += blockDim.x) {
    const int ci = c[i];
    v_max = max(v_max, (long long)ci);
    v_min = min(v_min, (long long)ci);
    v_over += max(0, ci - capacity);
    v_strag += (ci > capacity) ? 1 : 0;
    v_sum += ci;
    long long rank = 1;
    for (int q = 0; q < E; ++q) rank += (c[q] < ci) || (c[q] == ci && q < i);
    v_rank += rank * (long long)ci;
    if (mask) mask[i] = (ci > capacity) ? 1 : 0;
  }
  const int lane = j & 31, warp = j >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    v_max = max(v_max, __shfl_xor_sync(0xffffffffu, v_max, o));
    v_min = min(v_min, __shfl_xor_sync(0xffffffffu, v_min, o));
    v_over += __shfl_xor_sync(0xffffffffu, v_over, o);
    v_strag += __shfl_xor_sync(0xffffffffu, v_strag, o);
    v_sum += __shfl_xor_sync(0xffffffffu, v_sum, o);
    v_rank += __shfl_xor_sync(0xffffffffu, v_rank, o);
  }
  if (lane == 0) {
    red[0][warp] = v_max; red[1][warp] = v_min; red[2][warp] = v_over;
    red[3][warp] = v_strag; red[4][warp] = v_sum; red[5][warp] = v_rank;
  }
  __syncthreads();
  if (j == 0) {
    const int nw = blockDim.x >> 5;
    long long mx = LLONG_MIN, mn = LLONG_MAX, over = 0, strag = 0, S = 0, R = 0;
    for (int w = 0; w < nw; ++w) {
      mx = max(mx, red[0][w]); mn = min(mn, red[1][w]); over += red[2][w];
      strag += red[3][w]; S += red[4][w]; R += red[5][w];
    }
    moe_stats s;
    s.num_copies = TK;
    s.overflow = over;
    s.capacity = capacity;
    s.max_load = (int)mx;
    s.min_load = (int)mn;
    s.num_stragglers = (int)strag;
    s.skew_ratio = (double)mx / ((double)mn + 1e-5);
    const long long n = E;
    s.gini = (S == 0) ? 0.0 : (double)(2 * R - (n + 1) * S) / (double)(n * S);
    s.overflow_rate = (TK == 0) ? 0.0 : (double)over / (double)TK;
    s.max_over_mean = (TK == 0) ? 0.0 : (double)mx * (double)n / (double)TK;
    *out = s;
  }
}

cudaError_t launch_expert_stats(const moe_layer_desc& d, const int32_t* counts, uint8_t* mask,
                                moe_stats* out_dev, cudaStream_t st) {
  const long long TK = (long long)d.T * d.K;
  const long long cap = TK * d.cf_num / ((long long)d.E * d.cf_den);
  count_launch();
  expert_stats_kernel<<<1, 512, 0, st>>>(counts, d.E, TK, (int)cap, mask, out_dev);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Dynamic expert bias update ("Kimi K3 专家路由不均衡诊断" §四): an expert that
// stayed overloaded over the caller's period (accumulated count > capacity)
// has its bias lowered by gamma, an idle one (count == 0) raised by gamma,
// in fp32; the others keep theirs.
__global__ void __launch_bounds__(512) bias_update_kernel(const int32_t* __restrict__ counts,
                                                          float* __restrict__ bias, int E,
                                                          long long capacity, float gamma) {
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long c = counts[e];
    float b = bias[e];
    if (c > capacity)
      b = __fsub_rn(b, gamma);
    else if (c == 0)
      b = __fadd_rn(b, gamma);
    bias[e] = b;
  }
}

cudaError_t launch_bias_update(const moe_layer_desc& d, const int32_t* counts, float* bias,
                               float gamma, cudaStream_t st) {
  const long long TK = (long long)d.T * d.K;
  const long long cap = TK * d.cf_num / ((long long)d.E * d.cf_den);
  return launch_pdl(bias_update_kernel, dim3(1), dim3(512), 0, st, counts, bias, d.E, cap, gamma);
}

}  // namespace moe
