// Grouped expert GEMM on CUDA cores (fp32 FFMA), used for MOE_F32 layers.
//
// Each expert is Linear -> GeLU -> Linear ("MoE architecture in production"
// §3.1). Work is a list of tiles (group, first row, rows); a CTA computes
// 64 rows x 64 output columns of one group with a 32-deep reduction step.
// GEMM1 reads token rows through the dispatch permutation (row r of the
// routed buffer is token perm[r] / K) and applies the exact GeLU; GEMM2
// reads the GEMM1 rows directly. The shared expert is group E.
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

constexpr int kBM = kSimtRows;   // rows per tile
constexpr int kBN = 64;          // output columns per tile
constexpr int kBK = 32;          // reduction step

template <typename TIn, typename TOut, bool kGelu>
__global__ void __launch_bounds__(256) grouped_gemm_simt(const Tile* __restrict__ tiles,
                                                         const int* __restrict__ n_tiles,
                                                         SimtProblem routed, SimtProblem shared,
                                                         int E) {
  pdl_wait();
  pdl_trigger();
  const int tile_id = blockIdx.x;
  if (tile_id >= *n_tiles) return;
  const Tile tl = tiles[tile_id];
  const SimtProblem& P = (tl.g < E) ? routed : shared;
  const int col0 = blockIdx.y * kBN;
  if (col0 >= P.N) return;
  const TIn* A = static_cast<const TIn*>(P.A);
  const TIn* B = static_cast<const TIn*>(P.B) + (tl.g < E ? (size_t)tl.g * P.b_group_stride : 0);
  TOut* C = static_cast<TOut*>(P.C);
  const int Kd = P.Kd;

  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  __shared__ int arow[kBM];
  if (threadIdx.x < kBM) {
    const int r = tl.r0 + threadIdx.x;
    int a = -1;
    if (threadIdx.x < tl.n) a = P.perm ? P.perm[r] / P.k_top : r;
    arow[threadIdx.x] = a;
  }
  __syncthreads();

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads, 4x4 outputs each
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < Kd; k0 += kBK) {
    // A tile: 64 rows x 32 k; B tile: 64 weight rows x 32 k (both k-contiguous in memory)
    for (int i = threadIdx.x; i < kBM * kBK; i += 256) {
      const int r = i / kBK, k = i % kBK;
      const int a = arow[r];
      float v = 0.f;
      if (a >= 0 && k0 + k < Kd) v = to_f32(A[(size_t)a * Kd + k0 + k]);
      As[k][r] = v;
    }
    for (int i = threadIdx.x; i < kBN * kBK; i += 256) {
      const int n = i / kBK, k = i % kBK;
      float v = 0.f;
      if (col0 + n < P.N && k0 + k < Kd) v = to_f32(B[(size_t)(col0 + n) * Kd + k0 + k]);
      Bs[k][n] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kBK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r >= tl.n) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = col0 + tx * 4 + j;
      if (n >= P.N) continue;
      float v = acc[i][j];
      if (kGelu) v = gelu_erf(v);
      C[(size_t)(tl.r0 + r) * P.N + n] = from_f32<TOut>(v);
    }
  }
}

template <typename TIn, typename TOut, bool kGelu>
static cudaError_t launch_simt_t(const SimtProblem& routed, const SimtProblem& shared, int E,
                                 const Tile* tiles, const int* n_tiles, int max_tiles, int max_n,
                                 cudaStream_t st) {
  if (max_tiles <= 0) return cudaSuccess;
  dim3 grid(max_tiles, (max_n + kBN - 1) / kBN);
  return launch_pdl(grouped_gemm_simt<TIn, TOut, kGelu>, grid, dim3(256), 0, st, tiles, n_tiles,
                    routed, shared, E);
}

// First layer: output in the input dtype with GeLU; second layer: fp32
// output without activation.
cudaError_t launch_grouped_gemm_simt(int dtype, bool first_layer, const SimtProblem& routed,
                                     const SimtProblem& shared, int E, const Tile* tiles,
                                     const int* n_tiles, int max_tiles, int max_n,
                                     cudaStream_t st) {
  if (dtype == MOE_BF16) {
    return first_layer
               ? launch_simt_t<__nv_bfloat16, __nv_bfloat16, true>(routed, shared, E, tiles,
                                                                   n_tiles, max_tiles, max_n, st)
               : launch_simt_t<__nv_bfloat16, float, false>(routed, shared, E, tiles, n_tiles,
                                                            max_tiles, max_n, st);
  }
  return first_layer
             ? launch_simt_t<float, float, true>(routed, shared, E, tiles, n_tiles, max_tiles,
                                                 max_n, st)
             : launch_simt_t<float, float, false>(routed, shared, E, tiles, n_tiles, max_tiles,
                                                  max_n, st);
}

}  // namespace moe
