// Expert-parallel helpers: the row gather that fills an All-to-All send
// buffer (or puts the returned expert outputs back in order), and the order
// of the rows one rank receives ("Kimi K3 fine-grained MoE under high
// concurrency", section "物理通信拓扑": dispatch All-to-All -> local experts ->
// combine All-to-All; "MoE architecture in production" §3.2, experts placed
// on different GPUs).
//
// A rank owns a contiguous range of El experts. From source rank s it
// receives, for each of its experts e in ascending order, cnt[s][e] rows
// (the source's dispatch order, ascending copy index inside an expert), all
// of source 0's rows first, then source 1's, ... The grouped expert FFN wants
// the rows of one expert together: expert-major order puts expert e's rows
// of source 0, then of source 1, ... contiguously.
#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

constexpr int kEpMaxCells = 4096;   // G * El (the counts and two tables fit in shared memory)

__global__ void __launch_bounds__(1024) ep_local_order_kernel(const int32_t* __restrict__ cnt,
                                                              int G, int El,
                                                              int32_t* __restrict__ offsets,
                                                              int32_t* __restrict__ perm,
                                                              int32_t* __restrict__ inv,
                                                              int capacity) {
  __shared__ int32_t c[kEpMaxCells];        // counts, then each cell's source-side start
  __shared__ int32_t em[kEpMaxCells];       // each cell's expert-major start
  __shared__ int32_t base_s[1024];          // first row of each source in the receive buffer
  __shared__ int32_t base_e[1025];          // first row of each expert in expert-major order
  const int tid = threadIdx.x, n = G * El;
  for (int i = tid; i < n; i += blockDim.x) c[i] = cnt[i];
  __syncthreads();
  // rows of each source and of each expert (one thread each)
  if (tid < G) {
    int run = 0;
    for (int e = 0; e < El; ++e) run += c[tid * El + e];
    base_s[tid] = run;
  }
  if (tid < El) {
    int run = 0;
    for (int s = 0; s < G; ++s) {
      em[s * El + tid] = run;               // this source's rows of the expert before
      run += c[s * El + tid];
    }
    base_e[tid] = run;
  }
  __syncthreads();
  if (tid == 0) {
    // exclusive prefix sums over sources and experts (G, El <= 1024)
    int run = 0;
    for (int s = 0; s < G; ++s) {
      const int v = base_s[s];
      base_s[s] = run;
      run += v;
    }
    run = 0;
    for (int e = 0; e < El; ++e) {
      const int v = base_e[e];
      base_e[e] = run;
      run += v;
    }
    base_e[El] = run;
  }
  __syncthreads();
  if (tid < G) {                            // source-side start of each cell
    int run = base_s[tid];
    for (int e = 0; e < El; ++e) {
      const int v = c[tid * El + e];
      c[tid * El + e] = run;
      run += v;
    }
  }
  for (int e = tid; e <= El; e += blockDim.x) offsets[e] = base_e[e];
  __syncthreads();
  // expand the cells: one warp per cell, lanes over its rows
  const int warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
  for (int cell = warp; cell < n; cell += nwarps) {
    const int s = cell / El, e = cell % El;
    const int src = c[cell];
    const int rows = cnt[cell];
    const int dst = base_e[e] + em[cell];
    // rows past the caller's buffers (counts that do not add up) are not written
    if (perm && inv)
      for (int i = lane; i < rows; i += 32)
        if (dst + i < capacity && src + i < capacity) {
          perm[dst + i] = src + i;
          inv[src + i] = dst + i;
        }
    (void)s;
  }
}

cudaError_t launch_ep_local_order(const int32_t* cnt, int G, int El, int32_t* offsets,
                                  int32_t* perm, int32_t* inv, int capacity, cudaStream_t st) {
  count_launch();
  ep_local_order_kernel<<<1, 1024, 0, st>>>(cnt, G, El, offsets, perm, inv, capacity);
  return cudaGetLastError();
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_gather_rows(const void* src, int64_t src_rows, const int32_t* idx,
                                      int32_t divisor, int64_t n_rows, int64_t row_bytes,
                                      void* dst, moe_stream stream) {
  if (n_rows < 0 || src_rows < 0 || divisor < 1 || row_bytes < 16 || row_bytes % 16)
    return MOE_ERR_INVALID_ARG;
  if (n_rows == 0) return MOE_OK;
  if (!src || !idx || !dst) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u)
    return MOE_ERR_INVALID_ARG;
  if (n_rows > INT_MAX || row_bytes / 16 > INT_MAX || src_rows * divisor > INT_MAX)
    return MOE_ERR_UNSUPPORTED;
  MOE_CUDA_TRY(launch_gather_rows_raw(src, (int)(src_rows * divisor), idx, (int)n_rows, divisor,
                                      (int)(row_bytes / 16), dst,
                                      static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

extern "C" moe_status moe_ep_local_order(const int32_t* recv_counts, int32_t G, int32_t El,
                                         int32_t* offsets, int32_t* perm, int32_t* inv,
                                         int64_t rows_capacity, moe_stream stream) {
  if (G < 1 || El < 1 || G > 1024 || El > 1024 || rows_capacity < 0) return MOE_ERR_INVALID_ARG;
  if ((long long)G * El > kEpMaxCells || rows_capacity > INT_MAX) return MOE_ERR_UNSUPPORTED;
  if (!recv_counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (rows_capacity > 0 && (!perm || !inv)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(launch_ep_local_order(recv_counts, G, El, offsets, perm, inv, (int)rows_capacity,
                                     static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}
