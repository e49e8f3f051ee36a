// Dispatch: group the T*K token copies by expert into expert-contiguous rows.
//
// "MoE architecture in production" §3.1 (MoEDispatcher): all experts share
// one pre-allocated buffer; for each expert the matching token indices are
// found (torch.where on the mask, so ascending order), gathered, run through
// the expert and scattered back. "Kimi K3 专家路由不均衡诊断" §三 counts hits
// per expert; §五 forbids dropping copies, so every copy gets a row.
//
// Three kernels, no global atomics:
//   1. chunk_histogram   per-chunk expert counts (shared-memory counters)
//   2. scan_and_tiles    one CTA: counts, exclusive offsets, per-(chunk,
//                        expert) bases, and the grouped-GEMM tile lists
//   3. chunk_scatter     stable placement: inside a chunk, warps own
//                        consecutive copy ranges and rank equal experts with
//                        __match_any_sync, so the order is ascending copy id.
#include "common.cuh"
#include "kernels.cuh"

namespace moe {

__global__ void __launch_bounds__(256) chunk_histogram(const int32_t* __restrict__ idx, int TK,
                                                       int E, int32_t* __restrict__ hist,
                                                       uint32_t* __restrict__ status) {
  __shared__ int h[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kChunk;
  const int c1 = min(TK, c0 + kChunk);
  bool bad = false;
  for (int i = c0 + threadIdx.x; i < c1; i += blockDim.x) {
    const int e = idx[i];
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&h[e], 1);
    else
      bad = true;
  }
  if (bad) atomicOr(status, kStatusBadIndex);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? sh[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    sh[32 + lane] = wi - w;
    if (lane == 31) sh[64] = wi;
  }
  __syncthreads();
  const int r = sh[32 + warp] + incl - v;
  *total = sh[64];
  __syncthreads();
  return r;
}

// Tile-list parameters for the grouped GEMMs.
struct TileSpec {
  Tile* simt;          // SIMT tiles: rows in blocks of kSimtRows, per group
  Tile* tc1;           // tensor-core tiles of GEMM1 (row block x output-column block)
  Tile* tc2;           // tensor-core tiles of GEMM2
  int m_tiles1_routed, m_tiles1_shared;   // output-column tiles (128 wide) of GEMM1
  int m_tiles2;                           // output-column tiles of GEMM2 (H / 128)
};

// Number of balanced row tiles for a group of c rows and the rows per tile
// (a multiple of 16, at most kTcRows).
__device__ __forceinline__ void tc_row_split(int c, int* nt, int* rows) {
  if (c <= 0) {
    *nt = 0;
    *rows = 0;
    return;
  }
  const int n = (c + kTcRows - 1) / kTcRows;
  int r = (c + n - 1) / n;
  r = (r + 15) & ~15;
  *nt = n;
  *rows = r;
}

// Writes the tile lists of every group; thread e < E owns expert e (c rows
// starting at row `off`), thread E owns the shared expert (T token rows).
__device__ void emit_tiles(int c, int off, int E, int T, int has_shared, const TileSpec& ts,
                           int* sh, WsHeader* hdr) {
  const int e = threadIdx.x;
  // SIMT tiles: ceil(rows / kSimtRows) row blocks per group.
  const int g_rows = (e < E) ? c : ((e == E && has_shared) ? T : 0);
  const int r_base = (e < E) ? off : 0;
  const int nt_simt = (g_rows + kSimtRows - 1) / kSimtRows;
  int tot_simt;
  const int first_simt = block_exclusive_scan(nt_simt, sh, &tot_simt);
  if (ts.simt) {
    for (int i = 0; i < nt_simt; ++i) {
      Tile t;
      t.g = e;
      t.r0 = r_base + i * kSimtRows;
      t.n = min(kSimtRows, g_rows - i * kSimtRows);
      t.m0 = 0;
      ts.simt[first_simt + i] = t;
    }
  }
  // Tensor-core tiles: balanced row blocks (<= kTcRows rows, multiple of 16)
  // times 128-wide output-column blocks.
  int nt_rows, rows_per;
  tc_row_split(g_rows, &nt_rows, &rows_per);
  const int mt1 = (e < E) ? ts.m_tiles1_routed : ts.m_tiles1_shared;
  int tot1, tot2;
  const int first1 = block_exclusive_scan(nt_rows * mt1, sh, &tot1);
  const int first2 = block_exclusive_scan(nt_rows * ts.m_tiles2, sh, &tot2);
  if (ts.tc1) {
    int o1 = first1, o2 = first2;
    for (int i = 0; i < nt_rows; ++i) {
      Tile t;
      t.g = e;
      t.r0 = r_base + i * rows_per;
      t.n = min(rows_per, g_rows - i * rows_per);
      for (int m = 0; m < mt1; ++m) {
        t.m0 = m * 128;
        ts.tc1[o1++] = t;
      }
      for (int m = 0; m < ts.m_tiles2; ++m) {
        t.m0 = m * 128;
        ts.tc2[o2++] = t;
      }
    }
  }
  if (threadIdx.x == 0) {
    hdr->n_tiles[0] = tot_simt;
    hdr->n_tiles[1] = ts.tc1 ? tot1 : 0;
    hdr->n_tiles[2] = ts.tc1 ? tot2 : 0;
  }
}

__global__ void __launch_bounds__(1024) scan_and_tiles(const int32_t* __restrict__ hist,
                                                       int n_chunks, int E, int T, int has_shared,
                                                       int32_t* __restrict__ counts,
                                                       int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ base,
                                                       TileSpec ts, WsHeader* __restrict__ hdr) {
  __shared__ int sh[96];
  const int e = threadIdx.x;   // one thread per expert slot (E <= 512 < 1024)
  int c = 0;
  if (e < E)
    for (int k = 0; k < n_chunks; ++k) c += hist[(size_t)k * E + e];
  int total;
  const int off = block_exclusive_scan(e < E ? c : 0, sh, &total);
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    int run = off;
    for (int k = 0; k < n_chunks; ++k) {
      base[(size_t)k * E + e] = run;
      run += hist[(size_t)k * E + e];
    }
  }
  if (e == E) offsets[E] = total;
  emit_tiles(c, off, E, T, has_shared, ts, sh, hdr);
}

// Tile lists from given offsets (moe_grouped_ffn called on its own).
__global__ void __launch_bounds__(1024) tiles_from_offsets(const int32_t* __restrict__ offsets,
                                                           int E, int T, int has_shared,
                                                           TileSpec ts,
                                                           WsHeader* __restrict__ hdr) {
  __shared__ int sh[96];
  const int e = threadIdx.x;
  int c = 0, off = 0;
  if (e < E) {
    off = offsets[e];
    c = offsets[e + 1] - off;
  }
  emit_tiles(c, off, E, T, has_shared, ts, sh, hdr);
}

constexpr int kScatterWarps = 8;

__global__ void __launch_bounds__(256) chunk_scatter(const int32_t* __restrict__ idx, int TK,
                                                     int E, const int32_t* __restrict__ base,
                                                     int32_t* __restrict__ perm,
                                                     int32_t* __restrict__ inv) {
  __shared__ int cnt[kScatterWarps][kMaxE];   // per-warp counts, then running ranks
  __shared__ int pre[kScatterWarps][kMaxE];   // exclusive prefix over warps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) cnt[i / E][i % E] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kChunk;
  const int per_warp = kChunk / kScatterWarps;
  const int w0 = c0 + warp * per_warp;
  const int w1 = min(TK, w0 + per_warp);
  for (int i = w0 + lane; i < w1; i += 32) {
    const int e = idx[i];
    if ((unsigned)e < (unsigned)E) atomicAdd(&cnt[warp][e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = base[(size_t)blockIdx.x * E + e];
    for (int w = 0; w < kScatterWarps; ++w) {
      pre[w][e] = run;
      run += cnt[w][e];
      cnt[w][e] = 0;
    }
  }
  __syncthreads();
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const bool live = i < w1;
    const int e = live ? idx[i] : -1;
    const bool ok = live && (unsigned)e < (unsigned)E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int row = pre[warp][e] + cnt[warp][e] + rank;
      perm[row] = i;
      inv[i] = row;
    }
    __syncwarp();
    if (ok && (peers & ((1u << lane) - 1u)) == 0) cnt[warp][e] += __popc(peers);
    __syncwarp();
  }
}

// Gather of dispatched activation rows: xp[row] = x[perm[row] / K] (bf16,
// 16-byte vectors), so the tensor-core GEMM reads contiguous rows.
__global__ void __launch_bounds__(256) gather_rows(const uint4* __restrict__ x,
                                                   const int32_t* __restrict__ perm, int TK,
                                                   int K, int row_vecs, uint4* __restrict__ xp) {
  const size_t total = (size_t)TK * row_vecs;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / row_vecs;
    const int v = (int)(i - row * row_vecs);
    const int t = perm[row] / K;
    xp[i] = x[(size_t)t * row_vecs + v];
  }
}

static TileSpec make_tile_spec(const moe_layer_desc& d, const WsLayout& L, char* ws,
                               bool tc_tiles) {
  TileSpec ts;
  ts.simt = reinterpret_cast<Tile*>(ws + L.tiles_simt);
  ts.tc1 = tc_tiles ? reinterpret_cast<Tile*>(ws + L.tiles_tc1) : nullptr;
  ts.tc2 = tc_tiles ? reinterpret_cast<Tile*>(ws + L.tiles_tc2) : nullptr;
  ts.m_tiles1_routed = d.D / 128;
  ts.m_tiles1_shared = d.Ds / 128;
  ts.m_tiles2 = d.H / 128;
  return ts;
}

cudaError_t launch_dispatch(const moe_layer_desc& d, const WsLayout& L, char* ws,
                            const int32_t* idx, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv, bool tc_tiles, cudaStream_t st) {
  const int TK = d.T * d.K;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* base = reinterpret_cast<int32_t*>(ws + L.base);
  const int n_chunks = L.n_chunks;
  if (TK > 0) {
    count_launch();
    chunk_histogram<<<n_chunks, 256, 0, st>>>(idx, TK, d.E, hist, &hdr->status);
  } else {
    cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)n_chunks * d.E, st);
  }
  const TileSpec ts = make_tile_spec(d, L, ws, tc_tiles);
  count_launch();
  scan_and_tiles<<<1, 1024, 0, st>>>(hist, n_chunks, d.E, d.T, d.Ds > 0 ? 1 : 0, counts, offsets,
                                     base, ts, hdr);
  if (TK > 0) {
    count_launch();
    chunk_scatter<<<n_chunks, 256, 0, st>>>(idx, TK, d.E, base, perm, inv);
  }
  return cudaGetLastError();
}

// The same three dispatch kernels with caller-provided scratch: hist and base
// hold n_chunks * E ints each; no tile lists are written.
cudaError_t launch_dispatch_scratch(const moe_layer_desc& d, int n_chunks, int32_t* hist,
                                   int32_t* base, WsHeader* hdr, const int32_t* idx,
                                   int32_t* counts, int32_t* offsets, int32_t* perm,
                                   int32_t* inv, cudaStream_t st) {
  const int TK = d.T * d.K;
  if (TK > 0) {
    count_launch();
    chunk_histogram<<<n_chunks, 256, 0, st>>>(idx, TK, d.E, hist, &hdr->status);
  } else {
    cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)n_chunks * d.E, st);
    if (e != cudaSuccess) return e;
  }
  TileSpec ts{};
  count_launch();
  scan_and_tiles<<<1, 1024, 0, st>>>(hist, n_chunks, d.E, d.T, d.Ds > 0 ? 1 : 0, counts, offsets,
                                     base, ts, hdr);
  if (TK > 0) {
    count_launch();
    chunk_scatter<<<n_chunks, 256, 0, st>>>(idx, TK, d.E, base, perm, inv);
  }
  return cudaGetLastError();
}

cudaError_t launch_tiles_from_offsets(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                      const int32_t* offsets, bool tc_tiles, cudaStream_t st) {
  const TileSpec ts = make_tile_spec(d, L, ws, tc_tiles);
  count_launch();
  tiles_from_offsets<<<1, 1024, 0, st>>>(offsets, d.E, d.T, d.Ds > 0 ? 1 : 0, ts,
                                         reinterpret_cast<WsHeader*>(ws + L.hdr));
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const moe_layer_desc& d, const void* x, const int32_t* perm,
                               void* xp, int num_sms, cudaStream_t st) {
  const int TK = d.T * d.K;
  if (TK == 0) return cudaSuccess;
  const int row_vecs = d.H * 2 / 16;
  const size_t total = (size_t)TK * row_vecs;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, (size_t)num_sms * 8);
  count_launch();
  gather_rows<<<blocks, 256, 0, st>>>((const uint4*)x, perm, TK, d.K, row_vecs, (uint4*)xp);
  return cudaGetLastError();
}

}  // namespace moe
