// Dispatch: group the T*K token copies by expert into expert-contiguous rows.
//
// "MoE architecture in production" §3.1 (MoEDispatcher): all experts share
// one pre-allocated buffer; for each expert the matching token indices are
// found (torch.where on the mask, so ascending order), gathered, run through
// the expert and scattered back. "Kimi K3 专家路由不均衡诊断" §三 counts hits
// per expert; §五 forbids dropping copies, so every copy gets a row.
//
// Three kernels, no atomics in the counting or the placement:
//   1. chunk_histogram   per-chunk expert counts: each warp counts its own
//                        range of copies into a private row of counters (the
//                        lanes holding one expert find each other with
//                        __match_any_sync and the lowest adds the group's size)
//   2. scan_and_tiles    one CTA: counts, exclusive offsets, per-(chunk,
//                        expert) bases, and the grouped-GEMM tile lists
//   3. chunk_scatter     stable placement: inside a chunk, warps own
//                        consecutive copy ranges and rank equal experts with
//                        __match_any_sync, so the order is ascending copy id.
// A copy whose expert index is outside [0, E) is not placed: its inv entry
// is -1, the rows past the placed copies hold perm = -1, and the status word
// records kStatusBadIndex.
// Batches of at most one chunk (kChunk copies) run all three steps in one CTA
// (dispatch_small). gather_rows then copies the dispatched activation rows
// for the tensor-core GEMMs; for the smallest batches (kFusedGatherCopies)
// dispatch_small copies them itself.
#include <atomic>

#include "common.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {

// Counts the copies [w0, w1) by expert into the warp's own counter row
// cnt_row[0..E) without atomics: in each round of 32 copies the lanes that
// hold the same expert find each other with __match_any_sync and the lowest
// of them adds the group's size, so no two lanes write one counter at once.
// Returns true (on every lane) if some copy's expert is outside [0, E).
__device__ __forceinline__ bool warp_count(const int32_t* __restrict__ idx, int w0, int w1, int E,
                                           int* cnt_row) {
  const int lane = threadIdx.x & 31;
  const unsigned below = (1u << lane) - 1u;
  bool bad = false;
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const bool live = i < w1;
    const int e = live ? idx[i] : -1;
    const bool ok = live && (unsigned)e < (unsigned)E;
    bad |= live && !ok;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    if (ok && (peers & below) == 0) cnt_row[e] += __popc(peers);
    __syncwarp();
  }
  return __any_sync(0xffffffffu, bad);
}

constexpr int kHistWarps = 8;

__global__ void __launch_bounds__(kHistWarps * 32) chunk_histogram(const int32_t* __restrict__ idx,
                                                                  int TK, int E,
                                                                  int32_t* __restrict__ hist,
                                                                  uint32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[kHistWarps][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kHistWarps * E; i += blockDim.x) cnt[i / E][i % E] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kChunk;
  const int per_warp = kChunk / kHistWarps;
  const int w0 = min(TK, c0 + warp * per_warp), w1 = min(TK, w0 + per_warp);
  if (warp_count(idx, w0, w1, E, cnt[warp]) && lane == 0) atomicOr(status, kStatusBadIndex);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kHistWarps; ++w) c += cnt[w][e];
    hist[(size_t)blockIdx.x * E + e] = c;
  }
}

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of
// 32, at most 1024).
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
  int splits1_routed, splits1_shared;     // reduction splits of GEMM1 tiles
  int splits2_routed, splits2_shared;     // reduction splits of GEMM2 tiles
  int mtile;                              // weight rows per tile: 128, or 256 on CTA pairs
  int lpt;                                // 1: experts by descending rows; 0: by index
  int tc_sliced;                          // 1: the tensor-core lists are written by
                                          // emit_tiles_sliced after the dispatch kernels
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

constexpr int kFlatTileList = 8192;   // tiles above which every thread shares the writing

// Writes the tile lists of every group; thread e < E owns expert e (c rows
// starting at row `off`), thread E owns the shared expert (T token rows).
// The tensor-core tile lists of emit_tiles (this CTA's slice of them).
// Thread e (one per expert slot, blockDim > E): c rows of expert e; g_rows
// and r_base the rows and first dispatched row of group e (group E: the
// shared expert's T rows when present).
__device__ void emit_tc_tiles(int c, int E, int T, int has_shared, const TileSpec& ts, int* sh,
                              WsHeader* hdr, int g_rows, int r_base, int slice, int n_slices) {
  const int e = threadIdx.x;
  // Tensor-core tiles: balanced row blocks (<= kTcRows rows, multiple of 16)
  // times weight-row blocks (128, or 256 on CTA pairs) times reduction
  // splits. Order: the shared expert first, then the routed experts by
  // descending row count (ties by index), so the longest work starts first;
  // the order inside a group is given where the tiles are written. Batches
  // of at most 4 copies per expert on average keep the experts in index
  // order instead: their tiles all cost about one weight slab, and the
  // O(E) ranking is a visible part of a decode step.
  __shared__ int s_cnt[kMaxE];
  __shared__ int s_pos1[kMaxE], s_pos2[kMaxE], s_grp[kMaxE];
  __shared__ int s_first1[kMaxE + 1], s_first2[kMaxE + 1], s_nt[kMaxE + 1], s_rper[kMaxE + 1],
      s_rows[kMaxE + 1], s_rbase[kMaxE + 1];
  int nt_rows, rows_per;
  tc_row_split(g_rows, &nt_rows, &rows_per);
  const int mt1 = (e < E) ? ts.m_tiles1_routed : ts.m_tiles1_shared;
  int sh_nt, sh_rper;
  tc_row_split(has_shared ? T : 0, &sh_nt, &sh_rper);
  const int sh1 = sh_nt * ts.m_tiles1_shared * ts.splits1_shared;
  const int sh2 = sh_nt * ts.m_tiles2 * ts.splits2_shared;
  if (e < E) s_cnt[e] = c;
  __syncthreads();
  int rank = 0;
  if (e < E) {
    if (ts.lpt) {
      for (int q = 0; q < E; ++q) {
        const int cq = s_cnt[q];
        rank += (cq > c) || (cq == c && q < e);
      }
    } else {
      rank = e;
    }
    s_grp[rank] = e;
    s_pos1[rank] = nt_rows * mt1 * ts.splits1_routed;   // tile counts in rank order
    s_pos2[rank] = nt_rows * ts.m_tiles2 * ts.splits2_routed;
  }
  __syncthreads();
  int tot1, tot2;
  const int p1 = block_exclusive_scan(e < E ? s_pos1[e] : 0, sh, &tot1);
  const int p2 = block_exclusive_scan(e < E ? s_pos2[e] : 0, sh, &tot2);
  if (e < E) {
    s_pos1[e] = p1;
    s_pos2[e] = p2;
  }
  __syncthreads();
  if (e <= E) {
    s_first1[e] = (e < E) ? sh1 + s_pos1[rank] : 0;
    s_first2[e] = (e < E) ? sh2 + s_pos2[rank] : 0;
    s_nt[e] = nt_rows;
    s_rper[e] = rows_per;
    s_rows[e] = g_rows;
    s_rbase[e] = r_base;
  }
  __syncthreads();
  if (ts.tc1) {
    const int n1_all = sh1 + tot1, n2_all = sh2 + tot2;
    // Long lists (a long batch: thousands of tiles in the shared expert's or
    // a hot expert's group) are spread over all threads, each finding its
    // tile's group by binary search over the groups' first positions;
    // shorter ones go one group per warp, which needs no search.
    const bool flat = n_slices > 1 || n1_all + n2_all > kFlatTileList;
    const int lo = (int)((long long)(n1_all + n2_all) * slice / n_slices);
    const int hi = (int)((long long)(n1_all + n2_all) * (slice + 1) / n_slices);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    int g = flat ? 0 : warp, i_begin = flat ? lo + (int)threadIdx.x : lane;
    const int i_step = flat ? (int)blockDim.x : 32;
    while (g <= E) {
      // tiles of group g (per-warp mode) or of both whole lists (flat mode)
      const int nt_g = s_nt[g];
      const int m1_g = (g < E) ? ts.m_tiles1_routed : ts.m_tiles1_shared;
      const int sp1_g = (g < E) ? ts.splits1_routed : ts.splits1_shared;
      const int sp2_g = (g < E) ? ts.splits2_routed : ts.splits2_shared;
      const int n_items = flat ? hi : nt_g * (m1_g * sp1_g + ts.m_tiles2 * sp2_g);
      for (int i = i_begin; i < n_items; i += i_step) {
        int gg = g, j;
        bool first;
        if (flat) {
          first = i < n1_all;
          const int li = first ? i : i - n1_all;   // position in its list
          const int shn = first ? sh1 : sh2;
          if (li < shn) {
            gg = E;
            j = li;
          } else {
            const int k = li - shn;
            const int* pos = first ? s_pos1 : s_pos2;
            int lo = 0, hi = E - 1;   // last rank position with pos <= k (a non-empty group)
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (pos[mid] <= k)
                lo = mid;
              else
                hi = mid - 1;
            }
            gg = s_grp[lo];
            j = k - pos[lo];
          }
        } else {
          const int n1 = nt_g * m1_g * sp1_g;
          first = i < n1;
          j = first ? i : i - n1;
        }
        const int nt = s_nt[gg];
        const int sp = first ? ((gg < E) ? ts.splits1_routed : ts.splits1_shared)
                             : ((gg < E) ? ts.splits2_routed : ts.splits2_shared);
        const int mt = first ? ((gg < E) ? ts.m_tiles1_routed : ts.m_tiles1_shared) : ts.m_tiles2;
        // Order inside the group: when the group has more activation rows than
        // weight rows the row blocks are outermost (the weight matrix stays in
        // L2 while the rows stream once); otherwise the weight blocks are
        // outermost (each weight slab streams once while its row blocks, on
        // neighbouring CTAs, reuse it from L2). Splits vary fastest after that.
        int r, q, j0;   // j0: the position of the split-0 tile of j in the group
        const bool row_outer = s_rows[gg] > mt * ts.mtile;
        if (row_outer) {
          r = j / (mt * sp);
          q = j - r * (mt * sp);
        } else {
          r = j % nt;
          q = j / nt;
        }
        Tile t;
        t.g = gg;
        t.r0 = s_rbase[gg] + r * s_rper[gg];
        t.n = min(s_rper[gg], s_rows[gg] - r * s_rper[gg]);
        t.m0 = (q / sp) * ts.mtile;
        t.ks = q % sp;
        j0 = row_outer ? j - t.ks : j - t.ks * nt;
        t.arrivals[0] = 0;
        t.arrivals[1] = 0;
        if (first) {
          t.first_split = s_first1[gg] + j0;
          ts.tc1[s_first1[gg] + j] = t;
        } else {
          t.first_split = s_first2[gg] + j0;
          ts.tc2[s_first2[gg] + j] = t;
        }
      }
      if (flat) break;
      g += nwarps;
    }
  }
  if (threadIdx.x == 0 && slice == 0) {
    hdr->n_tiles[1] = tot1 + sh1;
    hdr->n_tiles[2] = tot2 + sh2;
  }
}

// slice / n_slices: with n_slices > 1 this CTA writes only its share
// [n * slice / n_slices, n * (slice + 1) / n_slices) of the n tensor-core
// tiles (both lists as one index space), slice 0 their counts; n_slices = 0
// writes no tensor-core tile. The SIMT list is written whole, by slice 0.
__device__ void emit_tiles(int c, int off, int E, int T, int has_shared, const TileSpec& ts,
                           int* sh, WsHeader* hdr, int slice = 0, int n_slices = 1) {
  const int e = threadIdx.x;
  // SIMT tiles: ceil(rows / kSimtRows) row blocks per group.
  const int g_rows = (e < E) ? c : ((e == E && has_shared) ? T : 0);
  const int r_base = (e < E) ? off : 0;
  const int nt_simt = (g_rows + kSimtRows - 1) / kSimtRows;
  int tot_simt = 0, first_simt = 0;
  if (ts.simt) first_simt = block_exclusive_scan(nt_simt, sh, &tot_simt);   // uniform branch
  if (ts.simt && slice == 0) {
    for (int i = 0; i < nt_simt; ++i) {
      Tile t;
      t.g = e;
      t.r0 = r_base + i * kSimtRows;
      t.n = min(kSimtRows, g_rows - i * kSimtRows);
      t.m0 = 0;
      t.ks = 0;
      ts.simt[first_simt + i] = t;
    }
  }
  if (threadIdx.x == 0 && slice == 0) {
    hdr->n_tiles[0] = tot_simt;
    if (!ts.tc1) {
      hdr->n_tiles[1] = 0;
      hdr->n_tiles[2] = 0;
    }
  }
  if (ts.tc1 && n_slices > 0)
    emit_tc_tiles(c, E, T, has_shared, ts, sh, hdr, g_rows, r_base, slice, n_slices);
}

__global__ void __launch_bounds__(1024) scan_and_tiles(const int32_t* __restrict__ hist,
                                                       int n_chunks, int E, int T, int has_shared,
                                                       int TK, int32_t* __restrict__ counts,
                                                       int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ base,
                                                       int32_t* __restrict__ perm,
                                                       TileSpec ts, WsHeader* __restrict__ hdr) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sh[96];
  const int e = threadIdx.x;   // one thread per expert slot (E <= 512 < 1024)
  int c = 0;
  if (e < E)
    for (int k0 = 0; k0 < n_chunks; k0 += 8) {   // 8 independent loads per round
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = (k0 + q < n_chunks) ? hist[(size_t)(k0 + q) * E + e] : 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) c += v[q];
    }
  int total;
  const int off = block_exclusive_scan(e < E ? c : 0, sh, &total);
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    int run = off;
    for (int k0 = 0; k0 < n_chunks; k0 += 8) {
      int v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = (k0 + q < n_chunks) ? hist[(size_t)(k0 + q) * E + e] : 0;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (k0 + q < n_chunks) {
          base[(size_t)(k0 + q) * E + e] = run;
          run += v[q];
        }
    }
  }
  if (e == E) offsets[E] = total;
  // rows no copy fills (only when some copy had an expert outside [0, E))
  for (int r = total + threadIdx.x; r < TK; r += blockDim.x) perm[r] = -1;
  emit_tiles(c, off, E, T, has_shared, ts, sh, hdr, 0, ts.tc_sliced ? 0 : 1);
}

// Tile lists from given offsets (moe_grouped_ffn called on its own).
__global__ void __launch_bounds__(1024) tiles_from_offsets(const int32_t* __restrict__ offsets,
                                                           int E, int T, int has_shared,
                                                           TileSpec ts,
                                                           WsHeader* __restrict__ hdr) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sh[96];
  const int e = threadIdx.x;
  int c = 0, off = 0;
  if (e < E) {
    off = offsets[e];
    c = offsets[e + 1] - off;
  }
  emit_tiles(c, off, E, T, has_shared, ts, sh, hdr);
}

// The tensor-core tile lists from the offsets a dispatch kernel wrote, over
// many CTAs: each recomputes the groups' table from the offsets and writes
// its slice of the tiles (one tile per thread or so).
__global__ void __launch_bounds__(1024) emit_tiles_sliced(const int32_t* __restrict__ offsets,
                                                          int E, int T, int has_shared,
                                                          TileSpec ts,
                                                          WsHeader* __restrict__ hdr) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sh[96];
  const int e = threadIdx.x;
  int c = 0, off = 0;
  if (e < E) {
    off = offsets[e];
    c = offsets[e + 1] - off;
  }
  emit_tc_tiles(c, E, T, has_shared, ts, sh, hdr, (e < E) ? c : ((e == E && has_shared) ? T : 0),
                (e < E) ? off : 0, (int)blockIdx.x, (int)gridDim.x);
}

constexpr int kScatterWarps = 8;

__global__ void __launch_bounds__(256) chunk_scatter(const int32_t* __restrict__ idx, int TK,
                                                     int E, const int32_t* __restrict__ base,
                                                     int32_t* __restrict__ perm,
                                                     int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[kScatterWarps][kMaxE];   // per-warp counts, then running ranks
  __shared__ int pre[kScatterWarps][kMaxE];   // exclusive prefix over warps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) cnt[i / E][i % E] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kChunk;
  const int per_warp = kChunk / kScatterWarps;
  const int w0 = min(TK, c0 + warp * per_warp);
  const int w1 = min(TK, w0 + per_warp);
  warp_count(idx, w0, w1, E, cnt[warp]);
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
    } else if (live) {
      inv[i] = -1;   // not placed (expert outside [0, E), reported in the status)
    }
    __syncwarp();
    if (ok && (peers & ((1u << lane) - 1u)) == 0) cnt[warp][e] += __popc(peers);
    __syncwarp();
  }
}

// Dispatch of a small batch (T*K <= kChunk, every decode step) in one CTA:
// the per-chunk histogram, the scan with the tile lists and the stable
// scatter of the three kernels above, without their two launch gaps. Warp w
// owns the consecutive copies [w * per_warp, (w + 1) * per_warp); counts per
// (warp, expert) live in dynamic shared memory (32 * E ints, twice).
constexpr int kSmallWarps = 32;   // warps of the one-CTA dispatch (at most)

// The whole dispatch of at most kChunk copies by one CTA of more than E
// threads (a multiple of 32; dyn_smem: 2 * (blockDim / 32) * E ints). Each
// warp counts and places a contiguous range of the copies.
__device__ void dispatch_block(const int32_t* __restrict__ idx, int TK, int E, int T,
                               int has_shared, int32_t* __restrict__ counts,
                               int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
                               int32_t* __restrict__ inv, const TileSpec& ts,
                               WsHeader* __restrict__ hdr, int* dyn_smem) {
  const int nw = blockDim.x >> 5;
  int* cnt = dyn_smem;             // [nw][E]
  int* pre = dyn_smem + nw * E;    // [nw][E]
  __shared__ int sh[96];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < nw * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int per_warp = (TK + nw - 1) / nw;
  const int w0 = min(TK, warp * per_warp), w1 = min(TK, w0 + per_warp);
  if (warp_count(idx, w0, w1, E, cnt + warp * E) && lane == 0)
    atomicOr(&hdr->status, kStatusBadIndex);
  __syncthreads();
  const int e = threadIdx.x;   // one thread per expert slot (blockDim > E)
  int c = 0;
  if (e < E)
    for (int w = 0; w < nw; ++w) c += cnt[w * E + e];
  int total;
  const int off = block_exclusive_scan(e < E ? c : 0, sh, &total);
  if (e < E) {
    counts[e] = c;
    offsets[e] = off;
    int run = off;
    for (int w = 0; w < nw; ++w) {
      pre[w * E + e] = run;
      run += cnt[w * E + e];
      cnt[w * E + e] = 0;
    }
  }
  if (e == E) offsets[E] = total;
  for (int r = total + threadIdx.x; r < TK; r += blockDim.x) perm[r] = -1;   // unfilled rows
  emit_tiles(c, off, E, T, has_shared, ts, sh, hdr, 0, ts.tc_sliced ? 0 : 1);
  __syncthreads();
  for (int i0 = w0; i0 < w1; i0 += 32) {
    const int i = i0 + lane;
    const bool live = i < w1;
    const int ei = live ? idx[i] : -1;
    const bool ok = live && (unsigned)ei < (unsigned)E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? ei : -1);
    if (ok) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int row = pre[warp * E + ei] + cnt[warp * E + ei] + rank;
      perm[row] = i;
      inv[i] = row;
    } else if (live) {
      inv[i] = -1;   // not placed (expert outside [0, E), reported in the status)
    }
    __syncwarp();
    if (ok && (peers & ((1u << lane) - 1u)) == 0) cnt[warp * E + ei] += __popc(peers);
    __syncwarp();
  }
}

// One dispatched activation row, xp[row] = x[perm[row] / K] (bf16 as
// 16-byte vectors), copied by one warp: each lane issues up to 16 vector
// loads before its first store (a 4096-wide row in one memory round trip).
// A copy index outside [0, TK) (left by a dispatch that rejected an
// out-of-range expert, which it reports in the status word) copies nothing.
__device__ __forceinline__ void gather_row(const uint4* __restrict__ x,
                                           const int32_t* __restrict__ perm, int TK, int K,
                                           int row_vecs, uint4* __restrict__ xp, int row,
                                           int lane) {
  constexpr int kVecs = 16;   // vectors in flight per lane
  const int c = perm[row];
  if ((unsigned)c >= (unsigned)TK) return;
  const uint4* src = x + (size_t)(c / K) * row_vecs;
  uint4* dst = xp + (size_t)row * row_vecs;
  for (int v0 = lane; v0 < row_vecs; v0 += 32 * kVecs) {
    uint4 a[kVecs];
#pragma unroll
    for (int q = 0; q < kVecs; ++q)
      if (v0 + 32 * q < row_vecs) a[q] = src[v0 + 32 * q];
#pragma unroll
    for (int q = 0; q < kVecs; ++q)
      if (v0 + 32 * q < row_vecs) dst[v0 + 32 * q] = a[q];
  }
}

// xp non-null: the CTA also gathers the dispatched rows (one warp per row),
// which saves the gather launch for the smallest batches.
__global__ void __launch_bounds__(1024) dispatch_small(const int32_t* __restrict__ idx, int TK,
                                                       int E, int T, int has_shared,
                                                       int32_t* __restrict__ counts,
                                                       int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ perm,
                                                       int32_t* __restrict__ inv, TileSpec ts,
                                                       WsHeader* __restrict__ hdr,
                                                       const uint4* __restrict__ x, int K,
                                                       int row_vecs, uint4* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int dyn_smem[];
  dispatch_block(idx, TK, E, T, has_shared, counts, offsets, perm, inv, ts, hdr, dyn_smem);
  if (xp == nullptr) return;
  __syncthreads();   // every warp's perm rows are written and visible to the CTA
  // The rows' vectors spread over all threads, a few loads in flight each
  // (the CTA's 64 registers per thread leave no room for a warp per row).
  constexpr int kVecs = 4;
  const int total = TK * row_vecs;
  for (int i0 = threadIdx.x; i0 < total; i0 += kVecs * blockDim.x) {
    uint4 a[kVecs];
    int dst[kVecs];
#pragma unroll
    for (int q = 0; q < kVecs; ++q) {
      const int i = i0 + q * blockDim.x;
      dst[q] = -1;
      if (i < total) {
        const int row = i / row_vecs, v = i - row * row_vecs;
        const int c = perm[row];
        if ((unsigned)c < (unsigned)TK) {   // else: a rejected copy, reported in the status
          a[q] = x[(size_t)(c / K) * row_vecs + v];
          dst[q] = i;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kVecs; ++q)
      if (dst[q] >= 0) xp[dst[q]] = a[q];
  }
}

// Gather of dispatched activation rows, so the tensor-core GEMM reads
// contiguous rows: one warp per row.
__global__ void __launch_bounds__(256) gather_rows(const uint4* __restrict__ x,
                                                   const int32_t* __restrict__ perm, int TK,
                                                   int K, int row_vecs, uint4* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < TK; row += warps)
    gather_row(x, perm, TK, K, row_vecs, xp, row, threadIdx.x & 31);
}

// The same gather walked by token, for large batches: the warp of token t
// reads x[t] once and writes it to the dispatched rows inv[t*K + k] of its
// K copies (a copy with inv = -1 was not placed and is skipped). Every row of
// x is read once instead of once per copy: 134 MB instead of up to 1.07 GB at
// 16384 tokens of 4096, top-8, where the rows written leave x little room in L2.
__global__ void __launch_bounds__(256) gather_rows_by_token(const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ inv,
                                                           int T, int K, int TK, int row_vecs,
                                                           uint4* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  constexpr int kVecs = 16;   // vectors in flight per lane
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const uint4* src = x + (size_t)t * row_vecs;
    for (int v0 = lane; v0 < row_vecs; v0 += 32 * kVecs) {
      uint4 a[kVecs];
#pragma unroll
      for (int q = 0; q < kVecs; ++q)
        if (v0 + 32 * q < row_vecs) a[q] = src[v0 + 32 * q];
      for (int k = 0; k < K; ++k) {
        const int row = inv[(size_t)t * K + k];
        if ((unsigned)row >= (unsigned)TK) continue;
        uint4* dst = xp + (size_t)row * row_vecs;
#pragma unroll
        for (int q = 0; q < kVecs; ++q)
          if (v0 + 32 * q < row_vecs) dst[v0 + 32 * q] = a[q];
      }
    }
  }
}

// The same copy for any rows: dst[r] = src[idx[r] / divisor] for r < n_rows,
// idx values checked against idx_bound (rows with an index outside it are
// left unwritten).
__global__ void __launch_bounds__(256) gather_rows_any(const uint4* __restrict__ src,
                                                       const int32_t* __restrict__ idx,
                                                       int idx_bound, int n_rows, int divisor,
                                                       int row_vecs, uint4* __restrict__ dst) {
  pdl_wait();
  pdl_trigger();
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < n_rows; row += warps)
    gather_row(src, idx, idx_bound, divisor, row_vecs, dst, row, threadIdx.x & 31);
}

static TileSpec make_tile_spec(const moe_layer_desc& d, const WsLayout& L, char* ws,
                               bool tc_tiles, bool split) {
  TileSpec ts;
  // CUDA-core tile lists only for layers that run the CUDA-core GEMM
  ts.simt = tc_tiles ? nullptr : reinterpret_cast<Tile*>(ws + L.tiles_simt);
  ts.tc1 = tc_tiles ? reinterpret_cast<Tile*>(ws + L.tiles_tc1) : nullptr;
  ts.tc2 = tc_tiles ? reinterpret_cast<Tile*>(ws + L.tiles_tc2) : nullptr;
  ts.mtile = (split && L.sp.pair) ? 256 : 128;
  ts.lpt = ((long long)d.T * d.K > 4LL * d.E) ? 1 : 0;
  ts.tc_sliced = 0;
  ts.m_tiles1_routed = d.D / ts.mtile;
  ts.m_tiles1_shared = d.Ds / ts.mtile;
  ts.m_tiles2 = d.H / ts.mtile;
  ts.splits1_routed = split ? L.sp.gemm1_routed : 1;
  ts.splits1_shared = split ? L.sp.gemm1_shared : 1;
  ts.splits2_routed = split ? L.sp.gemm2_routed : 1;
  ts.splits2_shared = split ? L.sp.gemm2_shared : 1;
  return ts;
}

// Dispatch; with x and xp (bf16 layers) also the gather of the dispatched
// rows into xp, inside the one-CTA dispatch for batches of at most
// kFusedGatherCopies copies, else as its own launch after the dispatch.
static cudaError_t dispatch_impl(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                 const int32_t* idx, int32_t* counts, int32_t* offsets,
                                 int32_t* perm, int32_t* inv, bool tc_tiles, cudaStream_t st,
                                 bool shared_tiles, const void* x, void* xp, int num_sms) {
  const int TK = d.T * d.K;
  const bool fuse_gather = xp != nullptr && TK <= kFusedGatherCopies;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* base = reinterpret_cast<int32_t*>(ws + L.base);
  const int n_chunks = L.n_chunks;
  TileSpec ts = make_tile_spec(d, L, ws, tc_tiles, /*split=*/true);
  const int has_shared = (d.Ds > 0 && shared_tiles) ? 1 : 0;
  // Batches of more than kChunk copies (the three-kernel dispatch): the
  // tensor-core lists are written over all SMs by a launch of their own,
  // after the dispatch kernels (which then write only the counts, offsets,
  // perm and inv); at 16384 tokens of the 128-expert layer, 27 us faster.
  // Smaller batches keep the one-CTA writing: there the extra launch and the
  // table every CTA rebuilds cost as much as the writing saves (c3 T=16
  // 267.5 vs 269.7 us, c4 T=16 275.3 vs 279.5 us, measured).
  ts.tc_sliced = (tc_tiles && TK > kChunk) ? 1 : 0;
  auto emit_sliced = [&]() -> cudaError_t {
    return launch_pdl(emit_tiles_sliced, dim3(num_sms > 0 ? num_sms : 148), dim3(1024), 0, st,
                      (const int32_t*)offsets, d.E, d.T, has_shared, ts, hdr);
  };
  if (TK > 0 && TK <= kChunk) {
    // all 32 warps even for a handful of copies: they share the writing of
    // the tile lists (thousands of tiles for a few experts with a wide D)
    const int threads = 32 * kSmallWarps;
    const size_t smem = sizeof(int) * 2 * kSmallWarps * (size_t)d.E;
    static std::atomic<bool> attr_set[64];   // per device: dynamic smem above 48 KB
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
      e = cudaFuncSetAttribute(dispatch_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(sizeof(int) * 2 * kSmallWarps * kMaxE));
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    e = launch_pdl(dispatch_small, dim3(1), dim3(threads), smem, st, idx, TK, d.E, d.T,
                   has_shared, counts, offsets, perm, inv, ts, hdr,
                   static_cast<const uint4*>(fuse_gather ? x : nullptr), d.K, d.H * 2 / 16,
                   static_cast<uint4*>(fuse_gather ? xp : nullptr));
    if (e == cudaSuccess && ts.tc_sliced) e = emit_sliced();
    if (e != cudaSuccess || fuse_gather || xp == nullptr) return e;
    return launch_gather_rows(d, x, perm, xp, num_sms, st, inv);
  }
  cudaError_t e = cudaSuccess;
  if (TK > 0)
    e = launch_pdl(chunk_histogram, dim3(n_chunks), dim3(kHistWarps * 32), 0, st, idx, TK, d.E,
                   hist, &hdr->status);
  else
    e = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)n_chunks * d.E, st);
  if (e != cudaSuccess) return e;
  e = launch_pdl(scan_and_tiles, dim3(1), dim3(1024), 0, st, (const int32_t*)hist, n_chunks, d.E,
                 d.T, has_shared, TK, counts, offsets, base, perm, ts, hdr);
  if (e != cudaSuccess) return e;
  if (TK > 0)
    e = launch_pdl(chunk_scatter, dim3(n_chunks), dim3(256), 0, st, idx, TK, d.E,
                   (const int32_t*)base, perm, inv);
  if (e == cudaSuccess && ts.tc_sliced) e = emit_sliced();
  if (e != cudaSuccess || xp == nullptr) return e;
  return launch_gather_rows(d, x, perm, xp, num_sms, st, inv);
}

cudaError_t launch_dispatch(const moe_layer_desc& d, const WsLayout& L, char* ws,
                            const int32_t* idx, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv, bool tc_tiles, cudaStream_t st,
                            bool shared_tiles) {
  return dispatch_impl(d, L, ws, idx, counts, offsets, perm, inv, tc_tiles, st, shared_tiles,
                       nullptr, nullptr, 0);
}

cudaError_t launch_dispatch_gather(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                   const int32_t* idx, int32_t* counts, int32_t* offsets,
                                   int32_t* perm, int32_t* inv, cudaStream_t st,
                                   bool shared_tiles, const void* x, void* xp, int num_sms) {
  return dispatch_impl(d, L, ws, idx, counts, offsets, perm, inv, /*tc_tiles=*/true, st,
                       shared_tiles, x, xp, num_sms);
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
    chunk_histogram<<<n_chunks, kHistWarps * 32, 0, st>>>(idx, TK, d.E, hist, &hdr->status);
  } else {
    cudaError_t e = cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)n_chunks * d.E, st);
    if (e != cudaSuccess) return e;
  }
  TileSpec ts{};
  count_launch();
  scan_and_tiles<<<1, 1024, 0, st>>>(hist, n_chunks, d.E, d.T, d.Ds > 0 ? 1 : 0, TK, counts,
                                     offsets, base, perm, ts, hdr);
  if (TK > 0) {
    count_launch();
    chunk_scatter<<<n_chunks, 256, 0, st>>>(idx, TK, d.E, base, perm, inv);
  }
  return cudaGetLastError();
}

cudaError_t launch_tiles_from_offsets(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                      const int32_t* offsets, bool tc_tiles, cudaStream_t st) {
  const TileSpec ts = make_tile_spec(d, L, ws, tc_tiles, /*split=*/false);
  return launch_pdl(tiles_from_offsets, dim3(1), dim3(1024), 0, st, offsets, d.E, d.T,
                    d.Ds > 0 ? 1 : 0, ts, reinterpret_cast<WsHeader*>(ws + L.hdr));
}

cudaError_t launch_gather_rows_raw(const void* src, int idx_bound, const int32_t* idx, int n_rows,
                                   int divisor, int row_vecs, void* dst, cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int blocks = (int)std::min<long long>(((long long)n_rows + 7) / 8, (long long)sms * 8);
  return launch_pdl(gather_rows_any, dim3(std::max(1, blocks)), dim3(256), 0, st,
                    static_cast<const uint4*>(src), idx, idx_bound, n_rows, divisor, row_vecs,
                    static_cast<uint4*>(dst));
}

cudaError_t launch_gather_rows(const moe_layer_desc& d, const void* x, const int32_t* perm,
                               void* xp, int num_sms, cudaStream_t st, const int32_t* inv) {
  const int TK = d.T * d.K;
  if (TK == 0) return cudaSuccess;
  const int row_vecs = d.H * 2 / 16;
  if (inv && d.T >= kGatherByTokenMinT) {
    const int blocks = (int)std::min<long long>(((long long)d.T + 7) / 8, (long long)num_sms * 8);
    return launch_pdl(gather_rows_by_token, dim3(blocks), dim3(256), 0, st, (const uint4*)x, inv,
                      d.T, d.K, TK, row_vecs, (uint4*)xp);
  }
  const int blocks = (int)std::min<size_t>(((size_t)TK + 7) / 8, (size_t)num_sms * 8);   // 8 rows per block
  return launch_pdl(gather_rows, dim3(blocks), dim3(256), 0, st, (const uint4*)x, perm, TK, d.K,
                    row_vecs, (uint4*)xp);
}

}  // namespace moe
