// Shared device/host helpers of libmoe (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <climits>
#include <algorithm>

#include "../../include/moe.h"

namespace moe {

constexpr int kMaxK = 16;
constexpr int kMaxE = 512;
constexpr int kForwardEvents = 6;   // stage events of moe_layer_forward_profiled
// Tokens of the single-launch decode forward (at most). Measured on B200 at
// the 128- and 256-expert layers: 1 and 2 tokens run faster in one launch
// than on the multi-launch path (60.6 vs 77.1 us, 98.1 vs 107.5 us), 3 tokens
// slower (145.8 vs 122.1 us): their staged activations leave the weight
// rings two stages deep while the tensor-core GEMMs keep streaming.
constexpr int kDecodeMaxT = 2;

// Status bits written by kernels into the workspace header.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadIndex = 2u;   // a top-K index outside [0, E)

// Element access for the two layer dtypes.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Exact GeLU 0.5 z (1 + erf(z / sqrt 2)) with CUDA's erff.
__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
}

// Workspace header: control words the kernels share. Lives at offset 0.
struct WsHeader {
  uint32_t status;          // kStatus* bits, cleared by moe_check_status
  int32_t n_tiles[4];       // tile-list lengths written by the scan kernel
  uint32_t tickets[8];      // self-resetting arrival counters
  uint32_t pad[51];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// One unit of grouped-GEMM work: rows [r0, r0 + n) of group g.
// g < E: routed expert g (rows of the dispatched buffer);
// g == E: the shared expert (token rows).
struct Tile {
  int32_t g;
  int32_t r0;
  int32_t n;
  int32_t m0;   // first output column (weight row) of the tile; used by the tensor-core path
  int32_t ks;   // reduction split of the tile (tensor-core path), 0 when unsplit
  // First-layer tiles with reduction splits: in the split-0 tile, arrival
  // counters of the tile's splits for the CTA (or each CTA of a pair);
  // in every split, the list index of its split-0 tile. Written as 0 / the
  // index by the dispatch step each forward.
  int32_t arrivals[2];
  int32_t first_split;
};

// Reduction splits of the tensor-core GEMMs of one layer forward (chosen on
// the host from the shape alone). A split s of a tile covers reduction blocks
// [s * kb_per, (s + 1) * kb_per) and writes its own fp32 partial output. The
// partials are added in split order: by the selection kernel (gate GEMM), by
// the last split of a tile to finish (first expert layer, before its GeLU),
// or by the combine kernel (second expert layer).
struct Splits {
  int router;        // gate GEMM
  int gemm1_routed;  // first expert layer, routed experts
  int gemm1_shared;  // first expert layer, shared expert
  int gemm2_routed;  // second expert layer, routed experts
  int gemm2_shared;  // second expert layer, shared expert
  int pair;          // 1: expert GEMMs on CTA pairs (256 weight rows per tile)
};

// Offsets of each workspace region (bytes), 256-byte aligned.
struct WsLayout {
  size_t hdr, hist, base, tiles_simt, tiles_tc1, tiles_tc2, idx, w, counts, offsets, perm, inv,
      logits, logits_part, xp, hm, hs, p1r, p1s, yr, ys, stats, total;
  int n_chunks;
  int max_tiles_simt, max_tiles_tc1, max_tiles_tc2;
  Splits sp;
};

constexpr int kChunk = 2048;       // copies per dispatch chunk
constexpr int kSimtRows = 64;      // rows per SIMT FFN tile
constexpr int kTcRows = 256;       // max rows (MMA N) per tensor-core tile
constexpr int kMaxSplits = 64;

Splits choose_splits(const moe_layer_desc& d);
WsLayout workspace_layout(const moe_layer_desc& d);
void count_launch();   // bumps the process-wide kernel launch counter
size_t dtype_size(int dtype);

}  // namespace moe

#define MOE_CUDA_TRY(expr)                                      \
  do {                                                          \
    cudaError_t _e = (expr);                                    \
    if (_e != cudaSuccess) return MOE_ERR_CUDA;                 \
  } while (0)
