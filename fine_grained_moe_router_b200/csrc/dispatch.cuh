// Host entry point of the dispatch with the gather of the dispatched rows.
#pragma once

#include "common.cuh"

namespace moe {

// Batches of at most this many copies are gathered by the one-CTA dispatch
// itself, which saves the gather launch. Measured on B200: 1.2 us faster at
// 2 copies of 4096-wide rows; at 8 and 16 copies one CTA's copy costs more
// than the launch it saves.
constexpr int kFusedGatherCopies = 4;

// launch_dispatch with tensor-core tile lists, followed by the gather
// xp[row] = x[perm[row] / K] of the bf16 activation rows (x [T, H], xp
// [T*K, H]): inside the dispatch for at most kFusedGatherCopies copies,
// else as its own launch.
cudaError_t launch_dispatch_gather(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                   const int32_t* idx, int32_t* counts, int32_t* offsets,
                                   int32_t* perm, int32_t* inv, cudaStream_t st,
                                   bool shared_tiles, const void* x, void* xp, int num_sms);

}  // namespace moe
