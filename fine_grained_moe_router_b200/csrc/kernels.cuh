// Internal launcher declarations shared by the C-ABI translation unit.
#pragma once

#include "common.cuh"

namespace moe {

// One side (routed experts or shared expert) of a grouped GEMM on CUDA cores.
struct SimtProblem {
  const void* A;           // activation rows [*, Kd]
  const int32_t* perm;     // non-null: row r reads A row perm[r] / k_top
  int k_top;
  const void* B;           // weights [groups, N, Kd] (group stride b_group_stride elements)
  size_t b_group_stride;
  void* C;                 // output rows [*, N]
  int Kd;                  // reduction length
  int N;                   // output columns
};

// One side (routed experts or shared expert) of a grouped GEMM on the tensor
// cores. act [act_rows, kd] and w [w_rows, kd] are bf16 row-major; the
// group g occupies weight rows [g * m_rows, (g + 1) * m_rows).
struct TcProblem {
  const void* act;
  uint64_t act_rows;
  const void* w;
  uint64_t w_rows;
  int m_rows;
  int kd;
  void* out;               // [*, ld], bf16 (first layer) or fp32 (out_f32)
  int ld;
  bool out_f32;
  int splits;              // reduction splits (0 or 1: none); split s writes out + s * split_stride
  long long split_stride;
  int m_valid;             // output columns stored (0: all m_rows)
  // First (GeLU) layer with splits > 1: out receives the fp32 partials and
  // the last split of each tile writes GeLU(sum) as bf16 to fix_out [*, fix_ld].
  void* fix_out;
  int fix_ld;
};

// Tiling without a device tile list (gate GEMM): `rows` activation rows in
// blocks of kTcRows, `m_tiles` weight-row blocks, routed.splits splits.
struct DenseTiling {
  int tiles, rows, m_tiles;
};

// pair: tiles of 256 weight rows on two-CTA clusters (tile list built with
// 256-row weight blocks, or dense m_tiles of 256 rows); otherwise 128 weight
// rows per CTA. max_ctas > 0 caps the persistent grid (the rest of the SMs
// stay free for work on another stream).
cudaError_t launch_grouped_gemm_tc(const TcProblem& routed, const TcProblem& shared, int E,
                                   bool gelu, const Tile* tiles, const int* n_tiles,
                                   const DenseTiling* dense, bool pair, uint32_t* status,
                                   int num_sms, cudaStream_t st, int max_ctas = 0);

cudaError_t launch_gate_logits(const moe_layer_desc& d, const void* x, const void* wr,
                               float* logits, cudaStream_t st);
// noise (nullable): Gumbel draws [T, E] fp32 added after the bias.
cudaError_t launch_topk_select(const moe_layer_desc& d, const float* logits, int n_parts,
                               size_t part_stride, const float* bias, const float* noise,
                               int32_t* idx, float* w, float* logits_out, cudaStream_t st);
// Gate logits on the tensor cores (bf16 layers): `parts` receives
// L.sp.router partial sums [T, E] fp32, part stride T * E.
cudaError_t launch_gate_logits_tc(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                  const void* x, const void* wr, float* parts, int num_sms,
                                  cudaStream_t st);
// shared_tiles = false: the tile lists leave the shared expert out (it runs
// in launches of its own).
cudaError_t launch_dispatch(const moe_layer_desc& d, const WsLayout& L, char* ws,
                            const int32_t* idx, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv, bool tc_tiles, cudaStream_t st,
                            bool shared_tiles = true);
cudaError_t launch_dispatch_scratch(const moe_layer_desc& d, int n_chunks, int32_t* hist,
                                   int32_t* base, WsHeader* hdr, const int32_t* idx,
                                   int32_t* counts, int32_t* offsets, int32_t* perm,
                                   int32_t* inv, cudaStream_t st);
cudaError_t launch_tiles_from_offsets(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                      const int32_t* offsets, bool tc_tiles, cudaStream_t st);
// xp[row] = x[perm[row] / K]; with inv (from the same dispatch) and at least
// kGatherByTokenMinT tokens the copy is walked by token (each x row read once).
constexpr int kGatherByTokenMinT = 2048;
cudaError_t launch_gather_rows(const moe_layer_desc& d, const void* x, const int32_t* perm,
                               void* xp, int num_sms, cudaStream_t st,
                               const int32_t* inv = nullptr);
// dst[r] = src[idx[r] / divisor] (row_vecs 16-byte vectors a row) for r < n_rows; idx
// values at or above idx_bound (or negative) leave the row unwritten.
cudaError_t launch_gather_rows_raw(const void* src, int idx_bound, const int32_t* idx, int n_rows,
                                   int divisor, int row_vecs, void* dst, cudaStream_t st);
// Expert-major order of the rows one rank receives (see ep.cu).
cudaError_t launch_ep_local_order(const int32_t* cnt, int G, int El, int32_t* offsets,
                                  int32_t* perm, int32_t* inv, int capacity, cudaStream_t st);
cudaError_t launch_grouped_gemm_simt(int dtype, bool gelu, const SimtProblem& routed,
                                     const SimtProblem& shared, int E, const Tile* tiles,
                                     const int* n_tiles, int max_tiles, int max_n,
                                     cudaStream_t st);
// y_rows / y_shared may hold several partial sums (reduction splits of the
// second expert GEMM), T*K*H and T*H elements apart.
cudaError_t launch_combine(const moe_layer_desc& d, const void* y_rows, const float* w,
                           const int32_t* inv, const void* y_shared, void* y, cudaStream_t st,
                           int rows_parts = 1, int shared_parts = 1);
// Buffers of the single-launch decode forward (bf16 layers, T <= kDecodeMaxT):
// inputs, the output y, the routing outputs (caller's or workspace buffers),
// the first layer's outputs Hm [T*K, D] and Hs [T, Ds] in the workspace, and
// the workspace header (status word, grid barrier counters).
struct DecodeBuffers {
  const void *x, *w_router, *w1, *w2, *ws1, *ws2;
  const float* bias;    // nullable
  const float* noise;   // nullable
  void* y;
  float* logits;
  int32_t *idx, *counts, *offsets, *perm, *inv;
  float* tw;
  void *hm, *hs;
  WsHeader* hdr;
};
// True when the shape runs as one cooperative launch on this device.
bool decode_eligible(const moe_layer_desc& d);
cudaError_t launch_decode_forward(const moe_layer_desc& d, const DecodeBuffers& b,
                                  cudaStream_t st);
cudaError_t launch_bias_update(const moe_layer_desc& d, const int32_t* counts, float* bias,
                               float gamma, cudaStream_t st);
cudaError_t launch_expert_stats(const moe_layer_desc& d, const int32_t* counts, uint8_t* mask,
                                moe_stats* out_dev, cudaStream_t st);

}  // namespace moe
