/*
 * moe.h -- C ABI of libmoe: the single-GPU forward pass of one fine-grained
 * Mixture-of-Experts FFN layer on NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages define it:
 *   router GEMM      l = x W_r^T (no bias)           -- "Kimi K3 fine-grained
 *                    MoE under high concurrency", section "工业级细粒度 MoE 路由
 *                    与通信掩盖实战" (FineGrainedMoERouter); "MoE architecture in
 *                    production" §2.3 (gating network)
 *   selection        Softmax(l + B), top-K, renormalise the K weights
 *                    -- same router code; "Kimi K3 专家路由不均衡诊断" §四
 *                    (no-aux-loss dynamic bias B)
 *   dispatch         group the T*K token copies by expert into one shared
 *                    buffer -- "MoE architecture in production" §3.1
 *                    (MoEDispatcher); no copy is ever dropped -- "Kimi K3
 *                    专家路由不均衡诊断" §五
 *   expert FFN       Linear -> GeLU -> Linear per expert, plus an always-on
 *                    shared expert -- "MoE architecture in production" §3.1;
 *                    "Kimi K3 fine-grained MoE..." opening section
 *   combine          weighted sum of each token's K expert outputs, back in
 *                    token order -- "Kimi K3 fine-grained MoE...", section
 *                    "物理通信拓扑" (combine phase)
 *   statistics       counts, capacity, overflow, skew, Gini -- "Kimi K3
 *                    专家路由不均衡诊断" §三 (MoERouteDiagnostics)
 *
 * Conventions for every call
 *  - Pointers are DEVICE pointers unless the parameter says "host".
 *  - Tensors are dense row-major. Weights use the nn.Linear [out, in] layout,
 *    so every GEMM operand is contiguous along its reduction dimension:
 *      x [T, H], W_r [E, H], W1 [E, D, H], W2 [E, H, D], Ws1 [Ds, H],
 *      Ws2 [H, Ds], y [T, H].
 *    Element type of x / weights / y is desc->dtype (MOE_F32 or MOE_BF16).
 *    The per-copy expert outputs y_rows / y_shared are always fp32, so the
 *    combine rounds the layer output exactly once. Logits, top-K weights and
 *    the bias are fp32; indices, counts, offsets, perm and inv are int32.
 *  - Device pointers must be 16-byte aligned.
 *  - The caller owns every buffer, including the workspace; the library
 *    never allocates device memory. The workspace must hold
 *    moe_workspace_size(desc) bytes and must be zero-filled once before its
 *    first use; the library leaves its control words at zero after every
 *    completed call, so it can be reused without clearing.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream), except moe_expert_stats, which synchronises it.
 *    Calls sharing one workspace must not overlap on the GPU.
 *  - Argument errors are reported synchronously, before any launch:
 *    MOE_ERR_INVALID_ARG (null pointer, negative size, K > E, ...),
 *    MOE_ERR_UNSUPPORTED (a shape outside the supported range below),
 *    MOE_ERR_WORKSPACE (workspace missing or too small). A failed launch
 *    returns MOE_ERR_CUDA. Kernels never wait without bound: a device-side
 *    wait that runs out sets a status word in the workspace that
 *    moe_check_status() reports as MOE_ERR_TIMEOUT.
 *  - Supported shapes: T >= 0, 1 <= K <= min(E, 16), 1 <= E <= 512,
 *    H, D (and Ds when nonzero) multiples of 128 for MOE_BF16 and of 4 for
 *    MOE_F32. T = 0 is a valid empty batch.
 *
 * Routing is exact: ties between equal scores go to the lower expert
 * index (-0.0 and +0.0 tie), the K slots are in descending score order, and
 * inside each expert's segment the copies are in ascending token order.
 */
#ifndef FINE_GRAINED_MOE_ROUTER_B200_MOE_H
#define FINE_GRAINED_MOE_ROUTER_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* A cudaStream_t passed as a plain pointer. */
typedef void* moe_stream;

/* Shape of one layer. Ds = 0: no shared expert. cf_num / cf_den is the
 * capacity factor (5/4 = 1.25 on the diagnostics page). */
typedef struct {
  int32_t T, H, E, K, D, Ds;
  int32_t dtype;            /* moe_dtype */
  int32_t cf_num, cf_den;
} moe_layer_desc;

/* Weights of one layer (device pointers). expert_bias may be NULL (B = 0);
 * ws1 / ws2 are ignored when Ds = 0. */
typedef struct {
  const void* w_router;     /* [E, H]      */
  const void* w1;           /* [E, D, H]   */
  const void* w2;           /* [E, H, D]   */
  const void* ws1;          /* [Ds, H]     */
  const void* ws2;          /* [H, Ds]     */
  const float* expert_bias; /* [E] fp32    */
} moe_layer_weights;

/* Optional routing outputs of moe_layer_forward (each member may be NULL). */
typedef struct {
  int32_t* topk_idx;        /* [T, K]   */
  float* topk_w;            /* [T, K]   */
  int32_t* counts;          /* [E]      */
  int32_t* offsets;         /* [E + 1]  */
  int32_t* perm;            /* [T * K]  */
  int32_t* inv;             /* [T * K]  */
  float* logits;            /* [T, E]   */
} moe_routing;

/* Load statistics of one routing step (host struct). */
typedef struct {
  int64_t num_copies;       /* T * K */
  int64_t overflow;         /* sum_e max(0, counts[e] - capacity) */
  int32_t capacity;         /* floor(T*K*cf_num / (E*cf_den)) */
  int32_t max_load, min_load;
  int32_t num_stragglers;   /* #experts with counts[e] > capacity */
  double skew_ratio;        /* max_load / (min_load + 1e-5) */
  double gini;              /* (2*sum_i i*c_(i) - (n+1)*S) / (n*S), 0 if S = 0 */
  double overflow_rate;     /* overflow / (T*K), 0 if T*K = 0 */
  double max_over_mean;     /* max_load / (T*K / E), 0 if T*K = 0 */
} moe_stats;

/* Bytes of workspace every call below needs for this shape (one size for
 * all calls). Returns 0 for an invalid descriptor. */
size_t moe_workspace_size(const moe_layer_desc* desc);

/* Router: logits, fp32 selection scores s = l + B, top-K, renormalised
 * weights.  "Kimi K3 fine-grained MoE ...", FineGrainedMoERouter.forward;
 * "Kimi K3 专家路由不均衡诊断" §四 (Score = Softmax(Logits + B)).
 *   x [T, H], w_router [E, H] (desc->dtype); bias [E] fp32 or NULL;
 *   logits_or_null [T, E] fp32 output (optional);
 *   topk_idx [T, K] int32 and topk_w [T, K] fp32 outputs. */
moe_status moe_router_topk(const moe_layer_desc* desc, const void* x, const void* w_router,
                           const float* bias, float* logits_or_null, int32_t* topk_idx,
                           float* topk_w, void* ws, size_t ws_bytes, moe_stream stream);

/* The selection step alone, from given fp32 logits [T, E]: s = l + B (fp32
 * add), top-K with ties to the lower index, w_k = exp(s_k - s_max) / sum.
 * Same router code as above. */
moe_status moe_topk_from_logits(const moe_layer_desc* desc, const float* logits,
                                const float* bias, int32_t* topk_idx, float* topk_w,
                                moe_stream stream);

/* Noisy routing: "MoE architecture in production" §2.3 adds Gumbel noise to
 * the logits before the softmax at inference, so the top-K choice is
 * randomised and hot experts do not stay fixed. The caller draws the noise:
 *   gumbel_noise [T, E] fp32 (device, required, 16-byte aligned), standard
 *   Gumbel draws (e.g. -log(-log(u)), u uniform in (0, 1)); scaling them
 *   sets the temperature.
 * Scores s = (l + B) + g, each add in fp32 in that order; selection, slot
 * order and weights (renormalised softmax of the selected noisy scores) as
 * in moe_topk_from_logits. Deterministic for given noise. */
moe_status moe_topk_from_logits_noisy(const moe_layer_desc* desc, const float* logits,
                                      const float* bias, const float* gumbel_noise,
                                      int32_t* topk_idx, float* topk_w, moe_stream stream);

/* Dispatch: per-expert histogram, exclusive prefix-sum offsets and the
 * stable permutation of the T*K copies into expert-contiguous rows.
 * "MoE architecture in production" §3.1 (MoEDispatcher.dispatch);
 * "Kimi K3 专家路由不均衡诊断" §三 (np.add.at counts) and §五 (no dropping).
 *   topk_idx [T, K] int32 in [0, E) (input);
 *   counts [E], offsets [E + 1], perm [T*K], inv [T*K] int32 outputs:
 *   copy c = t*K + k lands in row inv[c]; perm[row] = c.
 * A copy whose index is outside [0, E) is not placed: counts then sum to
 * less than T*K, its inv entry is -1 and the rows past the placed copies
 * hold perm = -1; the workspace status word records it, and moe_check_status
 * reports MOE_ERR_INVALID_ARG. moe_combine skips copies with inv = -1. */
moe_status moe_dispatch(const moe_layer_desc* desc, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                        size_t ws_bytes, moe_stream stream);

/* moe_dispatch for callers that cannot allocate device memory (a plugin
 * whose host runtime owns every allocation, a server whose memory pool is
 * fully reserved after warm-up, a latency-critical path that cannot afford
 * cudaMalloc's implicit synchronisation). The pages have no counterpart of
 * this call; it exists only for such callers.
 * Same arguments and results as moe_dispatch, without a workspace: the
 * scratch (per-chunk histograms) lives in a 128.25 KiB array of device
 * memory inside the library, held by every GPU that loads it until the
 * process exits. Limit: T*K <= 65536 (plus the usual E <= 512, K <= 16);
 * larger batches return MOE_ERR_UNSUPPORTED without launching. The first
 * call on a device looks up the array's device address (once per device,
 * with that device current) and caches it: do not call it after
 * cudaDeviceReset on that device (the cached address belongs to the
 * destroyed context). All calls share
 * the array, so calls that overlap on the GPU race.
 * Out-of-range indices are handled as in moe_dispatch (inv = -1, perm = -1
 * past the placed copies, counts summing to less than T*K) but are not
 * reported through a status word: a caller that cannot trust its indices
 * checks that counts sum to T*K. Allocates nothing. */
moe_status moe_dispatch_noalloc(const moe_layer_desc* desc, const int32_t* topk_idx,
                                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                moe_stream stream);

/* Grouped expert FFN over the dispatched rows, plus the shared expert.
 * "MoE architecture in production" §3.1 (experts of Linear, GeLU, Linear);
 * "Kimi K3 fine-grained MoE ...", section "通信-计算时间比的代数拐点"
 * (2*H*D multiply-adds per copy and layer).
 *   y_rows[row, :] = GeLU(x[perm[row] / K] W1[e]^T) W2[e]^T for every row of
 *   expert e's segment offsets[e] .. offsets[e+1]-1; y_rows [T*K, H] fp32.
 *   y_shared [T, H] fp32 = GeLU(x Ws1^T) Ws2^T when Ds > 0 (else may be NULL).
 *   GeLU is the exact erf form. Accumulation is fp32; the GeLU output that
 *   feeds the second Linear is rounded to desc->dtype (the tensor-core
 *   operand type for bf16 layers). */
moe_status moe_grouped_ffn(const moe_layer_desc* desc, const void* x, const int32_t* perm,
                           const int32_t* offsets, const void* w1, const void* w2,
                           const void* ws1, const void* ws2, void* y_rows, void* y_shared,
                           void* ws, size_t ws_bytes, moe_stream stream);

/* Combine: y[t] = sum_{k=0}^{K-1} topk_w[t,k] * y_rows[inv[t*K+k]] (+ y_shared[t]),
 * y_rows / y_shared fp32, summed in fp32 in that order, rounded once to
 * desc->dtype. No residual.
 * "Kimi K3 fine-grained MoE ...", section "物理通信拓扑" (combine phase);
 * "MoE architecture in production" §3.1 (scatter back to original order). */
moe_status moe_combine(const moe_layer_desc* desc, const void* y_rows, const float* topk_w,
                       const int32_t* inv, const void* y_shared_or_null, void* y,
                       moe_stream stream);

/* The whole layer: router, dispatch, grouped FFN (+ shared), combine.
 * y [T, H]. routing_or_null: optional copies of the routing tensors.
 * Every launch goes to `stream`, and no host decision depends on device
 * data, so the call can be captured into a CUDA graph and replayed (the
 * graph keeps the pointers and the shape of the captured call). The first
 * call for a device must run outside capture: it sets kernel attributes. */
moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* weights,
                             const void* x, void* y, const moe_routing* routing_or_null,
                             void* ws, size_t ws_bytes, moe_stream stream);

/* moe_layer_forward with noisy routing (see moe_topk_from_logits_noisy):
 * gumbel_noise [T, E] fp32 (device, required) is added to l + B before the
 * top-K; everything after the selection is unchanged. Graph capture as for
 * moe_layer_forward (the noise pointer is captured; refill its contents
 * before each replay). */
moe_status moe_layer_forward_noisy(const moe_layer_desc* desc, const moe_layer_weights* weights,
                                   const void* x, const float* gumbel_noise, void* y,
                                   const moe_routing* routing_or_null, void* ws, size_t ws_bytes,
                                   moe_stream stream);

/* moe_layer_forward that also records caller-created CUDA events
 * (cudaEvent_t passed as plain pointers, n_events >= 6) on `stream`
 * between its stages, for timing inside a measured region:
 *   [0] start, [1] after router + selection, [2] after dispatch,
 *   [3] after expert GEMM1 (+ GeLU), [4] after expert GEMM2, [5] after combine.
 * Same results as moe_layer_forward. */
moe_status moe_layer_forward_profiled(const moe_layer_desc* desc,
                                      const moe_layer_weights* weights, const void* x, void* y,
                                      const moe_routing* routing_or_null, void* ws,
                                      size_t ws_bytes, moe_stream stream,
                                      void* const* stage_events, int n_events);

/* The two grouped expert-GEMM launches (first layer with its GeLU, second
 * layer) of the most recent moe_layer_forward on this workspace, run again
 * on the dispatched rows and tile lists that forward left in it, for timing
 * the dominant kernels of a step in isolation. Same desc, weights and x as
 * that forward; overwrites only the workspace's expert outputs. bf16 layers
 * that take the multi-launch path only (MOE_ERR_UNSUPPORTED otherwise); a
 * shared expert that ran on the library's side stream is not included.
 * "MoE architecture in production" §3.1 (experts of Linear, GeLU, Linear). */
moe_status moe_expert_gemms(const moe_layer_desc* desc, const moe_layer_weights* weights,
                            const void* x, void* ws, size_t ws_bytes, moe_stream stream);

/* Load statistics from counts [E] (device). "Kimi K3 专家路由不均衡诊断" §三
 * (analyze_batch_routing, compute_gini_coefficient); overflow copies are
 * counted, never dropped (§五). straggler_mask_or_null [E] uint8 device
 * output (1 where counts[e] > capacity). out_host: host struct. Synchronises
 * `stream`. */
moe_status moe_expert_stats(const moe_layer_desc* desc, const int32_t* counts,
                            uint8_t* straggler_mask_or_null, moe_stats* out_host, void* ws,
                            size_t ws_bytes, moe_stream stream);

/* Dynamic expert bias update, the monitor side of no-aux-loss routing:
 * "Kimi K3 专家路由不均衡诊断" §四 (an expert that stays overloaded has its
 * bias B_i lowered by a small step, one that stays idle has it raised).
 *   counts [E] int32 (device): expert loads accumulated over the caller's
 *   update period; desc->T: the tokens of that period (with K, E and the
 *   capacity factor it sets capacity = floor(T*K*cf_num / (E*cf_den)));
 *   bias [E] fp32 (device, updated in place): B_e -= gamma where
 *   counts[e] > capacity, B_e += gamma where counts[e] == 0, in fp32.
 * Asynchronous on `stream`; the next moe_layer_forward on the stream sees
 * the new bias. */
moe_status moe_bias_update(const moe_layer_desc* desc, const int32_t* counts, float* bias,
                           float gamma, moe_stream stream);

/* Expert parallelism ("Kimi K3 fine-grained MoE ...", section "物理通信拓扑":
 * dispatch All-to-All, local experts, combine All-to-All; "MoE architecture
 * in production" §3.2). Ranks own contiguous ranges of experts; the
 * exchanges themselves are the caller's collective (NCCL All-to-All into
 * each rank's own buffers); these two calls prepare the rows around them.
 *
 * Row gather: dst[r] = src[idx[r] / divisor] for r < n_rows, rows of
 * row_bytes bytes (a multiple of 16; src, dst 16-byte aligned). idx values
 * outside [0, src_rows * divisor) leave their row unwritten. With the
 * dispatch's perm and divisor K it fills an All-to-All send buffer from x;
 * with moe_ep_local_order's inv and divisor 1 it puts expert outputs back
 * in receive order. */
moe_status moe_gather_rows(const void* src, int64_t src_rows, const int32_t* idx,
                           int32_t divisor, int64_t n_rows, int64_t row_bytes, void* dst,
                           moe_stream stream);

/* Order of the rows a rank receives from G source ranks for its El
 * experts: recv_counts [G, El] int32 (device; rows of expert e from source
 * s), the rows arriving source by source, each source's in ascending expert
 * order. Outputs (device): offsets [El + 1], the expert-major segment of
 * each local expert (expert e's rows of source 0, then source 1, ...);
 * perm [R] (expert-major position -> receive position) and inv [R] (the
 * inverse), R = sum(recv_counts) <= rows_capacity (entries past the
 * capacity are not written; perm / inv may be NULL when rows_capacity = 0).
 * Limits: G, El <= 1024, G * El <= 4096. */
moe_status moe_ep_local_order(const int32_t* recv_counts, int32_t G, int32_t El,
                              int32_t* offsets, int32_t* perm, int32_t* inv,
                              int64_t rows_capacity, moe_stream stream);

/* Reads and clears the workspace status word (synchronises `stream`):
 * MOE_OK; MOE_ERR_TIMEOUT if a bounded device wait ran out (this takes
 * precedence); MOE_ERR_INVALID_ARG if a dispatch met a top-K index outside
 * [0, E). */
moe_status moe_check_status(void* ws, size_t ws_bytes, moe_stream stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status status);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all streams); for counting launches inside a measured region. */
uint64_t moe_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* FINE_GRAINED_MOE_ROUTER_B200_MOE_H */
