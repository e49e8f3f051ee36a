// Grouped expert GEMM on the 5th-generation tensor cores (sm_100a).
//
// One launch computes every tile of one of the two expert layers ("MoE
// architecture in production" §3.1: Linear -> GeLU -> Linear per expert),
// for all routed experts plus the shared expert, from a device-side tile list
// written by the dispatch step. A tile is 128 weight rows (the MMA M side) by
// up to 256 dispatched activation rows (the MMA N side, rounded up to 16):
// weights are the A operand and tokens the B operand, so a decode step with a
// handful of rows per expert still fills the 128-row MMA and the kernel
// streams each touched weight slab once.
//
// Per CTA (persistent, one per SM, 192 threads):
//   warp 4  TMA producer: weight slab [128 x 64] + activation rows [n x 64]
//           per stage into 128-byte-swizzled shared memory, 4-stage ring
//   warp 5  TMEM allocator and MMA issuer: tcgen05.mma kind::f16 (bf16 in,
//           fp32 accumulate), two 256-column TMEM accumulators so the
//           epilogue of one tile overlaps the MMAs of the next
//   warps 0-3  epilogue: tcgen05.ld of the accumulator (thread = weight row),
//           exact GeLU for the first layer, bf16 stores into row-major output
// Every mbarrier wait is bounded in time; on expiry the CTA records
// kStatusTimeout in the workspace, drains its in-flight copies and MMAs,
// frees its TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {
namespace tc {

constexpr int kBM = 128;                        // weight rows per tile (MMA M)
constexpr int kBK = 64;                         // reduction elements per stage (128 bytes)
constexpr int kBoxRows = 32;                    // activation rows per TMA box
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB
constexpr int kBBytes = kTcRows * kBK * 2;      // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccCols = 256;                   // fp32 columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024 + 256;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s bound on any wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity. Gives up (returns
// false) after kWaitNs, recording the timeout, or as soon as another role
// of this CTA has given up (when `abort_flag` is non-null).
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                             uint32_t* status) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try(bar, parity)) return true;
    if (abort_flag && *abort_flag) return false;
    if (global_ns() - t0 > kWaitNs) {
      if (abort_flag) *abort_flag = 1u;
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle (8-row atoms of 1024 bytes): start address, leading byte
// offset 16 B (unused for this layout), stride byte offset 1024 B between
// 8-row groups, descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B (both K-major), fp32
// accumulator, M = 128, N = n (multiple of 16, <= 256).
__device__ __forceinline__ uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct Side {        // routed experts (0) or the shared expert (1)
  void* out;         // output rows, row stride `ld` elements
  int ld;
  int kb;            // reduction blocks of kBK
  int m_rows;        // weight rows per group (row stride of groups in the A map)
  int out_f32;       // 1: fp32 output, 0: bf16 output
};

struct Args {
  Side side[2];
  const Tile* tiles;
  const int* n_tiles;
  uint32_t* status;
  int E;
  int gelu;
};

__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA0,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB1, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kStages * kStageBytes);
  uint64_t* full = bars;                   // [kStages] TMA landed
  uint64_t* empty = bars + kStages;        // [kStages] MMAs done reading
  uint64_t* tfull = bars + 2 * kStages;    // [2] accumulator ready
  uint64_t* tempty = bars + 2 * kStages + 2;   // [2] accumulator drained
  uint64_t* drain = bars + 2 * kStages + 4;    // [1] all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), kEpiThreads);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = *args.n_tiles;

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[kStages];
      bool issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = false, issued_parity[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const Tile tl = args.tiles[t];
        const int sd = (tl.g < args.E) ? 0 : 1;
        const Side& S = args.side[sd];
        const CUtensorMap* ma = sd ? &tmA1 : &tmA0;
        const CUtensorMap* mb = sd ? &tmB1 : &tmB0;
        const int arow = (sd ? 0 : tl.g * S.m_rows) + tl.m0;
        const int nmma = (tl.n + 15) & ~15;
        const int nbox = (nmma + kBoxRows - 1) / kBoxRows;
        const uint32_t bytes = kABytes + nbox * kBoxRows * kBK * 2;
        for (int kb = 0; kb < S.kb; ++kb) {
          if (!wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, bytes);
          const uint32_t sa = smem_u32(smem + (size_t)stage * kStageBytes);
          const uint32_t sb = sa + kABytes;
          tma_load_2d(sa, ma, kb * kBK, arow, fb);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(sb + i * kBoxRows * kBK * 2, mb, kb * kBK, tl.r0 + i * kBoxRows, fb);
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy this thread started has landed before the CTA tears down
      for (int s = 0; s < kStages; ++s)
        if (issued[s]) wait_bounded(smem_u32(&full[s]), issued_parity[s], nullptr, args.status);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const Tile tl = args.tiles[t];
        const Side& S = args.side[(tl.g < args.E) ? 0 : 1];
        const uint32_t idesc = idesc_bf16((tl.n + 15) & ~15);
        if (!wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
        for (int kb = 0; kb < S.kb; ++kb) {
          if (!wait_bounded(smem_u32(&full[stage]), phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)stage * kStageBytes);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + kABytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)   // 16 elements = 32 bytes per MMA
            mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          mma_commit(smem_u32(&empty[stage]));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&tfull[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // retire every MMA this thread issued before TMEM is released
      mma_commit(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, nullptr, args.status);
    }
  } else {
    // --------------------------------------------------------- epilogue
    int acc = 0;
    uint32_t acc_phase = 0;
    const int row = warp * 32 + lane;   // weight row of this thread within the tile
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
      const Tile tl = args.tiles[t];
      const int sd = (tl.g < args.E) ? 0 : 1;
      const Side& S = args.side[sd];
      int ok = 1;
      if (lane == 0)
        ok = wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, args.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(acc * kAccCols);
      const size_t col = (size_t)tl.m0 + row;
      for (int c0 = 0; c0 < tl.n; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)c0, r);
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int j = c0 + q;
          if (j < tl.n) {
            float v = __uint_as_float(r[q]);
            if (args.gelu) v = gelu_erf(v);
            const size_t o = (size_t)(tl.r0 + j) * S.ld + col;
            if (S.out_f32)
              static_cast<float*>(S.out)[o] = v;
            else
              static_cast<__nv_bfloat16*>(S.out)[o] = __float2bfloat16_rn(v);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols));
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D bf16 map over a row-major [rows, cols] matrix, boxes of 64 columns x
// box_rows rows, 128-byte swizzle, zero fill outside the matrix.
static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

cudaError_t launch_grouped_gemm_tc(const TcProblem& routed, const TcProblem& shared, int E,
                                   bool gelu, const Tile* tiles, const int* n_tiles,
                                   uint32_t* status, int num_sms, cudaStream_t st) {
  using namespace tc;
  static bool attr_set[64] = {false};   // per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    e = cudaFuncSetAttribute(grouped_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  CUtensorMap a0, b0, a1, b1;
  if (!make_map(&a0, routed.w, routed.w_rows, routed.kd, kBM) ||
      !make_map(&b0, routed.act, routed.act_rows, routed.kd, kBoxRows))
    return cudaErrorInvalidValue;
  const TcProblem& sh = shared.w ? shared : routed;   // unused maps still need valid encodings
  if (!make_map(&a1, sh.w, sh.w_rows, sh.kd, kBM) ||
      !make_map(&b1, sh.act, sh.act_rows, sh.kd, kBoxRows))
    return cudaErrorInvalidValue;
  Args args;
  args.side[0] = Side{routed.out, routed.ld, routed.kd / kBK, routed.m_rows, routed.out_f32};
  args.side[1] = Side{sh.out, sh.ld, sh.kd / kBK, sh.m_rows, sh.out_f32};
  args.tiles = tiles;
  args.n_tiles = n_tiles;
  args.status = status;
  args.E = E;
  args.gelu = gelu ? 1 : 0;
  count_launch();
  grouped_gemm_tc<<<num_sms, kThreads, kSmemBytes, st>>>(a0, b0, a1, b1, args);
  return cudaGetLastError();
}

}  // namespace moe
