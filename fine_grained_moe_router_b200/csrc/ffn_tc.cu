// Grouped expert GEMM on the 5th-generation tensor cores (sm_100a).
//
// One launch computes every tile of one of the two expert layers ("MoE
// architecture in production" §3.1: Linear -> GeLU -> Linear per expert),
// for all routed experts plus the shared expert, from a device-side tile list
// written by the dispatch step (or a dense tiling: the gate GEMM, and the
// shared expert when it runs on its own stream). A tile is 128 weight rows
// (the MMA M side; 256 on a CTA pair) by up to 256 dispatched activation
// rows (the MMA N side, rounded up to 16), optionally one reduction split of
// them: weights are the A operand and tokens the B operand, so a decode step
// with a handful of rows per expert still fills the MMA and the kernel
// streams each touched weight slab once.
//
// Per CTA (persistent, one per SM, 320 threads):
//   warp 8  TMA producer: weight slab [128 x 64] + activation rows [n x 64]
//           per reduction block into 128-byte-swizzled shared memory; a
//           prefill-sized CTA pair takes two reduction blocks per stage (one
//           3D box per operand: each TMA instruction costs the issuing thread
//           about a hundred cycles, which at full MMA rate made the producer
//           the bottleneck), smaller launches one per stage and up to 12
//           stages when the batch is small
//   warp 9  TMEM allocator and MMA issuer: tcgen05.mma kind::f16 (bf16 in,
//           fp32 accumulate), two 256-column TMEM accumulators so the
//           epilogue of one tile overlaps the MMAs of the next
//   warps 0-7  epilogue: tcgen05.ld of the accumulator (thread = weight row,
//           two warps per TMEM lane quarter splitting the columns), exact
//           GeLU for the first layer, stores into row-major output; a split
//           first-layer tile stores fp32 partials and its last split adds
//           them up before the GeLU
// Every mbarrier wait is bounded in time; on expiry the CTA records
// kStatusTimeout in the workspace, drains its in-flight copies and MMAs,
// frees its TMEM and returns.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "kernels.cuh"
#include "launch.cuh"

namespace moe {
namespace tc {

constexpr int kBM = 128;                        // weight rows per tile (MMA M)
constexpr int kBK = 64;                         // reduction elements per stage (128 bytes)
constexpr int kBoxRows = 32;                    // activation rows per TMA box
constexpr int kBoxBytes = kBoxRows * kBK * 2;   // 4 KB
// Tiles with more than kWideMin activation rows per CTA load them in boxes
// of kWideRows: each TMA instruction costs the issuing thread on the order
// of a hundred cycles whatever its size, so at full MMA rate four 32-row
// boxes per stage keep the producer busy most of the time.
constexpr int kWideRows = 128;
constexpr int kWideMin = 64;
constexpr int kABytes = kBM * kBK * 2;          // 16 KB
constexpr int kMaxStages = 12;
constexpr int kStageArea = 192 * 1024;          // shared memory of the operand ring
constexpr int kAccCols = 256;                   // fp32 columns per accumulator
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kEpiWarps = 8;                    // two per TMEM lane quarter
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr size_t kSmemBytes = 1024 /*barriers*/ + 1024 /*alignment*/ + kStageArea;
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
// accumulator, M = m (128, or 256 for a CTA pair), N = n (multiple of 16,
// <= 256).
__device__ __forceinline__ uint32_t idesc_bf16(int n, int m) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
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

// ---- CTA-pair (cta_group::2) forms: two SMs of a cluster share one MMA
// of M = 256; each holds half of the weight rows and half of the
// activation rows of every stage, and its own half of the accumulator.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier of either CTA of the pair (here always the leader's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x,
                                                 int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t tmem_d, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// 3D form: a box spanning two consecutive reduction blocks (the map's third
// dimension steps 64 elements along the rows), written as two K-major tiles
// one after the other.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, int y,
                                                 int z, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once every
// MMA issued so far has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
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

// 32 lanes x 64 consecutive fp32 columns of the accumulator (one register
// per column), waited for before returning.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct Side {          // routed experts (0) or the shared expert (1)
  void* out;           // output rows, row stride `ld` elements
  long long split_stride;   // elements between the partial outputs of two splits
  int ld;
  int kb;              // reduction blocks of kBK
  int kb_per;          // reduction blocks per split
  int m_rows;          // weight rows per group (row stride of groups in the A map)
  int m_valid;         // output columns below this bound are stored
  int out_f32;         // 1: fp32 output, 0: bf16 output
  int a_rows;          // rows of the weight box (kBM, or fewer for a short gate matrix)
  int splits;          // reduction splits of this side's tiles
  void* fix_out;       // first layer with splits: bf16 GeLU output (out holds fp32 partials)
  int fix_ld;
};

struct Args {
  Side side[2];
  const Tile* tiles;   // device tile list; null: dense tiling (below)
  const int* n_tiles;  // device tile count of the list
  int dense_tiles;     // dense tiling: row tiles x weight-row tiles x splits
  int dense_rows, dense_m_tiles, dense_splits;
  int dense_mtile;     // weight rows per dense tile: kBM, or 2 * kBM on CTA pairs
  int nbox_max;        // activation boxes per stage (rows per tile <= 32 * nbox_max)
  int wide;            // 1: the wide-box maps may be used (the stage holds whole wide boxes)
  int stage_bytes;     // kABytes + nbox_max * kBoxBytes
  int n_stages;        // stages in the ring (<= kMaxStages)
  uint32_t* status;
  int E;
  int gelu;
  int lockstep;        // 1: some tiles need the split fixup (epilogue warps in lockstep)
};

// Tile t of the launch: from the list, or (dense tiling, used by the gate
// GEMM) split fastest, then weight-row block, then row block.
__device__ __forceinline__ Tile tile_at(const Args& a, int t) {
  if (a.tiles) return a.tiles[t];
  Tile tl;
  tl.ks = t % a.dense_splits;
  const int q = t / a.dense_splits;
  tl.m0 = (q % a.dense_m_tiles) * a.dense_mtile;
  tl.r0 = (q / a.dense_m_tiles) * kTcRows;
  tl.n = min(kTcRows, a.dense_rows - tl.r0);
  tl.g = 0;
  return tl;
}

// Epilogue of one accumulator for the warp's TMEM lane quarter. Thread = one
// output column (o0 = its offset in output row tl.r0); accumulator column j
// goes to output row tl.r0 + j. The two warps of a quarter take alternate
// chunks of kW columns (kW = 64 for plain stores, 32 with the GeLU, whose
// temporaries need the registers). The output mode is a template
// parameter, so the per-element loop carries no branches.
enum EpiMode { kEpiF32 = 0, kEpiBf16 = 1, kEpiGeluBf16 = 2 };

template <int kW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[kW]) {
  if constexpr (kW == 64)
    tmem_ld64(taddr, r);
  else
    tmem_ld32(taddr, r);
}

template <int kMode, int kW>
__device__ __forceinline__ void epilogue_columns(uint32_t taddr, int half, int n, bool store,
                                                 void* out, size_t o0, int ld) {
  for (int c0 = half * kW; c0 < n; c0 += 2 * kW) {
    uint32_t r[kW];
    __syncwarp();
    tmem_ld_cols<kW>(taddr + (uint32_t)c0, r);
    if (!store) continue;
    const int cnt = min(kW, n - c0);
    const size_t o = o0 + (size_t)c0 * (size_t)ld;
    if (kMode == kEpiF32) {
      float* p = static_cast<float*>(out) + o;
#pragma unroll
      for (int q = 0; q < kW; ++q)
        if (q < cnt) p[(size_t)q * ld] = __uint_as_float(r[q]);
    } else {
      __nv_bfloat16* p = static_cast<__nv_bfloat16*>(out) + o;
#pragma unroll
      for (int q = 0; q < kW; ++q)
        if (q < cnt) {
          float v = __uint_as_float(r[q]);
          if (kMode == kEpiGeluBf16) v = gelu_erf(v);
          p[(size_t)q * ld] = __float2bfloat16_rn(v);
        }
    }
  }
}

__device__ __forceinline__ void epilogue_bar_sync() {   // the kEpiWarps epilogue warps only
  asm volatile("bar.sync 1, %0;" ::"r"(kEpiWarps * 32) : "memory");
}

// First-layer tile with reduction splits, after this CTA stored its fp32
// partial: the last of the tile's splits to arrive adds the partials of all
// splits in split order, applies the GeLU and stores the bf16 output. Thread
// = output column `col`; the two warps of a lane quarter take alternate rows.
// Arrivals are counted in the split-0 tile of the list (one counter per CTA
// of a pair), which the dispatch step writes as 0 every forward and the last
// arrival puts back to 0. All
// epilogue warps call this together (it holds named barriers).
constexpr int kFixRows = 4;   // rows per thread and round of loads

__device__ __noinline__ void split_fixup(const Args& args, const Tile& tl, const Side& S,
                                            uint32_t rank, int half, int col, int n,
                                            volatile int* owner) {
  __threadfence();   // this thread's partial stores are visible to the other CTAs
  epilogue_bar_sync();
  if (threadIdx.x == 0) {
    int* arrivals = const_cast<int*>(&args.tiles[tl.first_split].arrivals[rank]);
    const bool last = atomicAdd(arrivals, 1) == S.splits - 1;
    // every split has arrived, so nothing else touches the counter in this
    // launch: leave it at zero for the next launch on the same tile list
    if (last) *arrivals = 0;
    *owner = last ? 1 : 0;
  }
  epilogue_bar_sync();
  if (!*owner) return;
  __threadfence();   // the other splits' partials are visible to this CTA
  const float* src = static_cast<const float*>(S.out) + (size_t)tl.r0 * S.ld + col;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(S.fix_out) + (size_t)tl.r0 * S.fix_ld + col;
  for (int j0 = half; j0 < n; j0 += 2 * kFixRows) {
    float a[kFixRows];
#pragma unroll
    for (int i = 0; i < kFixRows; ++i) a[i] = 0.f;
    for (int p0 = 0; p0 < S.splits; p0 += 4) {
      float v[kFixRows][4];
#pragma unroll
      for (int i = 0; i < kFixRows; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = j0 + 2 * i;
          v[i][q] = (j < n && p0 + q < S.splits)
                        ? __ldcg(src + (size_t)(p0 + q) * S.split_stride + (size_t)j * S.ld)
                        : 0.f;
        }
#pragma unroll
      for (int i = 0; i < kFixRows; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (p0 + q < S.splits) a[i] = (p0 + q == 0) ? v[i][q] : __fadd_rn(a[i], v[i][q]);
    }
#pragma unroll
    for (int i = 0; i < kFixRows; ++i) {
      const int j = j0 + 2 * i;
      if (j < n) dst[(size_t)j * S.fix_ld] = __float2bfloat16_rn(gelu_erf(a[i]));
    }
  }
}

// kPair = false: one CTA per tile of 128 weight rows (MMA M = 128).
// kPair = true: a cluster of two CTAs per tile of 256 weight rows (one MMA of
// M = 256 issued by the even CTA); each CTA loads its 128 weight rows and half
// of the tile's activation rows per stage, so an SM streams a third less
// operand data per MMA cycle than with single-CTA tiles of the same N.
// kKpb: reduction blocks per ring stage (2 only on CTA pairs whose weight and
// activation maps are the 3D two-block maps).
template <bool kPair, int kKpb>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA0,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmB0w,
                    const __grid_constant__ CUtensorMap tmB1w, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base);     // first 1 KB: control
  uint64_t* full = bars;                                  // [kMaxStages] TMA landed
  uint64_t* empty = bars + kMaxStages;                    // [kMaxStages] MMAs done reading
  uint64_t* tfull = bars + 2 * kMaxStages;                // [2] accumulator ready
  uint64_t* tempty = bars + 2 * kMaxStages + 2;           // [2] accumulator drained
  uint64_t* drain = bars + 2 * kMaxStages + 4;            // [1] all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kMaxStages + 5);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile int* epi_flags = reinterpret_cast<volatile int*>(tmem_slot + 2);   // [4]
  uint8_t* ring = base + 1024;                            // stage s at s * stage_bytes
  const int n_stages = args.n_stages;
  const int stage_bytes = args.stage_bytes;
  const uint32_t rank = kPair ? cluster_rank() : 0u;     // 0: the CTA that issues the MMAs
  const bool leader = rank == 0;
  const int unit = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int n_units = kPair ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  constexpr int kTileM = kPair ? 2 * kBM : kBM;
  const int n_max = (kPair ? 2 : 1) * args.nbox_max * kBoxRows;   // rows per tile

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), (kPair ? 2 : 1) * kEpiWarps);   // one arrival per warp
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    if (kPair) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();   // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above overlaps the previous kernel; its outputs are read below
  pdl_wait();
  pdl_trigger();
  const int n_tiles = args.tiles ? *args.n_tiles : args.dense_tiles;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[kMaxStages];
      bool issued[kMaxStages];
      for (int s = 0; s < kMaxStages; ++s) issued[s] = false, issued_parity[s] = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units) {
        const Tile tl = tile_at(args, t);
        const int sd = (tl.g < args.E) ? 0 : 1;
        const Side& S = args.side[sd];
        const CUtensorMap* ma = sd ? &tmA1 : &tmA0;
        const CUtensorMap* mb = sd ? &tmB1 : &tmB0;   // (or the wide-box map, below)
        const int arow = (sd ? 0 : tl.g * S.m_rows) + tl.m0 + (int)rank * kBM;
        int nmma = (tl.n + 15) & ~15;
        if (nmma > n_max) {   // never by construction; keeps the ring in bounds
          atomicOr(args.status, kStatusBadIndex);
          nmma = n_max;
        }
        const int rows_here = kPair ? nmma / 2 : nmma;   // activation rows this CTA loads
        const int brow = tl.r0 + (int)rank * rows_here;
        // wide boxes when the tile has enough rows and the stage holds them
        // (rows past the tile's, loaded as well, feed no MMA column)
        const bool wide = args.wide && rows_here > kWideMin;
        const int box_rows = wide ? kWideRows : kBoxRows;
        const int nbox = (rows_here + box_rows - 1) / box_rows;
        if (wide) mb = sd ? &tmB1w : &tmB0w;
        // weight rows actually loaded: 128, or fewer for a gate matrix with
        // E < 128 rows (the other rows of the smem tile only feed outputs
        // that are never stored)
        const uint32_t bytes_here =
            (uint32_t)S.a_rows * kBK * 2 + (uint32_t)(nbox * box_rows) * kBK * 2;
        const int kb0 = tl.ks * S.kb_per, kb1 = min(S.kb, kb0 + S.kb_per);
        for (int kb = kb0; kb < kb1; kb += kKpb) {
          if (!wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort_flag, args.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[stage]);
          const uint32_t sa = smem_u32(ring + (size_t)stage * stage_bytes);
          const uint32_t sb = sa + kABytes;
          if constexpr (kPair && kKpb == 2) {
            // two reduction blocks (a last odd block's box reaches into the
            // next split's or past the matrix's end: loaded, never multiplied)
            if (leader) mbar_expect_tx(fb, 2u * 2u * 2u * (uint32_t)kABytes);
            const uint32_t fb0 = map_to_rank(fb, 0);
            tma_load_3d_pair(sa, ma, arow, kb, fb0);
            tma_load_3d_pair(sa + 2 * kABytes, sd ? &tmB1w : &tmB0w, brow, kb, fb0);
          } else if (kPair) {
            // the leader's barrier counts the bytes of both CTAs
            if (leader) mbar_expect_tx(fb, 2u * bytes_here);
            const uint32_t fb0 = map_to_rank(fb, 0);
            tma_load_2d_pair(sa, ma, kb * kBK, arow, fb0);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d_pair(sb + i * box_rows * kBK * 2, mb, kb * kBK, brow + i * box_rows, fb0);
          } else {
            mbar_expect_tx(fb, bytes_here);
            tma_load_2d(sa, ma, kb * kBK, arow, fb);
            for (int i = 0; i < nbox; ++i)
              tma_load_2d(sb + i * box_rows * kBK * 2, mb, kb * kBK, brow + i * box_rows, fb);
          }
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == n_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy started here has landed before the CTA pair tears down
      // (the leader's barriers count the copies of both CTAs)
      if (leader)
        for (int s = 0; s < n_stages; ++s)
          if (issued[s]) wait_bounded(smem_u32(&full[s]), issued_parity[s], nullptr, args.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = unit; ok && t < n_tiles; t += n_units) {
        const Tile tl = tile_at(args, t);
        const Side& S = args.side[(tl.g < args.E) ? 0 : 1];
        const int nmma = min((tl.n + 15) & ~15, n_max);
        const uint32_t idesc = idesc_bf16(nmma, kTileM);
        const int kb0 = tl.ks * S.kb_per, kb1 = min(S.kb, kb0 + S.kb_per);
        if (!wait_bounded(smem_u32(&tempty[acc]), acc_phase ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kAccCols);
        for (int kb = kb0; kb < kb1; kb += kKpb) {
          if (!wait_bounded(smem_u32(&full[stage]), phase, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + (size_t)stage * stage_bytes);
          // stage layout: kKpb weight tiles, then kKpb activation tiles
          const uint32_t sb = sa + (uint32_t)(kKpb * kABytes);
#pragma unroll
          for (int j = 0; j < kKpb; ++j) {
            if (kb + j >= kb1) break;
            const uint64_t adesc = sw128_desc(sa + j * kABytes);
            const uint64_t bdesc = sw128_desc(sb + j * kABytes);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {   // 16 elements = 32 bytes per MMA
              const uint32_t accum = (kb + j != kb0 || k != 0) ? 1u : 0u;
              if (kPair)
                mma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
              else
                mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
            }
          }
          if (kPair)
            mma_commit_pair(smem_u32(&empty[stage]));
          else
            mma_commit(smem_u32(&empty[stage]));
          if (++stage == n_stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (kPair)
          mma_commit_pair(smem_u32(&tfull[acc]));
        else
          mma_commit(smem_u32(&tfull[acc]));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // retire every MMA issued before TMEM is released (in both CTAs)
      if (kPair)
        mma_commit_pair(smem_u32(drain));
      else
        mma_commit(smem_u32(drain));
      wait_bounded(smem_u32(drain), 0, nullptr, args.status);
    } else if (kPair && lane == 0) {
      // the other CTA of the pair: its accumulators are written by the
      // leader's MMAs; wait for the leader's final commit before release
      wait_bounded(smem_u32(drain), 0, nullptr, args.status);
    }
  } else {
    // --------------------------------------------------------- epilogue
    // warp w reads TMEM lanes 32*(w%4) .. +31 (thread = weight row of the
    // tile) and every other column chunk of the accumulator, starting at
    // chunk w/4 (column = activation row of the tile).
    // A launch with split first-layer tiles runs the epilogue warps in
    // lockstep: one thread waits for each accumulator and the others follow
    // it through a named barrier, so all of them take the same path through
    // the barriers of the split fixup. Flags alternate by tile parity: a slot
    // is rewritten only after every warp has passed the next tile's barrier.
    // Other launches let each warp wait for the accumulator on its own.
    int acc = 0;
    uint32_t acc_phase = 0;
    const int quarter = warp & 3, half = warp >> 2;
    const int row = (int)rank * kBM + quarter * 32 + lane;
    int it = 0;
    for (int t = unit; t < n_tiles; t += n_units, ++it) {
      const Tile tl = tile_at(args, t);
      const int sd = (tl.g < args.E) ? 0 : 1;
      const Side& S = args.side[sd];
      int ok = 1;
      if (args.lockstep) {
        if (threadIdx.x == 0)
          epi_flags[it & 1] =
              wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, args.status) ? 1 : 0;
        epilogue_bar_sync();
        ok = epi_flags[it & 1];
      } else {
        if (lane == 0)
          ok = wait_bounded(smem_u32(&tfull[acc]), acc_phase, abort_flag, args.status) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * kAccCols);
      const int col = tl.m0 + row;
      const bool store = col < S.m_valid;
      const size_t part = (size_t)tl.ks * (size_t)S.split_stride;
      const int n = min(tl.n, n_max);
      const size_t o0 = part + (size_t)tl.r0 * (size_t)S.ld + (size_t)col;
      const bool fix = args.gelu && S.splits > 1;   // split first layer: partial, GeLU later
      if (fix)
        epilogue_columns<kEpiF32, 64>(taddr, half, n, store, S.out, o0, S.ld);
      else if (args.gelu)
        epilogue_columns<kEpiGeluBf16, 32>(taddr, half, n, store, S.out, o0, S.ld);
      else if (S.out_f32)
        epilogue_columns<kEpiF32, 64>(taddr, half, n, store, S.out, o0, S.ld);
      else
        epilogue_columns<kEpiBf16, 64>(taddr, half, n, store, S.out, o0, S.ld);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        const uint32_t te = smem_u32(&tempty[acc]);
        if (kPair)
          mbar_arrive_cluster(map_to_rank(te, 0));   // the leader reuses the accumulator
        else
          mbar_arrive(te);
      }
      if (fix) split_fixup(args, tl, S, rank, half, col, n, epi_flags + 2 + (it & 1));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync();   // no CTA of the pair leaves while the other may signal it
  if (warp == kMmaWarp) {
    tc_fence_after();
    if (kPair)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(kTmemCols));
    else
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
  static const EncodeTiledFn fn = [] {   // thread-safe one-time lookup
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// 2D bf16 map over a row-major [rows, cols] matrix, boxes of 64 columns x
// box_rows rows, 128-byte swizzle, zero fill outside the matrix.
// 3D bf16 map over the same matrix: (64 columns, rows, column block of 64)
// with boxes of 64 x box_rows x 2, i.e. two consecutive reduction blocks of
// box_rows rows, 128-byte swizzle, zero fill outside the matrix.
static bool make_map_2kb(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kBK, rows, cols / kBK};
  cuuint64_t strides[2] = {cols * 2, (cuuint64_t)kBK * 2};
  cuuint32_t box[3] = {(cuuint32_t)kBK, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
                                   const DenseTiling* dense, bool pair, uint32_t* status,
                                   int num_sms, cudaStream_t st, int max_ctas) {
  using namespace tc;
  // a split first layer needs the tile list (its fixup counts arrivals there)
  if (dense && gelu && routed.splits > 1) return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];   // per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(grouped_gemm_tc<false, 1>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(grouped_gemm_tc<true, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(grouped_gemm_tc<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
  }
  // A weight matrix shorter than one tile (a gate matrix with E < 128) is
  // loaded with a box of its own rows rounded up to a swizzle atom (8 rows).
  auto a_rows_of = [](const TcProblem& p) {
    return p.w_rows >= (uint64_t)kBM ? kBM : (int)((p.w_rows + 7) & ~7ull);
  };
  CUtensorMap a0, b0, a1, b1, b0w, b1w;
  if (!make_map(&a0, routed.w, routed.w_rows, routed.kd, a_rows_of(routed)) ||
      !make_map(&b0, routed.act, routed.act_rows, routed.kd, kBoxRows))
    return cudaErrorInvalidValue;
  const TcProblem& sh = shared.w ? shared : routed;   // unused maps still need valid encodings
  if (!make_map(&a1, sh.w, sh.w_rows, sh.kd, a_rows_of(sh)) ||
      !make_map(&b1, sh.act, sh.act_rows, sh.kd, kBoxRows))
    return cudaErrorInvalidValue;
  auto side = [&](const TcProblem& p) {
    Side s;
    s.a_rows = a_rows_of(p);
    s.out = p.out;
    s.split_stride = p.split_stride;
    s.ld = p.ld;
    s.kb = p.kd / kBK;
    const int splits = p.splits > 0 ? p.splits : 1;
    s.kb_per = (s.kb + splits - 1) / splits;
    s.m_rows = p.m_rows;
    s.m_valid = p.m_valid > 0 ? p.m_valid : p.m_rows;
    s.out_f32 = p.out_f32 ? 1 : 0;
    s.splits = splits;
    s.fix_out = p.fix_out;
    s.fix_ld = p.fix_ld;
    return s;
  };
  Args args;
  args.side[0] = side(routed);
  args.side[1] = side(sh);
  args.tiles = dense ? nullptr : tiles;
  args.n_tiles = n_tiles;
  args.dense_tiles = dense ? dense->tiles : 0;
  args.dense_rows = dense ? dense->rows : 0;
  args.dense_m_tiles = dense ? dense->m_tiles : 1;
  args.dense_splits = dense ? (routed.splits > 0 ? routed.splits : 1) : 1;
  args.dense_mtile = pair ? 2 * kBM : kBM;
  // Ring shape: no tile has more rows than its activation matrix, so small
  // batches get small activation boxes per stage and a deeper ring (more
  // weight bytes in flight per SM). A CTA of a pair loads half of the rows.
  uint64_t rows = routed.act_rows;
  if (shared.w) rows = std::max<uint64_t>(rows, shared.act_rows);
  const int max_n = (int)std::min<uint64_t>(kTcRows, (rows + 15) & ~15ull);
  const int rows_per_cta = pair ? max_n / 2 : max_n;
  args.nbox_max = std::max(1, (rows_per_cta + kBoxRows - 1) / kBoxRows);
  args.stage_bytes = kABytes + args.nbox_max * kBoxBytes;
  // Wide boxes where a stage holds a whole number of them and both
  // activation matrices have at least a wide box of rows.
  args.wide = ((args.nbox_max * kBoxRows) % kWideRows == 0 &&
               routed.act_rows >= (uint64_t)kWideRows && sh.act_rows >= (uint64_t)kWideRows)
                  ? 1
                  : 0;
  if (args.wide) {
    if (!make_map(&b0w, routed.act, routed.act_rows, routed.kd, kWideRows) ||
        !make_map(&b1w, sh.act, sh.act_rows, sh.kd, kWideRows))
      return cudaErrorInvalidValue;
  } else {
    b0w = b0;
    b1w = b1;
  }
  // Prefill-sized CTA pairs (a full 128-row activation box per CTA and
  // 128-row weight boxes): two reduction blocks per stage, 3D maps.
  const bool two_blocks = pair && args.wide && args.nbox_max * kBoxRows == kWideRows &&
                          a_rows_of(routed) == kBM && a_rows_of(sh) == kBM;
  if (two_blocks) {
    args.stage_bytes = 2 * (kABytes + kWideRows * kBK * 2);
    if (!make_map_2kb(&a0, routed.w, routed.w_rows, routed.kd, kBM) ||
        !make_map_2kb(&a1, sh.w, sh.w_rows, sh.kd, kBM) ||
        !make_map_2kb(&b0w, routed.act, routed.act_rows, routed.kd, kWideRows) ||
        !make_map_2kb(&b1w, sh.act, sh.act_rows, sh.kd, kWideRows))
      return cudaErrorInvalidValue;
  }
  args.n_stages = std::min(kMaxStages, kStageArea / args.stage_bytes);
  args.status = status;
  args.E = E;
  args.gelu = gelu ? 1 : 0;
  args.lockstep = (gelu && (args.side[0].splits > 1 || args.side[1].splits > 1)) ? 1 : 0;
  const int sms = (max_ctas > 0) ? std::min(num_sms, max_ctas) : num_sms;
  if (!pair) {
    const int grid = dense ? std::min(sms, std::max(1, dense->tiles)) : sms;
    return launch_pdl(grouped_gemm_tc<false, 1>, dim3(grid), dim3(kThreads), kSmemBytes, st, a0,
                      b0, a1, b1, b0w, b1w, args);
  }
  const int pairs = dense ? std::min(sms / 2, std::max(1, dense->tiles)) : sms / 2;
  if (two_blocks)
    return launch_pdl_cluster2(grouped_gemm_tc<true, 2>, dim3(2 * std::max(1, pairs)),
                               dim3(kThreads), kSmemBytes, st, a0, b0, a1, b1, b0w, b1w, args);
  return launch_pdl_cluster2(grouped_gemm_tc<true, 1>, dim3(2 * std::max(1, pairs)), dim3(kThreads),
                             kSmemBytes, st, a0, b0, a1, b1, b0w, b1w, args);
}

}  // namespace moe
