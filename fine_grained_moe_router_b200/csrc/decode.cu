// Single-launch forward of a bf16 MoE layer for a handful of tokens (decode).
//
// With T <= 2 tokens every expert GEMM of the layer is a matrix-vector
// product against at most four activation rows: the step is bound by the
// weight bytes it streams from HBM ("Kimi K3 fine-grained MoE under high
// concurrency", section "通信-计算时间比的代数拐点": 2*H*D multiply-adds per
// copy against 2*H*D weight elements per touched expert). The multi-launch
// path spends a large part of such a step between kernels, so this kernel
// runs the whole layer in one cooperative launch (one CTA per SM):
//
//   router   gate logits l = x W_r^T, W_r rows split over the CTAs
//            ("Kimi K3 ...", FineGrainedMoERouter; "MoE architecture in
//            production" §2.3); grid barrier 1
//   select   warp 0 of every CTA takes the top K of s = l + B (+ g) and
//            renormalises ("Kimi K3 专家路由不均衡诊断" §四), then sorts the T*K
//            copies by expert, stable in copy order ("MoE architecture in
//            production" §3.1): counts, offsets, perm, inv; meanwhile the
//            other warps run the shared expert's first layer, which does not
//            depend on the routing
//   GEMM1    Hm = GeLU(x W1[e]^T) for the touched experts and Hs = GeLU(x
//            Ws1^T) for the shared expert: each kind of weight rows is split
//            evenly over the CTAs; grid barrier 2
//   GEMM2    CTA i owns the output columns h of one contiguous range and
//            computes, for each touched expert, Yr[row, h] = Hm[row] . W2[e,h]
//            and S[t, h] = Hs[t] . Ws2[h]; the combine y[t, h] = sum_k w[t,k]
//            Yr[inv[t,k], h] + S[t, h] ("Kimi K3 ...", section "物理通信拓扑",
//            combine phase) follows in the same CTA, k ascending, fp32.
//
// Weight streaming: a phase's weight rows are cut into chunks of 32 16-byte
// vectors, and each warp of the CTA takes an equal contiguous range of them
// (whatever the rows' lengths), copied from HBM with cp.async into a private
// ring of shared-memory stages of 4 KB, a few segments in flight while one
// is multiplied (fused bf16 x bf16 + fp32 multiply-adds) with the activation
// rows, which are staged once per phase in shared memory (x, then the first
// layer's outputs). The lanes' partial sums of a row are added by a shuffle
// butterfly; a row that a warp boundary cuts is finished after the phase
// from the warps' sums, in warp order. Every order of additions is fixed, so
// results are deterministic. The only CTA-wide synchronisation is at phase
// boundaries.
//
// Every wait is bounded in time (the grid barriers): on expiry the CTA sets
// kStatusTimeout in the workspace and skips the rest of the layer. The grid
// barrier counters live in the workspace header and are reset to zero by the
// last CTA to finish.
#include <atomic>

#include "common.cuh"
#include "kernels.cuh"
#include "select.cuh"

namespace moe {
namespace dec {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxRowLen = 16384;                    // elements of the longest weight row
constexpr int kMaxCopies = kDecodeMaxT * kMaxK;      // 32
constexpr unsigned long long kWaitNs = 2000000000ull;

struct Params {
  const __nv_bfloat16* x;
  const __nv_bfloat16* wr;
  const float* bias;     // nullable
  const float* noise;    // nullable
  const __nv_bfloat16* w1;
  const __nv_bfloat16* w2;
  const __nv_bfloat16* ws1;
  const __nv_bfloat16* ws2;
  __nv_bfloat16* y;
  float* logits;
  int32_t* idx;
  float* tw;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  __nv_bfloat16* hm;     // [T*K, D], rows in dispatch order
  __nv_bfloat16* hs;     // [T, Ds]
  WsHeader* hdr;
  int T, H, E, K, D, Ds;
  int h_rows;            // rows of the largest GEMM2 column range of one CTA
};

// Shared memory: this struct, then the ycache / scache of the fused combine,
// then the activation staging area.
struct Smem {
  int32_t perm[kMaxCopies];
  int32_t inv[kMaxCopies];
  int32_t idx[kMaxCopies];
  float w[kMaxCopies];
  int32_t seg_e[kMaxCopies];
  int32_t seg_off[kMaxCopies + 1];
  int32_t n_seg;
  uint32_t abort_flag;
};

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// 16 bytes of a weight row, read once: not kept in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// [i*n/G, (i+1)*n/G): CTA i's share of n units.
__device__ __forceinline__ void share(long long n, int i, int G, int* a, int* b) {
  *a = (int)(n * i / G);
  *b = (int)(n * (i + 1) / G);
}

// acc + the dot product of 8 bf16 pairs, in element order: each step is one
// fused multiply-add of two bf16 values (exact in fp32) into the fp32
// accumulator with a single rounding, i.e. fmaf on the widened values.
__device__ __forceinline__ float fma_bf16x2(uint32_t w, uint32_t a, float acc) {
  asm("{\n\t.reg .b16 wl, wh, al, ah;\n\t"
      "mov.b32 {wl, wh}, %1;\n\tmov.b32 {al, ah}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wl, al, %0;\n\tfma.rn.f32.bf16 %0, wh, ah, %0;\n\t}"
      : "+f"(acc)
      : "r"(w), "r"(a));
  return acc;
}

__device__ __forceinline__ float dot8(const uint4& w, const uint4& a, float acc) {
  acc = fma_bf16x2(w.x, a.x, acc);
  acc = fma_bf16x2(w.y, a.y, acc);
  acc = fma_bf16x2(w.z, a.z, acc);
  acc = fma_bf16x2(w.w, a.w, acc);
  return acc;
}

// Waits (one thread) until a grid barrier counter reaches `target`; false
// (and the CTA's abort flag, the status bit) after kWaitNs.
__device__ bool grid_wait(const uint32_t* ctr, uint32_t target, Smem& s, const Params& p) {
  const uint64_t t0 = global_ns();
  while (ld_acquire(ctr) < target) {
    if (global_ns() - t0 > kWaitNs) {
      s.abort_flag = 1u;
      atomicOr(&p.hdr->status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// This CTA's arrival on the grid barrier, after every thread's stores of the
// phase (the __syncthreads orders them before thread 0's fence and release).
__device__ __forceinline__ void grid_arrive(const Params& p) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    red_release_add(&p.hdr->tickets[0], 1u);
  }
}

enum Out : int { kLogits = 0, kHs, kHm, kYr, kS };

// One matrix's rows [r0, r1) for this CTA (row length L): a job. A phase is a
// list of jobs, each against A <= kDecodeMaxT activation rows staged in
// shared memory (16-byte vector offsets act[0..A) from the staging base). Row
// r's result for activation row a goes to the output `out`: logits[a, r];
// Hs[a, r] or Hm[seg_off + a, r] after the GeLU (bf16); Yr (ycache[r - h0,
// seg_off + a]) or S (scache[r - h0, a]).
//
// The phase's weight bytes are cut into chunks of 32 16-byte vectors (one
// per lane; a row of nvec vectors takes cpr = ceil(nvec / 32) chunks, the
// last one masked past nvec), numbered job by job, row by row; chunk c0 is
// the job's first. Warp wi of nw takes the contiguous chunks [C wi / nw,
// C (wi + 1) / nw) of the phase's C, so every warp streams the same number of
// bytes whatever the rows' lengths; a row cut by a warp boundary is finished
// after the phase from the warps' partial sums, added in warp order.
struct RowJob {
  const __nv_bfloat16* w;
  int r0, r1, L;
  int act[kDecodeMaxT];
  int A, out, seg_off, h0;
  int nvec, cpr, c0;
};

// Fills nvec, cpr and c0 of a phase's jobs; returns the phase's chunks.
__device__ __forceinline__ int number_chunks(RowJob* jobs, int n) {
  int c = 0;
  for (int j = 0; j < n; ++j) {
    jobs[j].nvec = jobs[j].L / 8;
    jobs[j].cpr = (jobs[j].nvec + 31) / 32;
    jobs[j].c0 = c;
    c += (jobs[j].r1 - jobs[j].r0) * jobs[j].cpr;
  }
  return c;
}

// A row that a warp boundary cuts: each warp's sum over its part (slot 0:
// the first row of the warp's range, slot 1: the last). `head`: the part
// holds the row's first chunk; `tail`: its last.
struct Partial {
  int valid, head, tail, job, row;
  float v[kDecodeMaxT];
};

constexpr int kMaxJobs = kMaxCopies + 1;   // every touched expert + the shared expert
// A CTA's share of the first layer's rows (ns * D rows of ns <= 64 touched
// experts, over at least 64 CTAs) is at most D rows, so it meets at most two
// experts' row blocks.
constexpr int kMaxG1Jobs = 4;
constexpr int kMinCtas = kMaxCopies;
constexpr int kVpl = 8;                    // chunks per lane per stage (4 KB a warp)
// shared memory of the per-warp rings with kStages stages
constexpr size_t ring_bytes(int stages) { return (size_t)kWarps * stages * kVpl * 32 * 16; }

// Result v of row r (of job jb) for activation row a.
__device__ __forceinline__ void emit(const RowJob& jb, const Params& p, int r, int a, float v,
                                     float* ycache, float* scache) {
  switch (jb.out) {
    case kLogits:
      p.logits[(size_t)a * p.E + r] = v;
      break;
    case kHs:
      p.hs[(size_t)a * p.Ds + r] = __float2bfloat16_rn(gelu_erf(v));
      break;
    case kHm:
      p.hm[(size_t)(jb.seg_off + a) * p.D + r] = __float2bfloat16_rn(gelu_erf(v));
      break;
    case kYr:
      ycache[(size_t)(r - jb.h0) * p.T * p.K + jb.seg_off + a] = v;
      break;
    default:
      scache[(size_t)(r - jb.h0) * p.T + a] = v;
      break;
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Position in a warp's chunk range: job j, row `row` of the job, chunk cc of
// the row, `left` chunks to go.
struct Cursor {
  int j, row, cc, left;
};

// Cursor at chunk c of the phase with `left` chunks to go.
__device__ __forceinline__ Cursor seek(const RowJob* jobs, int n_jobs, int c, int left) {
  Cursor k{0, 0, 0, left};
  if (left <= 0) return k;
  // the last job starting at or before c (jobs without rows share their c0
  // with the next one)
  while (k.j + 1 < n_jobs && jobs[k.j + 1].c0 <= c) ++k.j;
  const int local = c - jobs[k.j].c0;
  k.row = local / jobs[k.j].cpr;
  k.cc = local % jobs[k.j].cpr;
  return k;
}

// Moves k past `run` chunks of its current row (run <= the chunks left in
// the row); at the row's end to the next row, or the next job with rows.
__device__ __forceinline__ void step(Cursor& k, const RowJob* jobs, int n_jobs, int run, int cpr,
                                     int rows) {
  k.left -= run;
  k.cc += run;
  if (k.cc < cpr) return;
  k.cc = 0;
  if (++k.row < rows) return;
  k.row = 0;
  do ++k.j;
  while (k.j < n_jobs && jobs[k.j].r1 == jobs[k.j].r0);
}

// The calling warp's range of a phase's chunks as a stream: each lane copies
// its own vectors of the next segments (kVpl chunks) into the warp's private
// ring of kStages stages with cp.async (kStages - 1 segments in flight while
// one is multiplied; a lane reads back only what it copied itself, so no
// synchronisation is needed). prime() puts the first kStages - 1 segments in
// flight (weights only: it may run before the activations are staged); run()
// multiplies the whole range. A segment is walked in runs of chunks of one
// row; each row keeps two partial sums per activation row (alternate chunks
// of a run), added before the lanes' butterfly.
template <int kStages>
struct JobStream {
  const RowJob* jobs;
  int n_jobs, wi, n;
  Cursor in, out;
  uint4* my_ring;
  uint32_t my_ring_s;

  __device__ void init(const RowJob* jobs_, int n_jobs_, int chunks, int wi_, int nw,
                       uint4* ring) {
    const int lane = threadIdx.x & 31;
    jobs = jobs_;
    n_jobs = n_jobs_;
    wi = wi_;
    n = 0;
    my_ring = ring + (size_t)(threadIdx.x >> 5) * kStages * kVpl * 32 + lane;
    my_ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(my_ring));
    const int c0 = (int)((long long)chunks * wi / nw);
    const int c1 = (int)((long long)chunks * (wi + 1) / nw);
    in = seek(jobs, n_jobs, c0, c1 - c0);
    out = in;
  }
  // copies of the next segment at `in` into stage st
  __device__ void issue(int st) {
    const int lane = threadIdx.x & 31;
    const int nq = min(kVpl, in.left);
    for (int q = 0; q < nq;) {
      const RowJob& jb = jobs[in.j];
      const int cpr = jb.cpr;
      const int run = min(nq - q, cpr - in.cc);
      const int v0 = in.cc * 32 + lane;
      const uint4* src =
          reinterpret_cast<const uint4*>(jb.w + (size_t)(jb.r0 + in.row) * jb.L) + v0;
      const int vleft = jb.nvec - v0;   // vectors of the row from this lane's first on
      uint32_t dst = my_ring_s + (uint32_t)((st * kVpl + q) * 32 * 16);
      for (int i = 0; i < run; ++i, dst += 32 * 16)
        if (32 * i < vleft) cp_async16(dst, src + 32 * i);
      q += run;
      step(in, jobs, n_jobs, run, cpr, jb.r1 - jb.r0);
    }
    cp_async_commit();   // (an empty group at the end keeps the wait count uniform)
  }
  __device__ void prime() {
    for (int st = 0; st < kStages - 1; ++st) issue(st);
  }
  template <int kA>
  __device__ void run(const Params& p, const uint4* stage, float* ycache, float* scache,
                      Partial* part) {
    const int lane = threadIdx.x & 31;
    float acc0[kA], acc1[kA];
#pragma unroll
    for (int a = 0; a < kA; ++a) acc0[a] = acc1[a] = 0.f;
    bool head = out.cc == 0;   // the current row's first chunk is in this range
    int slot = 0;              // partial slot of the next row finished here
    while (out.left > 0) {
      issue((n + kStages - 1) % kStages);
      asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1) : "memory");   // segment n landed
      const uint4* buf = my_ring + (size_t)(n % kStages) * kVpl * 32;
      const int nq = min(kVpl, out.left);
      for (int q = 0; q < nq;) {
        const RowJob& jb = jobs[out.j];
        const int cpr = jb.cpr, A = jb.A;
        const int run = min(nq - q, cpr - out.cc);
        const int v0 = out.cc * 32 + lane;
        const int vleft = jb.nvec - v0;
        const uint4* w = buf + q * 32;
        const uint4* x[kA];
#pragma unroll
        for (int a = 0; a < kA; ++a) x[a] = stage + jb.act[a] + v0;
        int i = 0;
        for (; i + 1 < run; i += 2) {
          if (32 * i < vleft) {
            const uint4 wv = w[32 * i];
#pragma unroll
            for (int a = 0; a < kA; ++a)
              if (a < A) acc0[a] = dot8(wv, x[a][32 * i], acc0[a]);
          }
          if (32 * (i + 1) < vleft) {
            const uint4 wv = w[32 * (i + 1)];
#pragma unroll
            for (int a = 0; a < kA; ++a)
              if (a < A) acc1[a] = dot8(wv, x[a][32 * (i + 1)], acc1[a]);
          }
        }
        if (i < run && 32 * i < vleft) {
          const uint4 wv = w[32 * i];
#pragma unroll
          for (int a = 0; a < kA; ++a)
            if (a < A) acc0[a] = dot8(wv, x[a][32 * i], acc0[a]);
        }
        q += run;
        const bool tail = out.cc + run == cpr;
        if (tail || out.left == run) {   // the row ends here, or the range does
          float sum[kA];
#pragma unroll
          for (int a = 0; a < kA; ++a) {
            sum[a] = acc0[a] + acc1[a];
            acc0[a] = acc1[a] = 0.f;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int a = 0; a < kA; ++a) sum[a] += __shfl_xor_sync(0xffffffffu, sum[a], o);
          float mine = sum[0];
#pragma unroll
          for (int a = 1; a < kA; ++a)
            if (lane == a) mine = sum[a];
          if (head && tail) {
            if (lane < A) emit(jb, p, jb.r0 + out.row, lane, mine, ycache, scache);
          } else {
            Partial& pt = part[2 * wi + slot];
            if (lane < kDecodeMaxT) pt.v[lane] = mine;
            if (lane == 0) {
              pt.valid = 1;
              pt.head = head ? 1 : 0;
              pt.tail = tail ? 1 : 0;
              pt.job = out.j;
              pt.row = out.row;
            }
          }
          slot = 1;
          head = true;
        }
        step(out, jobs, n_jobs, run, cpr, jb.r1 - jb.r0);
      }
      ++n;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  }
};

// Rows cut by the warp boundaries of a phase (nw warps): the part holding a
// row's first chunk adds the parts of the following warps in warp order and
// emits the row. Called by all threads after the phase's parts are visible
// (a __syncthreads); each row is finished by one thread.
__device__ void finish_cut_rows(const RowJob* jobs, const Partial* part, int nw, const Params& p,
                                float* ycache, float* scache) {
  const int i = threadIdx.x;
  if (i >= 2 * nw) return;
  const Partial& h = part[i];
  if (!h.valid || !h.head) return;
  float v[kDecodeMaxT];
#pragma unroll
  for (int a = 0; a < kDecodeMaxT; ++a) v[a] = h.v[a];
  bool done = h.tail != 0;
  for (int w = (i >> 1) + 1; w < nw && !done; ++w) {
    const Partial& c = part[2 * w];   // the row goes on as the next range's first row
    if (!c.valid) continue;           // (a warp with an empty range)
#pragma unroll
    for (int a = 0; a < kDecodeMaxT; ++a) v[a] += c.v[a];
    done = c.tail != 0;
  }
  const RowJob& jb = jobs[h.job];
#pragma unroll
  for (int a = 0; a < kDecodeMaxT; ++a)
    if (a < jb.A) emit(jb, p, jb.r0 + h.row, a, v[a], ycache, scache);
}

// Top-K selection and dispatch of the T <= 2 tokens by one warp, into shared
// memory; CTA 0 also writes the routing outputs.
__device__ void route(Smem& s, const Params& p, const float* bias, const float* noise) {
  const int lane = threadIdx.x & 31;
  const int T = p.T, E = p.E, K = p.K, TK = T * K;
  for (int t = 0; t < T; ++t) {
    float sc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int e = lane + 32 * j;
      float v = -INFINITY;
      if (e < E) {
        const float l = __ldcg(p.logits + (size_t)t * E + e);
        v = __fadd_rn(l, bias[e]);
        if (noise) v = __fadd_rn(v, noise[(size_t)t * E + e]);   // Gumbel noise, after B
      }
      sc[j] = v;
    }
    select_topk_warp<16>(sc, E, K, s.idx + t * K, s.w + t * K);
  }
  __syncwarp();
  // stable sort of the copies by expert: row of copy c = #{c' : (e', c') < (e, c)}
  int rank[2] = {0, 0}, ec[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) ec[h] = (lane + 32 * h < TK) ? s.idx[lane + 32 * h] : INT_MAX;
  for (int c2 = 0; c2 < TK; ++c2) {
    const int e2 = s.idx[c2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = lane + 32 * h;
      rank[h] += (e2 < ec[h]) || (e2 == ec[h] && c2 < c);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = lane + 32 * h;
    if (c < TK) {
      s.inv[c] = rank[h];
      s.perm[rank[h]] = c;
    }
  }
  __syncwarp();
  // segments of equal experts in dispatch order
  int starts = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = lane + 32 * h;
    bool st = false;
    if (r < TK) st = (r == 0) || (s.idx[s.perm[r]] != s.idx[s.perm[r - 1]]);
    const unsigned b = __ballot_sync(0xffffffffu, st);
    if (st) {
      const int si = starts + __popc(b & ((1u << lane) - 1u));
      s.seg_e[si] = s.idx[s.perm[r]];
      s.seg_off[si] = r;
    }
    starts += __popc(b);
  }
  if (lane == 0) {
    s.n_seg = starts;
    s.seg_off[starts] = TK;
  }
  __syncwarp();
  if (blockIdx.x != 0) return;
  // routing outputs (CTA 0)
  for (int c = lane; c < TK; c += 32) {
    p.idx[c] = s.idx[c];
    p.tw[c] = s.w[c];
    p.perm[c] = s.perm[c];
    p.inv[c] = s.inv[c];
  }
  const int ns = s.n_seg;
  for (int e = lane; e <= E; e += 32) {
    // offsets[e] = rows of the experts below e: the first segment with expert >= e
    int lo = 0, hi = ns;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s.seg_e[mid] < e) lo = mid + 1; else hi = mid;
    }
    p.offsets[e] = s.seg_off[lo];
    if (e < E) p.counts[e] = (lo < ns && s.seg_e[lo] == e) ? s.seg_off[lo + 1] - s.seg_off[lo] : 0;
  }
}

// Job lists of the phases (shared memory).
struct Jobs {
  RowJob router;            // this CTA's W_r rows
  RowJob shared1;           // this CTA's Ws1 rows
  RowJob g1[kMaxG1Jobs];    // the routed experts' W1 rows of this CTA
  RowJob g2[kMaxJobs];      // this CTA's output columns of each touched W2, then of Ws2
  int n_g1, n_g2;
  int c_router, c_shared1, c_g1, c_g2;   // chunks of each phase's jobs
  // rows cut between warps: [0] the shared expert's first layer, [1] the
  // routed first layer, then (after grid barrier 2) the second layer
  Partial part[2][2 * kWarps];
};

// Lists the first- and second-layer jobs of this CTA once the routing is in
// shared memory (one thread).
__device__ void list_jobs(const Smem& s, Jobs& J, const Params& p, int h0, int h1) {
  const int G = gridDim.x, cta = blockIdx.x;
  const int ns = s.n_seg, H = p.H, K = p.K, TK = p.T * p.K;
  // the touched experts' W1 rows, in ascending expert order, split evenly
  // over the CTAs: one job per expert in this CTA's range
  int a, b, n = 0;
  share((long long)ns * p.D, cta, G, &a, &b);
  for (int j = 0; j < ns; ++j) {
    const int lo = max(a, j * p.D), hi = min(b, (j + 1) * p.D);
    if (lo >= hi) continue;
    if (n == kMaxG1Jobs) {   // never with at least kMinCtas CTAs (above)
      atomicOr(&p.hdr->status, kStatusBadIndex);
      break;
    }
    RowJob jb{};
    jb.w = p.w1 + (size_t)s.seg_e[j] * p.D * H;
    jb.r0 = lo - j * p.D;
    jb.r1 = hi - j * p.D;
    jb.L = H;
    jb.seg_off = s.seg_off[j];
    jb.A = s.seg_off[j + 1] - s.seg_off[j];
    for (int q = 0; q < kDecodeMaxT; ++q)
      jb.act[q] = s.perm[jb.seg_off + (q < jb.A ? q : 0)] / K * (H / 8);
    jb.out = kHm;
    J.g1[n++] = jb;
  }
  J.n_g1 = n;
  // this CTA's output columns [h0, h1) of every touched expert's W2, then of Ws2
  n = 0;
  for (int j = 0; j < ns; ++j) {
    RowJob jb{};
    jb.w = p.w2 + (size_t)s.seg_e[j] * H * p.D;
    jb.r0 = h0;
    jb.r1 = h1;
    jb.h0 = h0;
    jb.L = p.D;
    jb.seg_off = s.seg_off[j];
    jb.A = s.seg_off[j + 1] - s.seg_off[j];
    for (int q = 0; q < kDecodeMaxT; ++q) jb.act[q] = (jb.seg_off + (q < jb.A ? q : 0)) * (p.D / 8);
    jb.out = kYr;
    J.g2[n++] = jb;
  }
  if (p.Ds > 0) {
    RowJob jb{};
    jb.w = p.ws2;
    jb.r0 = h0;
    jb.r1 = h1;
    jb.h0 = h0;
    jb.L = p.Ds;
    jb.A = p.T;
    for (int q = 0; q < kDecodeMaxT; ++q) jb.act[q] = (TK * p.D + (q < p.T ? q : 0) * p.Ds) / 8;
    jb.out = kS;
    J.g2[n++] = jb;
  }
  J.n_g2 = n;
  J.c_g1 = number_chunks(J.g1, J.n_g1);
  J.c_g2 = number_chunks(J.g2, J.n_g2);
}

template <int kA, int kStages>
__global__ void __launch_bounds__(kThreads, 1) decode_forward(const Params p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  size_t off = (sizeof(Smem) + 127) & ~size_t(127);
  Jobs& J = *reinterpret_cast<Jobs*>(smem_raw + off);
  off += (sizeof(Jobs) + 127) & ~size_t(127);
  float* ycache = reinterpret_cast<float*>(smem_raw + off);
  off += (size_t)p.h_rows * p.T * p.K * sizeof(float);
  float* scache = reinterpret_cast<float*>(smem_raw + off);
  off += (size_t)p.h_rows * p.T * sizeof(float);
  float* s_bias = reinterpret_cast<float*>(smem_raw + off);    // [E] (B = 0 when absent)
  off += (size_t)p.E * sizeof(float);
  float* s_noise = reinterpret_cast<float*>(smem_raw + off);   // [T, E] when given
  off += p.noise ? (size_t)p.T * p.E * sizeof(float) : 0;
  off = (off + 127) & ~size_t(127);
  uint4* ring = reinterpret_cast<uint4*>(smem_raw + off);
  off += ring_bytes(kStages);
  uint4* stage = reinterpret_cast<uint4*>(smem_raw + off);     // 16-byte vectors
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int T = p.T, H = p.H, K = p.K, TK = T * K;
  uint32_t* ctr = &p.hdr->tickets[0];
  int h0, h1;
  share(H, cta, G, &h0, &h1);

  if (tid == 0) {
    s.abort_flag = 0u;
    // gate logits of this CTA's W_r rows; the shared expert's first layer
    RowJob jb{};
    jb.L = H;
    jb.A = T;
    for (int a = 0; a < kDecodeMaxT; ++a) jb.act[a] = (a < T ? a : 0) * (H / 8);
    jb.w = p.wr;
    share(p.E, cta, G, &jb.r0, &jb.r1);
    jb.out = kLogits;
    J.router = jb;
    jb.w = p.ws1;
    share(p.Ds, cta, G, &jb.r0, &jb.r1);
    jb.out = kHs;
    J.shared1 = jb;
    J.c_router = number_chunks(&J.router, 1);
    J.c_shared1 = p.Ds > 0 ? number_chunks(&J.shared1, 1) : 0;
  }
  for (int i = tid; i < 2 * 2 * kWarps; i += kThreads) (&J.part[0][0])[i].valid = 0;
  // x (every token), the bias and the noise first, while nothing else is in
  // flight
  for (int v = tid; v < T * H / 8; v += kThreads)
    stage[v] = __ldg(reinterpret_cast<const uint4*>(p.x) + v);
  for (int e = tid; e < p.E; e += kThreads) s_bias[e] = p.bias ? p.bias[e] : 0.f;
  if (p.noise)
    for (int i = tid; i < T * p.E; i += kThreads) s_noise[i] = p.noise[i];
  __syncthreads();
  // warp 0 computes the gate logits of this CTA's rows, the other warps the
  // shared expert's first layer (it does not depend on the routing); the gate
  // rows are requested first, so they are at the head of the memory queues
  JobStream<kStages> js;
  if (warp == 0) {
    js.init(&J.router, 1, J.c_router, 0, 1, ring);
    js.prime();
  }
  __syncthreads();
  if (warp != 0) {
    js.init(&J.shared1, 1, J.c_shared1, warp - 1, kWarps - 1, ring);
    js.prime();
  }
  // (warp 0 streams its whole router job, so it never cuts a row)
  js.template run<kA>(p, stage, nullptr, nullptr, J.part[0]);
  if (warp == 0) {
    // grid barrier 1 (one arrival per CTA, after this warp's logit stores),
    // then the routing and the job lists of both layers
    __syncwarp();
    int ok = 1;
    if (lane == 0) {
      __threadfence();
      red_release_add(ctr, 1u);
      ok = grid_wait(ctr, (uint32_t)G, s, p) ? 1 : 0;
    }
    if (__shfl_sync(0xffffffffu, ok, 0)) {
      ld_acquire(ctr);
      route(s, p, s_bias, p.noise ? s_noise : nullptr);
      if (lane == 0) list_jobs(s, J, p, h0, h1);
    }
  }
  __syncthreads();
  JobStream<kStages> js2;
  if (!s.abort_flag) {
    ld_acquire(ctr);
    js.init(J.g1, J.n_g1, J.c_g1, warp, kWarps, ring);
    js.prime();
    js.template run<kA>(p, stage, nullptr, nullptr, J.part[1]);
    // the second layer's weights do not depend on the first layer's
    // outputs: they are in flight while grid barrier 2 is pending
    js2.init(J.g2, J.n_g2, J.c_g2, warp, kWarps, ring);
    js2.prime();
  }
  __syncthreads();
  if (!s.abort_flag) {
    // rows cut between warps: the shared expert's (warps 1-15 of phase 1)
    // and the routed experts' first layer
    finish_cut_rows(&J.shared1, J.part[0], kWarps - 1, p, nullptr, nullptr);
    finish_cut_rows(J.g1, J.part[1], kWarps, p, nullptr, nullptr);
  }
  grid_arrive(p);   // grid barrier 2: every CTA's Hm and Hs
  // (every thread has passed the cut-row pass above: the slots are free for
  // the second layer)
  if (tid < 2 * kWarps) J.part[1][tid].valid = 0;
  if (tid == 0 && !s.abort_flag) grid_wait(ctr, 2u * (uint32_t)G, s, p);
  __syncthreads();
  if (!s.abort_flag) {
    ld_acquire(ctr);
    // Hm [T*K, D] and Hs [T, Ds] (written by every CTA) over the x rows
    const int n_hm = TK * p.D / 8, n_all = n_hm + T * p.Ds / 8;
    for (int v = tid; v < n_all; v += kThreads)
      stage[v] = (v < n_hm) ? __ldcg(reinterpret_cast<const uint4*>(p.hm) + v)
                            : __ldcg(reinterpret_cast<const uint4*>(p.hs) + (v - n_hm));
  }
  __syncthreads();
  if (!s.abort_flag) js2.template run<kA>(p, stage, ycache, scache, J.part[1]);
  // (a CTA that gave up may still have second-layer copies in flight)
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  if (!s.abort_flag) {
    finish_cut_rows(J.g2, J.part[1], kWarps, p, ycache, scache);
    __syncthreads();
  }
  if (!s.abort_flag) {
    // combine of this CTA's output columns: y[t, h] = sum_k w[t,k]
    // Yr[inv[t,k], h] (+ S[t, h]), fp32 in k order, one rounding
    const int n = (h1 - h0) * T;
    for (int f = tid; f < n; f += kThreads) {
      const int hl = f / T, t = f % T;
      float acc = 0.f;
      for (int k = 0; k < K; ++k)
        acc = fmaf(s.w[t * K + k], ycache[(size_t)hl * TK + s.inv[t * K + k]], acc);
      if (p.Ds > 0) acc += scache[(size_t)hl * T + t];
      p.y[(size_t)t * H + h0 + hl] = __float2bfloat16_rn(acc);
    }
  }
  if (tid == 0) {
    // the last CTA to finish resets the grid barrier counters: every CTA has
    // passed both barriers (or given up) before it counts itself out here
    __threadfence();
    const uint32_t n = atomicAdd(&p.hdr->tickets[1], 1u);
    if (n == gridDim.x - 1) {
      atomicExch(&p.hdr->tickets[0], 0u);
      atomicExch(&p.hdr->tickets[1], 0u);
    }
  }
}

struct Layout {
  size_t total;
  int h_rows, stages;
};

static Layout layout_for(const moe_layer_desc& d, int grid, bool noise, int smem_max) {
  Layout l{};
  size_t fixed = ((sizeof(Smem) + 127) & ~size_t(127)) + ((sizeof(Jobs) + 127) & ~size_t(127));
  l.h_rows = (d.H + grid - 1) / grid;
  fixed += (size_t)l.h_rows * d.T * d.K * sizeof(float) + (size_t)l.h_rows * d.T * sizeof(float);
  fixed += (size_t)d.E * sizeof(float) + (noise ? (size_t)d.T * d.E * sizeof(float) : 0);
  fixed = (fixed + 127) & ~size_t(127);
  const size_t stage =
      std::max((size_t)d.T * d.H, (size_t)d.T * d.K * d.D + (size_t)d.T * d.Ds) * 2;
  // the deepest per-warp pipeline that fits beside the staged activations
  l.stages = 0;
  for (int st : {3, 2}) {
    if (fixed + ring_bytes(st) + stage <= (size_t)smem_max) {
      l.stages = st;
      break;
    }
  }
  l.total = fixed + ring_bytes(l.stages ? l.stages : 4) + stage;
  return l;
}

}  // namespace dec

// Per-device launch limits of the decode kernel (SM count, shared memory).
static bool decode_device_limits(int* sms, int* smem_max) {
  static std::atomic<int> cache_sms[64], cache_smem[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  int n = cache_sms[dev].load(std::memory_order_relaxed);
  int m = cache_smem[dev].load(std::memory_order_relaxed);
  if (!n || !m) {
    int v = 0, w = 0, coop = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&w, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
      return false;
    n = v;
    m = w;
    if (v < dec::kMinCtas) return false;
    cache_sms[dev].store(n, std::memory_order_relaxed);
    cache_smem[dev].store(m, std::memory_order_relaxed);
  }
  *sms = n;
  *smem_max = m;
  return true;
}

bool decode_eligible(const moe_layer_desc& d) {
  if (d.dtype != MOE_BF16 || d.T < 1 || d.T > kDecodeMaxT) return false;
  if (d.H > dec::kMaxRowLen || d.D > dec::kMaxRowLen || d.Ds > dec::kMaxRowLen) return false;
  int sms = 0, smem_max = 0;
  if (!decode_device_limits(&sms, &smem_max)) return false;
  // (sized with the noise input, so the answer does not depend on it)
  return dec::layout_for(d, sms, /*noise=*/true, smem_max).stages > 0;
}

cudaError_t launch_decode_forward(const moe_layer_desc& d, const DecodeBuffers& b,
                                  cudaStream_t st) {
  using namespace dec;
  int sms = 0, smem_max = 0;
  if (!decode_device_limits(&sms, &smem_max)) return cudaErrorNotSupported;
  const Layout l = layout_for(d, sms, b.noise != nullptr, smem_max);
  if (l.stages == 0) return cudaErrorInvalidValue;
  Params p{};
  p.x = static_cast<const __nv_bfloat16*>(b.x);
  p.wr = static_cast<const __nv_bfloat16*>(b.w_router);
  p.bias = b.bias;
  p.noise = b.noise;
  p.w1 = static_cast<const __nv_bfloat16*>(b.w1);
  p.w2 = static_cast<const __nv_bfloat16*>(b.w2);
  p.ws1 = static_cast<const __nv_bfloat16*>(b.ws1);
  p.ws2 = static_cast<const __nv_bfloat16*>(b.ws2);
  p.y = static_cast<__nv_bfloat16*>(b.y);
  p.logits = b.logits;
  p.idx = b.idx;
  p.tw = b.tw;
  p.counts = b.counts;
  p.offsets = b.offsets;
  p.perm = b.perm;
  p.inv = b.inv;
  p.hm = static_cast<__nv_bfloat16*>(b.hm);
  p.hs = static_cast<__nv_bfloat16*>(b.hs);
  p.hdr = b.hdr;
  p.T = d.T;
  p.H = d.H;
  p.E = d.E;
  p.K = d.K;
  p.D = d.D;
  p.Ds = d.Ds;
  p.h_rows = l.h_rows;
  // instantiations by activation rows (1, 2) and pipeline depth (3, 2)
  void (*const kernels[2][2])(const Params) = {
      {decode_forward<1, 3>, decode_forward<1, 2>},
      {decode_forward<2, 3>, decode_forward<2, 2>}};
  static_assert(kDecodeMaxT == 2, "one instantiation per token count");
  const int which = d.T == 1 ? 0 : 1;
  const int deep = l.stages == 3 ? 0 : 1;
  void (*kern)(const Params) = kernels[which][deep];
  static std::atomic<bool> attr_set[64][2][2];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev][which][deep].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, (size_t)smem_max);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) attr_set[dev][which][deep].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = l.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace moe
