// C ABI of libmoe: argument checks, workspace layout and the launch sequence.
// Every compute step runs in this library's kernels; nothing here computes
// on the host except sizes.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "dispatch.cuh"
#include "kernels.cuh"

namespace moe {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

size_t dtype_size(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Reduction splits for the tensor-core GEMMs. A decode-sized step has too
// few (128-row x all-K) tiles to give every one of the 148 SMs an equal share
// of the weight stream; splitting the reduction multiplies the tiles. The
// choice depends on the shape only (so the workspace size does too).
static int split_count(long long tiles, int kb, int want_tiles, int min_kb) {
  if (tiles <= 0 || tiles >= want_tiles) return 1;
  int sp = (int)((want_tiles + tiles - 1) / tiles);
  sp = std::min(sp, std::max(1, kb / min_kb));
  sp = std::max(1, std::min(sp, kMaxSplits));
  const int per = (kb + sp - 1) / sp;
  return (kb + per - 1) / per;
}

// Splits that leave no empty split: kb blocks in ceil(kb / ceil(kb / sp)).
static int normalise_splits(int kb, int sp) {
  const int per = (kb + sp - 1) / sp;
  return (kb + per - 1) / per;
}

// Largest share of one persistent unit, in reduction blocks, when ns tiles
// of cost cs and then nr tiles of cost cr are dealt round-robin to `units`
// units: the order of the device tile list when every touched expert has one
// row tile (the shared expert's tiles come first).
static double deal_makespan(long long ns, double cs, long long nr, double cr, int units) {
  double worst = 0.0;
  const long long n = ns + nr;
  for (int u = 0; u < units && u < n; ++u) {
    const long long k_all = (n - u + units - 1) / units;
    const long long k_sh = ns > u ? (ns - u + units - 1) / units : 0;
    worst = std::max(worst, (double)k_sh * cs + (double)(k_all - k_sh) * cr);
  }
  return worst;
}

// Splits (routed, shared) of one weight-streaming GEMM launch with ns shared
// tiles of kbs reduction blocks and nr_lo .. nr_hi routed tiles of kbr blocks
// (the routed count depends on how many experts the batch touches, which
// the shape alone does not fix). Each candidate is scored by its per-unit
// share relative to a perfect spread, averaged over the low, middle and high
// routed counts; each tile also costs tile_cost blocks of fixed work, and
// near-ties go to fewer splits. At most max_r / max_s splits and at least
// kMinKb blocks per split.
static void pick_splits(long long nr_lo, long long nr_hi, int kbr, long long ns, int kbs,
                        int units, int max_r, int max_s, double tile_cost, int* sr_out,
                        int* ss_out) {
  constexpr int kMinKb = 4;
  static const int kCand[] = {1, 2, 3, 4, 5, 6, 8, 10, 12, 16};
  const long long nr_at[3] = {nr_lo, (nr_lo + nr_hi) / 2, nr_hi};
  double best = 1e300;
  int br = 1, bs = 1;
  for (int cr : kCand) {
    if (cr > 1 && (cr > max_r || kbr / cr < kMinKb)) break;
    const int sr = normalise_splits(kbr, cr);
    for (int cs : kCand) {
      if (cs > 1 && (ns == 0 || cs > max_s || kbs / cs < kMinKb)) break;
      const int ss = normalise_splits(kbs > 0 ? kbs : 1, cs);
      const double per_r = (double)((kbr + sr - 1) / sr);
      const double per_s = kbs ? (double)((kbs + ss - 1) / ss) : 0.0;
      double score = 0.0;
      for (long long nr : nr_at) {
        const double ideal =
            std::max(1.0, ((double)ns * kbs + (double)nr * kbr) / (double)units);
        score += deal_makespan(ns * ss, per_s + tile_cost, nr * sr, per_r + tile_cost, units) /
                 ideal;
      }
      score *= 1.0 + 0.01 * (sr + ss - 2);
      if (score < best * 0.999) {
        best = score;
        br = sr;
        bs = ss;
      }
    }
  }
  *sr_out = br;
  *ss_out = bs;
}

static Splits compute_splits(const moe_layer_desc& d) {
  Splits s{1, 1, 1, 1, 1, 0};
  if (d.dtype != MOE_BF16 || d.T == 0) return s;
  const long long T = d.T, TK = (long long)d.T * d.K;
  // CTA pairs (256 weight rows per tile) when the touched experts average
  // at least 64 rows each: then the tiles are wide enough in N for the
  // halved per-SM operand traffic to matter.
  const long long touched = std::min<long long>(d.E, TK);
  s.pair = (d.D % 256 == 0 && d.H % 256 == 0 && d.Ds % 256 == 0 && TK >= 64 * touched) ? 1 : 0;
  const long long row_tiles = (T + kTcRows - 1) / kTcRows;
  s.router = std::min(16, split_count(row_tiles * ((d.E + 127) / 128), d.H / 64, 148, 2));
  s.router = normalise_splits(d.H / 64, s.router);   // no empty split after the cap
  // Routed row tiles: each touched expert has at least one. A batch touches
  // between K and min(E, T*K) experts (all of them once it holds several
  // copies per expert); the model averages over that range.
  const long long r_rows = std::max(touched, (TK + kTcRows - 1) / kTcRows);
  const long long r_lo = (TK >= 8LL * d.E) ? r_rows
                         : std::max<long long>(d.K + (touched - d.K) / 2,
                                               (TK + kTcRows - 1) / kTcRows);
  if (!s.pair) {
    // Weight-streaming regime: balance both expert GEMMs over the SMs. The
    // first GEMM's splits are added up by the last split of each tile, one
    // round of loads per few rows, so they are used for short tiles only
    // (at most kFixupRows rows per routed expert on average, or per shared
    // tile) and their fixed cost per tile is higher.
    constexpr int kFixupRows = 16;
    const int max_r1 = (TK <= kFixupRows * touched) ? 16 : 1;
    const int max_s1 = (T <= kFixupRows) ? 16 : 1;
    pick_splits(r_lo * (d.D / 128), r_rows * (d.D / 128), d.H / 64,
                d.Ds ? row_tiles * (d.Ds / 128) : 0, d.H / 64, 148, max_r1, max_s1, 6.0,
                &s.gemm1_routed, &s.gemm1_shared);
    pick_splits(r_lo * (d.H / 128), r_rows * (d.H / 128), d.D / 64,
                d.Ds ? row_tiles * (d.H / 128) : 0, d.Ds ? d.Ds / 64 : 0, 148, 16, 16, 2.0,
                &s.gemm2_routed, &s.gemm2_shared);
    return s;
  }
  // CTA pairs: the second GEMM's splits from the same model over the 74
  // pairs (its partials are added by the combine); the first layer stays
  // unsplit on pairs.
  const int mt2 = d.H / 256;
  pick_splits(r_lo * mt2, r_rows * mt2, d.D / 64, d.Ds ? row_tiles * mt2 : 0,
              d.Ds ? d.Ds / 64 : 0, 74, 16, 16, 2.0, &s.gemm2_routed, &s.gemm2_shared);
  return s;
}

// The choice is a pure function of the descriptor; a small cache keeps its
// search off the per-call host path.
Splits choose_splits(const moe_layer_desc& d) {
  struct Entry {
    moe_layer_desc d;
    Splits s;
    bool used;
  };
  static std::mutex mu;
  static Entry cache[16] = {};
  static int next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
      if (e.used && std::memcmp(&e.d, &d, sizeof(d)) == 0) return e.s;
  }
  const Splits s = compute_splits(d);
  std::lock_guard<std::mutex> lock(mu);
  cache[next] = Entry{d, s, true};
  next = (next + 1) % 16;
  return s;
}

WsLayout workspace_layout(const moe_layer_desc& d) {
  WsLayout L{};
  const size_t T = d.T, K = d.K, E = d.E, H = d.H, D = d.D, Ds = d.Ds;
  const size_t TK = T * K;
  const size_t es = dtype_size(d.dtype);
  L.n_chunks = (int)std::max<size_t>(1, (TK + kChunk - 1) / kChunk);
  const size_t rows_bound = std::min(E, TK);          // groups that can hold rows
  L.max_tiles_simt = (int)((TK + kSimtRows - 1) / kSimtRows + rows_bound +
                           (Ds ? (T + kSimtRows - 1) / kSimtRows : 0));
  const size_t rt_routed = (TK + kTcRows - 1) / kTcRows + rows_bound;
  const size_t rt_shared = Ds ? (T + kTcRows - 1) / kTcRows : 0;
  L.sp = choose_splits(d);
  L.max_tiles_tc1 =
      (int)((rt_routed * L.sp.gemm1_routed * (D / 128) + rt_shared * L.sp.gemm1_shared * (Ds / 128)));
  L.max_tiles_tc2 =
      (int)((rt_routed * L.sp.gemm2_routed + rt_shared * L.sp.gemm2_shared) * (H / 128));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.hdr = take(sizeof(WsHeader));
  L.hist = take(sizeof(int32_t) * L.n_chunks * E);
  L.base = take(sizeof(int32_t) * L.n_chunks * E);
  L.tiles_simt = take(sizeof(Tile) * std::max(1, L.max_tiles_simt));
  L.tiles_tc1 = take(sizeof(Tile) * std::max(1, L.max_tiles_tc1));
  L.tiles_tc2 = take(sizeof(Tile) * std::max(1, L.max_tiles_tc2));
  L.idx = take(sizeof(int32_t) * TK);
  L.w = take(sizeof(float) * TK);
  L.counts = take(sizeof(int32_t) * E);
  L.offsets = take(sizeof(int32_t) * (E + 1));
  L.perm = take(sizeof(int32_t) * TK);
  L.inv = take(sizeof(int32_t) * TK);
  L.logits = take(sizeof(float) * T * E);
  L.logits_part = take(d.dtype == MOE_BF16 ? sizeof(float) * T * E * L.sp.router : 0);
  L.xp = take(d.dtype == MOE_BF16 ? es * TK * H : 0);
  L.hm = take(es * TK * D);
  L.hs = take(es * T * Ds);
  // fp32 partial outputs of the first GEMM when its reduction is split
  L.p1r = take(L.sp.gemm1_routed > 1 ? sizeof(float) * TK * D * L.sp.gemm1_routed : 0);
  L.p1s = take(Ds && L.sp.gemm1_shared > 1 ? sizeof(float) * T * Ds * L.sp.gemm1_shared : 0);
  // expert outputs are fp32, one copy per reduction split of the second GEMM
  L.yr = take(sizeof(float) * TK * H * L.sp.gemm2_routed);
  L.ys = take(sizeof(float) * T * H * (Ds ? L.sp.gemm2_shared : 0));
  L.stats = take(sizeof(moe_stats) + E);
  L.total = o;
  return L;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static moe_status check_desc(const moe_layer_desc* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->H < 1 || d->E < 1 || d->K < 1 || d->D < 1 || d->Ds < 0)
    return MOE_ERR_INVALID_ARG;
  if (d->dtype != MOE_F32 && d->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (d->cf_num < 0 || d->cf_den < 1) return MOE_ERR_INVALID_ARG;
  if (d->K > d->E) return MOE_ERR_INVALID_ARG;
  if (d->K > kMaxK || d->E > kMaxE) return MOE_ERR_UNSUPPORTED;
  const int q = (d->dtype == MOE_BF16) ? 128 : 4;
  if (d->H % q || d->D % q || d->Ds % q) return MOE_ERR_UNSUPPORTED;
  if ((long long)d->T * d->K > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

static moe_status check_ws(const moe_layer_desc& d, const void* ws, size_t ws_bytes) {
  if (!ws || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (ws_bytes < workspace_layout(d).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// All listed pointers must be non-null and 16-byte aligned.
static moe_status check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

static int num_sms() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n = v > 0 ? v : 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

#define MOE_TRY(expr)                 \
  do {                                \
    moe_status _s = (expr);           \
    if (_s != MOE_OK) return _s;      \
  } while (0)

// Grouped FFN body shared by moe_grouped_ffn and moe_layer_forward. The
// tile lists must already be in the workspace.
static moe_status run_grouped_ffn(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                  const void* x, const int32_t* perm, const void* w1,
                                  const void* w2, const void* ws1, const void* ws2, void* y_rows,
                                  void* y_shared, cudaStream_t st, bool split,
                                  cudaEvent_t const* ev_after_gemm1 = nullptr,
                                  bool with_shared = true) {
  if (d.T == 0) return MOE_OK;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
  void* hm = ws + L.hm;
  void* hs = ws + L.hs;
  const bool shared = d.Ds > 0 && with_shared;
  if (d.dtype == MOE_BF16) {
    // Tensor-core path: the dispatched activation rows are in ws + L.xp.
    const uint64_t TK = (uint64_t)d.T * d.K;
    auto problem = [](const void* act, uint64_t act_rows, const void* w, uint64_t w_rows,
                      int m_rows, int kd, void* out, int ld, bool out_f32, int splits,
                      long long split_stride) {
      TcProblem p{};
      p.act = act;
      p.act_rows = act_rows;
      p.w = w;
      p.w_rows = w_rows;
      p.m_rows = m_rows;
      p.kd = kd;
      p.out = out;
      p.ld = ld;
      p.out_f32 = out_f32;
      p.splits = splits;
      p.split_stride = split_stride;
      p.m_valid = m_rows;
      return p;
    };
    const int sp_r = split ? L.sp.gemm2_routed : 1, sp_s = split ? L.sp.gemm2_shared : 1;
    const int sp1_r = split ? L.sp.gemm1_routed : 1, sp1_s = split ? L.sp.gemm1_shared : 1;
    // A split first layer writes fp32 partials; the last split of each tile
    // to finish adds them and writes the GeLU output.
    auto split_first_layer = [](TcProblem& p, void* partials, int splits, long long rows) {
      p.fix_out = p.out;
      p.fix_ld = p.ld;
      p.out = partials;
      p.out_f32 = true;
      p.splits = splits;
      p.split_stride = rows * p.ld;
    };
    TcProblem r1 = problem(ws + L.xp, TK, w1, (uint64_t)d.E * d.D, d.D, d.H, hm, d.D, false, 1, 0);
    if (sp1_r > 1) split_first_layer(r1, ws + L.p1r, sp1_r, (long long)TK);
    TcProblem r2 = problem(hm, TK, w2, (uint64_t)d.E * d.H, d.H, d.D, y_rows, d.H, true, sp_r,
                           (long long)TK * d.H);
    TcProblem s1{}, s2{};
    if (shared) {
      s1 = problem(x, (uint64_t)d.T, ws1, (uint64_t)d.Ds, d.Ds, d.H, hs, d.Ds, false, 1, 0);
      if (sp1_s > 1) split_first_layer(s1, ws + L.p1s, sp1_s, (long long)d.T);
      s2 = problem(hs, (uint64_t)d.T, ws2, (uint64_t)d.H, d.H, d.Ds, y_shared, d.H, true, sp_s,
                   (long long)d.T * d.H);
    }
    // the tile lists of a split (layer-forward) dispatch follow L.sp.pair
    const bool pair = split && L.sp.pair;
    MOE_CUDA_TRY(launch_grouped_gemm_tc(r1, s1, d.E, true,
                                        reinterpret_cast<const Tile*>(ws + L.tiles_tc1),
                                        &hdr->n_tiles[1], nullptr, pair, &hdr->status, num_sms(),
                                        st));
    if (ev_after_gemm1) MOE_CUDA_TRY(cudaEventRecord(*ev_after_gemm1, st));
    MOE_CUDA_TRY(launch_grouped_gemm_tc(r2, s2, d.E, false,
                                        reinterpret_cast<const Tile*>(ws + L.tiles_tc2),
                                        &hdr->n_tiles[2], nullptr, pair, &hdr->status, num_sms(),
                                        st));
    return MOE_OK;
  }
  SimtProblem r1{x, perm, d.K, w1, (size_t)d.D * d.H, hm, d.H, d.D};
  SimtProblem s1{x, nullptr, 1, ws1, 0, hs, d.H, d.Ds};
  SimtProblem r2{hm, nullptr, 1, w2, (size_t)d.H * d.D, y_rows, d.D, d.H};
  SimtProblem s2{hs, nullptr, 1, ws2, 0, y_shared, d.Ds, d.H};
  const Tile* tiles = reinterpret_cast<const Tile*>(ws + L.tiles_simt);
  MOE_CUDA_TRY(launch_grouped_gemm_simt(d.dtype, true, r1, s1, d.E, tiles, &hdr->n_tiles[0],
                                        L.max_tiles_simt, std::max(d.D, shared ? d.Ds : 0), st));
  if (ev_after_gemm1) MOE_CUDA_TRY(cudaEventRecord(*ev_after_gemm1, st));
  MOE_CUDA_TRY(launch_grouped_gemm_simt(d.dtype, false, r2, s2, d.E, tiles, &hdr->n_tiles[0],
                                        L.max_tiles_simt, d.H, st));
  return MOE_OK;
}

// The shared expert does not depend on the routing, so a bf16 layer runs its
// two GEMMs on a second stream of the library (one per device, created on
// the first call) while the router, the dispatch and the routed experts run
// on the caller's stream; the combine waits for both. The fork and join are
// event record / wait pairs, so the whole forward stays capturable in a CUDA
// graph once the first (eager) call has created the stream.
constexpr int kSideStreamMinT = 8;

struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;   // serialises the use of the two events
};

static SideStream* side_stream() {
  static SideStream side[64];
  static std::mutex init_mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = side[dev];
  std::lock_guard<std::mutex> lock(init_mu);
  if (!ss.stream) {
    cudaStream_t s = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&a, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&b, cudaEventDisableTiming) != cudaSuccess) {
      if (a) cudaEventDestroy(a);
      cudaStreamDestroy(s);
      return nullptr;
    }
    ss.fork = a;
    ss.join = b;
    ss.stream = s;
  }
  return &ss;
}

// Shared expert of a bf16 layer as two dense launches on `st`: Hs = GeLU(x
// Ws1^T) (bf16) and S = Hs Ws2^T (fp32, L.sp.gemm2_shared partials). At most
// half of the SMs, so the caller's stream keeps the rest.
static moe_status run_shared_ffn(const moe_layer_desc& d, const WsLayout& L, char* ws,
                                 const void* x, const void* ws1, const void* ws2, cudaStream_t st) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.hdr);
  const bool pair = L.sp.pair != 0;
  const int mt = pair ? 256 : 128;
  const int row_tiles = (d.T + kTcRows - 1) / kTcRows;
  const int sms = num_sms();
  TcProblem s1{};
  s1.act = x;
  s1.act_rows = (uint64_t)d.T;
  s1.w = ws1;
  s1.w_rows = (uint64_t)d.Ds;
  s1.m_rows = d.Ds;
  s1.kd = d.H;
  s1.out = ws + L.hs;
  s1.ld = d.Ds;
  s1.splits = 1;
  s1.m_valid = d.Ds;
  DenseTiling t1{row_tiles * (d.Ds / mt), d.T, d.Ds / mt};
  MOE_CUDA_TRY(launch_grouped_gemm_tc(s1, TcProblem{}, 1, true, nullptr, nullptr, &t1, pair,
                                      &hdr->status, sms, st, sms / 2));
  TcProblem s2{};
  s2.act = ws + L.hs;
  s2.act_rows = (uint64_t)d.T;
  s2.w = ws2;
  s2.w_rows = (uint64_t)d.H;
  s2.m_rows = d.H;
  s2.kd = d.Ds;
  s2.out = ws + L.ys;
  s2.ld = d.H;
  s2.out_f32 = true;
  s2.splits = L.sp.gemm2_shared;
  s2.split_stride = (long long)d.T * d.H;
  s2.m_valid = d.H;
  DenseTiling t2{row_tiles * (d.H / mt) * L.sp.gemm2_shared, d.T, d.H / mt};
  MOE_CUDA_TRY(launch_grouped_gemm_tc(s2, TcProblem{}, 1, false, nullptr, nullptr, &t2, pair,
                                      &hdr->status, sms, st, sms / 2));
  return MOE_OK;
}

// Router: gate logits then selection. bf16 layers run the gate GEMM on the
// tensor cores (partial sums per reduction split, added by the selection
// kernel); fp32 layers on CUDA cores.
static moe_status run_router(const moe_layer_desc& d, const WsLayout& L, char* ws,
                             const void* x, const void* wr, const float* bias, int32_t* idx,
                             float* tw, float* logits_out, cudaStream_t st,
                             const float* noise = nullptr) {
  if (d.T == 0) return MOE_OK;
  if (d.dtype == MOE_BF16) {
    float* parts = reinterpret_cast<float*>(ws + L.logits_part);
    MOE_CUDA_TRY(launch_gate_logits_tc(d, L, ws, x, wr, parts, num_sms(), st));
    MOE_CUDA_TRY(launch_topk_select(d, parts, L.sp.router, (size_t)d.T * d.E, bias, noise, idx,
                                    tw, logits_out, st));
  } else {
    float* logits = logits_out ? logits_out : reinterpret_cast<float*>(ws + L.logits);
    MOE_CUDA_TRY(launch_gate_logits(d, x, wr, logits, st));
    MOE_CUDA_TRY(launch_topk_select(d, logits, 1, 0, bias, noise, idx, tw, nullptr, st));
  }
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_layer_desc* desc) {
  if (check_desc(desc) != MOE_OK) return 0;
  return workspace_layout(*desc).total;
}

moe_status moe_router_topk(const moe_layer_desc* desc, const void* x, const void* w_router,
                           const float* bias, float* logits_or_null, int32_t* topk_idx,
                           float* topk_w, void* ws, size_t ws_bytes, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  if (d.T == 0) return MOE_OK;
  MOE_TRY(check_ptrs({x, w_router, topk_idx, topk_w}));
  if (bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if (logits_or_null && !aligned16(logits_or_null)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = workspace_layout(d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return run_router(d, L, static_cast<char*>(ws), x, w_router, bias, topk_idx, topk_w,
                    logits_or_null, st);
}

static moe_status topk_from_logits_impl(const moe_layer_desc* desc, const float* logits,
                                        const float* bias, const float* noise, int32_t* topk_idx,
                                        float* topk_w, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  if (d.T == 0) return MOE_OK;
  MOE_TRY(check_ptrs({logits, topk_idx, topk_w}));
  if (bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(launch_topk_select(d, logits, 1, 0, bias, noise, topk_idx, topk_w, nullptr,
                                  static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_topk_from_logits(const moe_layer_desc* desc, const float* logits,
                                const float* bias, int32_t* topk_idx, float* topk_w,
                                moe_stream stream) {
  return topk_from_logits_impl(desc, logits, bias, nullptr, topk_idx, topk_w, stream);
}

moe_status moe_topk_from_logits_noisy(const moe_layer_desc* desc, const float* logits,
                                      const float* bias, const float* gumbel_noise,
                                      int32_t* topk_idx, float* topk_w, moe_stream stream) {
  if (!gumbel_noise || !aligned16(gumbel_noise)) return MOE_ERR_INVALID_ARG;
  return topk_from_logits_impl(desc, logits, bias, gumbel_noise, topk_idx, topk_w, stream);
}

moe_status moe_dispatch(const moe_layer_desc* desc, const int32_t* topk_idx, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, void* ws,
                        size_t ws_bytes, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  MOE_TRY(check_ptrs({counts, offsets}));
  if (d.T > 0) MOE_TRY(check_ptrs({topk_idx, perm, inv}));
  const WsLayout L = workspace_layout(d);
  MOE_CUDA_TRY(launch_dispatch(d, L, static_cast<char*>(ws), topk_idx, counts, offsets, perm,
                               inv, false, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_grouped_ffn(const moe_layer_desc* desc, const void* x, const int32_t* perm,
                           const int32_t* offsets, const void* w1, const void* w2,
                           const void* ws1, const void* ws2, void* y_rows, void* y_shared,
                           void* ws, size_t ws_bytes, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  if (d.T == 0) return MOE_OK;
  MOE_TRY(check_ptrs({x, perm, offsets, w1, w2, y_rows}));
  if (d.Ds > 0) MOE_TRY(check_ptrs({ws1, ws2, y_shared}));
  const WsLayout L = workspace_layout(d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const bool tc = d.dtype == MOE_BF16;
  MOE_CUDA_TRY(launch_tiles_from_offsets(d, L, w, offsets, tc, st));
  if (tc) MOE_CUDA_TRY(launch_gather_rows(d, x, perm, w + L.xp, num_sms(), st));
  return run_grouped_ffn(d, L, w, x, perm, w1, w2, ws1, ws2, y_rows, y_shared, st,
                         /*split=*/false);
}

moe_status moe_combine(const moe_layer_desc* desc, const void* y_rows, const float* topk_w,
                       const int32_t* inv, const void* y_shared_or_null, void* y,
                       moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  if (d.T == 0) return MOE_OK;
  MOE_TRY(check_ptrs({y_rows, topk_w, inv, y}));
  if (y_shared_or_null && !aligned16(y_shared_or_null)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(launch_combine(d, y_rows, topk_w, inv, y_shared_or_null, y,
                              static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

static moe_status layer_forward_impl(const moe_layer_desc* desc, const moe_layer_weights* weights,
                                     const void* x, void* y, const moe_routing* routing_or_null,
                                     void* ws, size_t ws_bytes, cudaStream_t st,
                                     cudaEvent_t const* ev, int n_ev,
                                     const float* noise = nullptr) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  if (!weights) return MOE_ERR_INVALID_ARG;
  if (ev && n_ev < kForwardEvents) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  const moe_layer_weights& W = *weights;
  MOE_TRY(check_ptrs({x, y, W.w_router, W.w1, W.w2}));
  if (d.Ds > 0) MOE_TRY(check_ptrs({W.ws1, W.ws2}));
  if (W.expert_bias && !aligned16(W.expert_bias)) return MOE_ERR_INVALID_ARG;
  moe_routing R{};
  if (routing_or_null) R = *routing_or_null;
  for (const void* p : {(const void*)R.topk_idx, (const void*)R.topk_w, (const void*)R.counts,
                        (const void*)R.offsets, (const void*)R.perm, (const void*)R.inv,
                        (const void*)R.logits})
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = workspace_layout(d);
  char* w = static_cast<char*>(ws);
  int32_t* idx = R.topk_idx ? R.topk_idx : reinterpret_cast<int32_t*>(w + L.idx);
  float* tw = R.topk_w ? R.topk_w : reinterpret_cast<float*>(w + L.w);
  int32_t* counts = R.counts ? R.counts : reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* offsets = R.offsets ? R.offsets : reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* perm = R.perm ? R.perm : reinterpret_cast<int32_t*>(w + L.perm);
  int32_t* inv = R.inv ? R.inv : reinterpret_cast<int32_t*>(w + L.inv);
  void* yr = w + L.yr;
  void* ys = d.Ds > 0 ? static_cast<void*>(w + L.ys) : nullptr;
  auto mark = [&](int i) -> cudaError_t { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };

  const bool tc = d.dtype == MOE_BF16;
  // A handful of bf16 tokens: the whole layer in one cooperative launch
  // (router, selection, dispatch, both expert layers, combine).
  if (tc && decode_eligible(d)) {
    DecodeBuffers b{};
    b.x = x;
    b.w_router = W.w_router;
    b.w1 = W.w1;
    b.w2 = W.w2;
    b.ws1 = W.ws1;
    b.ws2 = W.ws2;
    b.bias = W.expert_bias;
    b.noise = noise;
    b.y = y;
    b.logits = R.logits ? R.logits : reinterpret_cast<float*>(w + L.logits);
    b.idx = idx;
    b.tw = tw;
    b.counts = counts;
    b.offsets = offsets;
    b.perm = perm;
    b.inv = inv;
    b.hm = w + L.hm;
    b.hs = w + L.hs;
    b.hdr = reinterpret_cast<WsHeader*>(w + L.hdr);
    MOE_CUDA_TRY(mark(0));
    MOE_CUDA_TRY(launch_decode_forward(d, b, st));
    for (int i = 1; i < kForwardEvents; ++i) MOE_CUDA_TRY(mark(i));
    return MOE_OK;
  }
  // bf16 decode batches with a shared expert: its GEMMs go to the side stream
  // first. Measured on B200: 2-6% faster from T = 16 on; slower at T = 1
  // (the fork and join cost more than the overlap gains) and on CTA-pair
  // (prefill) shapes, where the shared expert's persistent grid takes SMs
  // the router and dispatch need.
  SideStream* side = nullptr;
  std::unique_lock<std::mutex> side_lock;
  // Once the side stream has forked from `st`, every return joins it back:
  // an error after the fork must not leave the shared expert's launches
  // running unjoined (that would also invalidate a graph capture).
  struct SideJoin {
    SideStream* side = nullptr;
    cudaStream_t st = nullptr;
    bool recorded = false;
    ~SideJoin() {
      if (!side) return;
      if (!recorded) cudaEventRecord(side->join, side->stream);
      cudaStreamWaitEvent(st, side->join, 0);
    }
  } join_guard;
  if (tc && d.Ds > 0 && !L.sp.pair && d.T >= kSideStreamMinT) {
    side = side_stream();
    if (!side) return MOE_ERR_CUDA;
    side_lock = std::unique_lock<std::mutex>(side->mu);
    MOE_CUDA_TRY(cudaEventRecord(side->fork, st));
    MOE_CUDA_TRY(cudaStreamWaitEvent(side->stream, side->fork, 0));
    join_guard.side = side;
    join_guard.st = st;
    MOE_TRY(run_shared_ffn(d, L, w, x, W.ws1, W.ws2, side->stream));
    MOE_CUDA_TRY(cudaEventRecord(side->join, side->stream));
    join_guard.recorded = true;
  }
  MOE_CUDA_TRY(mark(0));
  MOE_TRY(run_router(d, L, w, x, W.w_router, W.expert_bias, idx, tw, R.logits, st, noise));
  MOE_CUDA_TRY(mark(1));
  if (tc)
    MOE_CUDA_TRY(launch_dispatch_gather(d, L, w, idx, counts, offsets, perm, inv, st,
                                        /*shared_tiles=*/side == nullptr, x, w + L.xp,
                                        num_sms()));
  else
    MOE_CUDA_TRY(launch_dispatch(d, L, w, idx, counts, offsets, perm, inv, false, st,
                                 /*shared_tiles=*/side == nullptr));
  MOE_CUDA_TRY(mark(2));
  MOE_TRY(run_grouped_ffn(d, L, w, x, perm, W.w1, W.w2, W.ws1, W.ws2, yr, ys, st,
                          /*split=*/true, ev ? ev + 3 : nullptr, /*with_shared=*/side == nullptr));
  MOE_CUDA_TRY(mark(4));
  if (side) {
    join_guard.side = nullptr;   // joined here
    MOE_CUDA_TRY(cudaStreamWaitEvent(st, side->join, 0));
  }
  MOE_CUDA_TRY(launch_combine(d, yr, tw, inv, ys, y, st, L.sp.gemm2_routed, L.sp.gemm2_shared));
  MOE_CUDA_TRY(mark(5));
  return MOE_OK;
}

moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* weights,
                             const void* x, void* y, const moe_routing* routing_or_null,
                             void* ws, size_t ws_bytes, moe_stream stream) {
  return layer_forward_impl(desc, weights, x, y, routing_or_null, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream), nullptr, 0);
}

moe_status moe_layer_forward_noisy(const moe_layer_desc* desc, const moe_layer_weights* weights,
                                   const void* x, const float* gumbel_noise, void* y,
                                   const moe_routing* routing_or_null, void* ws, size_t ws_bytes,
                                   moe_stream stream) {
  if (!gumbel_noise || !aligned16(gumbel_noise)) return MOE_ERR_INVALID_ARG;
  return layer_forward_impl(desc, weights, x, y, routing_or_null, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream), nullptr, 0, gumbel_noise);
}

moe_status moe_layer_forward_profiled(const moe_layer_desc* desc,
                                      const moe_layer_weights* weights, const void* x, void* y,
                                      const moe_routing* routing_or_null, void* ws,
                                      size_t ws_bytes, moe_stream stream,
                                      void* const* stage_events, int n_events) {
  if (!stage_events) return MOE_ERR_INVALID_ARG;
  return layer_forward_impl(desc, weights, x, y, routing_or_null, ws, ws_bytes,
                            static_cast<cudaStream_t>(stream),
                            reinterpret_cast<cudaEvent_t const*>(stage_events), n_events);
}

moe_status moe_expert_gemms(const moe_layer_desc* desc, const moe_layer_weights* weights,
                            const void* x, void* ws, size_t ws_bytes, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  if (!weights) return MOE_ERR_INVALID_ARG;
  if (d.T == 0) return MOE_OK;
  if (d.dtype != MOE_BF16 || decode_eligible(d)) return MOE_ERR_UNSUPPORTED;
  const moe_layer_weights& W = *weights;
  MOE_TRY(check_ptrs({x, W.w1, W.w2}));
  if (d.Ds > 0) MOE_TRY(check_ptrs({W.ws1, W.ws2}));
  const WsLayout L = workspace_layout(d);
  char* w = static_cast<char*>(ws);
  // the same choice as moe_layer_forward: a shared expert on the side stream
  // is not part of the caller-stream launches
  const bool side = d.Ds > 0 && !L.sp.pair && d.T >= kSideStreamMinT;
  void* ys = d.Ds > 0 ? static_cast<void*>(w + L.ys) : nullptr;
  return run_grouped_ffn(d, L, w, x, reinterpret_cast<const int32_t*>(w + L.perm), W.w1, W.w2,
                         W.ws1, W.ws2, w + L.yr, ys, static_cast<cudaStream_t>(stream),
                         /*split=*/true, nullptr, /*with_shared=*/!side);
}

moe_status moe_expert_stats(const moe_layer_desc* desc, const int32_t* counts,
                            uint8_t* straggler_mask_or_null, moe_stats* out_host, void* ws,
                            size_t ws_bytes, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc& d = *desc;
  MOE_TRY(check_ws(d, ws, ws_bytes));
  if (!counts || !out_host) return MOE_ERR_INVALID_ARG;
  const WsLayout L = workspace_layout(d);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe_stats* dev = reinterpret_cast<moe_stats*>(static_cast<char*>(ws) + L.stats);
  MOE_CUDA_TRY(launch_expert_stats(d, counts, straggler_mask_or_null, dev, st));
  MOE_CUDA_TRY(cudaMemcpyAsync(out_host, dev, sizeof(moe_stats), cudaMemcpyDeviceToHost, st));
  MOE_CUDA_TRY(cudaStreamSynchronize(st));
  return MOE_OK;
}

moe_status moe_bias_update(const moe_layer_desc* desc, const int32_t* counts, float* bias,
                           float gamma, moe_stream stream) {
  MOE_TRY(check_desc(desc));
  if (!counts || !bias) return MOE_ERR_INVALID_ARG;
  if (!(gamma >= 0.f) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA_TRY(launch_bias_update(*desc, counts, bias, gamma, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_check_status(void* ws, size_t ws_bytes, moe_stream stream) {
  if (!ws || ws_bytes < sizeof(WsHeader)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t status = 0;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  MOE_CUDA_TRY(cudaMemcpyAsync(&status, &hdr->status, sizeof(status), cudaMemcpyDeviceToHost, st));
  MOE_CUDA_TRY(cudaMemsetAsync(&hdr->status, 0, sizeof(uint32_t), st));
  MOE_CUDA_TRY(cudaStreamSynchronize(st));
  if (status & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (status & kStatusBadIndex) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

uint64_t moe_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA launch or runtime error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

}  // extern "C"
