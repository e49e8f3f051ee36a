// moe_dispatch_noalloc: the dispatch step for callers that cannot allocate
// device memory.
//
// Some callers are not allowed to allocate: a plugin inside a host runtime
// that owns every device allocation itself, a serving process whose memory
// is fully reserved by its own pool after warm-up (a raw cudaMalloc would
// fail or fragment it), or a latency-critical path where the implicit
// synchronisation of cudaMalloc/cudaFree is not acceptable. moe_dispatch
// needs a caller-provided workspace for its per-chunk histograms; this
// variant keeps that scratch in a fixed array in device memory that belongs
// to the library instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its kNoAllocScratchBytes until the process exits. Host code
// cannot use the variable's name as a device address, so the first call on
// each device resolves the address with cudaGetSymbolAddress (with that
// device current) and caches it. All calls share the one array, so calls
// that overlap on the GPU (other streams, other host threads) race and
// corrupt each other's scratch.
// Every scratch word a call reads is written earlier in the same call, so
// nothing has to be cleared between calls.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kNoAllocMaxCopies = 65536;                            // T * K limit
constexpr int kNoAllocMaxChunks = kNoAllocMaxCopies / kChunk;       // 32
constexpr size_t kNoAllocHistBytes = sizeof(int32_t) * kNoAllocMaxChunks * kMaxE;
constexpr size_t kNoAllocScratchBytes = sizeof(WsHeader) + 2 * kNoAllocHistBytes;  // 128.25 KiB

static __device__ __align__(256) uint8_t g_dispatch_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
static void* g_scratch_addr[kMaxDevices] = {nullptr};
static std::mutex g_scratch_mutex;

// Device address of g_dispatch_scratch on the current device (resolved once).
static moe_status scratch_on_current_device(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_scratch_addr[dev]);
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const moe_layer_desc* desc, const int32_t* topk_idx,
                                           int32_t* counts, int32_t* offsets, int32_t* perm,
                                           int32_t* inv, moe_stream stream) {
  if (!desc) return MOE_ERR_INVALID_ARG;
  const moe_layer_desc& d = *desc;
  if (d.T < 0 || d.E < 1 || d.K < 1 || d.K > d.E) return MOE_ERR_INVALID_ARG;
  if (d.E > kMaxE || d.K > kMaxK) return MOE_ERR_UNSUPPORTED;
  if ((long long)d.T * d.K > kNoAllocMaxCopies) return MOE_ERR_UNSUPPORTED;   // beyond the array
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (d.T > 0 && (!topk_idx || !perm || !inv)) return MOE_ERR_INVALID_ARG;
  uint8_t* scratch = nullptr;
  const moe_status s = scratch_on_current_device(&scratch);
  if (s != MOE_OK) return s;
  const int TK = d.T * d.K;
  const int n_chunks = TK > 0 ? (TK + kChunk - 1) / kChunk : 1;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(scratch);
  int32_t* hist = reinterpret_cast<int32_t*>(scratch + sizeof(WsHeader));
  int32_t* base = reinterpret_cast<int32_t*>(scratch + sizeof(WsHeader) + kNoAllocHistBytes);
  if (launch_dispatch_scratch(d, n_chunks, hist, base, hdr, topk_idx, counts, offsets, perm, inv,
                              static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
