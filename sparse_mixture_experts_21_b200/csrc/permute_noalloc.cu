// moe_permute_noalloc: moe_permute with its scratch in a fixed device array.
//
// Some callers cannot allocate device memory at all: a plugin running inside a
// host application whose memory pool has already reserved the whole device (a
// cudaMalloc there fails, or fragments memory the host is managing), or a
// runtime with a static memory plan in which every device buffer is decided up
// front.  moe_permute needs a small per-block count table as scratch, which its
// caller normally allocates; this variant keeps that table in a file-scope
// device array instead, so such callers need to supply only inputs and outputs.
//
// Costs and limits:
//   * every GPU that loads this library holds the array (1 MiB) until exit;
//   * the count table needs ceil(T / 256) * N int32 entries, at most
//     kNoallocScratchInts (262144); larger calls are rejected;
//   * all calls share the one array: calls that overlap on the GPU (different
//     streams, or several threads) race and must be serialised by the caller.
//     The table is fully rewritten by each call before it is read, so nothing
//     from an earlier call leaks into a later one.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace noalloc {

constexpr int64_t kNoallocScratchInts = 262144;  // 1 MiB of int32

static __device__ __align__(256) int32_t g_permute_scratch[kNoallocScratchInts];

// Device address of the array, looked up with the device current once per device
// and context.  (In host code the array's name is only a host-side stand-in.)  The
// cache is keyed by the context's unique id, so after a device reset (a new
// primary context, in which the module and the array are loaded again) the next
// call looks the address up again instead of using a stale one.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_addr[kMaxDevices] = {nullptr};
unsigned long long g_ctx_id[kMaxDevices] = {0};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

// Unique id of the current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx) get_id(ctx, &id);
  return id;
}

cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // 0 until the runtime has made the device's context current: the lookup below
  // does that, and the next call then records the context's id
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev] || ctx == 0 || ctx != g_ctx_id[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<int32_t*>(p);
    g_ctx_id[dev] = ctx;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace noalloc
}  // namespace moe

extern "C" int moe_permute_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                   int32_t* counts, int32_t* offsets, int32_t* row_of_slot,
                                   int32_t* token_of_row, void* x_perm, int32_t* n_dropped,
                                   void* stream) {
  using namespace moe;
  const int st = capi::check_config(cfg);
  if (st != MOE_OK) return st;
  if (!counts || !offsets || !n_dropped) return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!topk_idx || !row_of_slot || !token_of_row || (x_perm && !x)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && x_perm && (!capi::aligned16(x) || !capi::aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if ((int64_t)permute_blocks(cfg->T) * cfg->n_experts > noalloc::kNoallocScratchInts)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  int32_t* scratch = nullptr;
  if (noalloc::scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  return capi::from_cuda(launch_permute(*cfg, capi::capacity_of(*cfg), x, topk_idx, counts, offsets,
                                        row_of_slot, token_of_row, x_perm, n_dropped, scratch,
                                        static_cast<cudaStream_t>(stream)));
}
