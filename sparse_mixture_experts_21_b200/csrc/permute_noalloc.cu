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

// Device address of the array, looked up once per device with that device
// current.  (In host code the array's name is only a host-side stand-in.)
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_addr[kMaxDevices] = {nullptr};

cudaError_t scratch_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = static_cast<int32_t*>(p);
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
  if (cfg->T > 0 && (!x || !topk_idx || !row_of_slot || !token_of_row || !x_perm))
    return MOE_ERR_INVALID_ARG;
  if (cfg->T > 0 && (!capi::aligned16(x) || !capi::aligned16(x_perm))) return MOE_ERR_INVALID_ARG;
  if ((int64_t)permute_blocks(cfg->T) * cfg->n_experts > noalloc::kNoallocScratchInts)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  int32_t* scratch = nullptr;
  if (noalloc::scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  return capi::from_cuda(launch_permute(*cfg, capi::capacity_of(*cfg), x, topk_idx, counts, offsets,
                                        row_of_slot, token_of_row, x_perm, n_dropped, scratch,
                                        static_cast<cudaStream_t>(stream)));
}
