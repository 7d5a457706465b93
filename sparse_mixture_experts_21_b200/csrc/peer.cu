// Peer mappings for the expert-parallel exchange over NVLink: a rank exports the
// address of a device buffer as a CUDA IPC handle plus the buffer's offset inside
// its allocation; the other ranks (processes on other GPUs of the node) import it
// and get a pointer their kernels load from and store to directly.
//
// The buffer may sit anywhere inside a cudaMalloc allocation (a caching allocator
// hands out sub-ranges of larger blocks): the handle names the allocation, the
// offset the buffer.  Two buffers of one allocation give the same allocation
// handle, and the runtime maps an allocation once per process, so imports are
// reference-counted per allocation.
#include <string.h>

#include <map>
#include <mutex>
#include <string>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace peer {

typedef CUresult (*MemGetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

MemGetAddressRangeFn address_range_fn() {
  static MemGetAddressRangeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<MemGetAddressRangeFn>(p);
    return static_cast<MemGetAddressRangeFn>(nullptr);
  }();
  return fn;
}

struct Mapping {
  void* base;
  int refs;
};

std::mutex g_mu;
std::map<std::string, Mapping> g_by_handle;     // allocation handle bytes -> mapping
std::map<uintptr_t, std::string> g_by_ptr;      // imported pointer -> allocation handle bytes
std::map<uintptr_t, int> g_ptr_refs;            // imported pointer -> imports not yet closed

}  // namespace peer

cudaError_t peer_export(const void* ptr, uint8_t* handle, int64_t* offset) {
  auto fn = peer::address_range_fn();
  if (!fn) return cudaErrorNotSupported;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return e;
  memcpy(handle, &h, sizeof(h));
  *offset = (int64_t)(reinterpret_cast<uintptr_t>(ptr) - (uintptr_t)base);
  return cudaSuccess;
}

cudaError_t peer_import(const uint8_t* handle, int64_t offset, void** ptr) {
  const std::string key(reinterpret_cast<const char*>(handle), sizeof(cudaIpcMemHandle_t));
  std::lock_guard<std::mutex> lock(peer::g_mu);
  auto it = peer::g_by_handle.find(key);
  void* base = nullptr;
  if (it != peer::g_by_handle.end()) {
    base = it->second.base;
    it->second.refs += 1;
  } else {
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof(h));
    cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return e;
    peer::g_by_handle[key] = peer::Mapping{base, 1};
  }
  *ptr = static_cast<uint8_t*>(base) + offset;
  const uintptr_t p = reinterpret_cast<uintptr_t>(*ptr);
  peer::g_by_ptr[p] = key;
  peer::g_ptr_refs[p] += 1;
  return cudaSuccess;
}

// 1 when ptr was never imported (or is already closed), else the CUDA status.
int peer_close(void* ptr) {
  std::lock_guard<std::mutex> lock(peer::g_mu);
  const uintptr_t p = reinterpret_cast<uintptr_t>(ptr);
  auto pi = peer::g_by_ptr.find(p);
  if (pi == peer::g_by_ptr.end()) return 1;
  const std::string key = pi->second;
  if (--peer::g_ptr_refs[p] == 0) {
    peer::g_ptr_refs.erase(p);
    peer::g_by_ptr.erase(pi);
  }
  auto it = peer::g_by_handle.find(key);
  if (it == peer::g_by_handle.end()) return 1;
  if (--it->second.refs > 0) return 0;
  void* base = it->second.base;
  peer::g_by_handle.erase(it);
  return (int)cudaIpcCloseMemHandle(base);
}

}  // namespace moe
