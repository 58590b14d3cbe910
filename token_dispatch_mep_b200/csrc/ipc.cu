// Buffer sharing between the processes of an expert-parallel group: one
// process per GPU exports its receive, expert-output and gradient buffers,
// the others map them, and the mapped addresses fill the device pointer
// arrays of the rank-addressed calls -- so dispatch's stores and combine's
// loads go straight to the GPU that owns each slot.
//
// CUDA IPC handles name whole allocations, while a caller's buffer is usually
// a range inside one (a caching allocator hands out pieces of larger
// cudaMalloc segments).  The export therefore finds the allocation that
// contains the range (the driver's address-range query, reached through the
// runtime's driver entry point so the library does not link the driver) and
// records the range's offset in it; the opening process adds the offset back.
// Several exported buffers can share one allocation, so the opening side
// maps each allocation once per device and counts its users: the last close
// unmaps it.
#include <array>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>

#include "mep.h"

namespace {

static_assert(sizeof(cudaIpcMemHandle_t) == sizeof(((mep_ipc_handle_t *)0)->handle),
              "mep_ipc_handle_t must hold a cudaIpcMemHandle_t");

using AddressRangeFn = CUresult (*)(CUdeviceptr *base, size_t *size, CUdeviceptr ptr);

// The driver's address-range query, looked up once.
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = []() -> AddressRangeFn {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<AddressRangeFn>(f);
  }();
  return fn;
}

// Allocations mapped by mep_ipc_open, keyed by (device, handle bytes).
struct Mapping {
  void *base = nullptr;
  int users = 0;
};
using MapKey = std::pair<int, std::array<unsigned char, 64>>;
std::mutex g_map_mu;
std::map<MapKey, Mapping> g_maps;

bool map_key(const mep_ipc_handle_t *h, MapKey *key) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  key->first = dev;
  std::memcpy(key->second.data(), h->handle, 64);
  return true;
}

}  // namespace

extern "C" {

mep_status_t mep_ipc_export(const void *ptr, uint64_t bytes, mep_ipc_handle_t *out) {
  if (ptr == nullptr || out == nullptr || bytes == 0) return MEP_ERR_INVALID_ARG;
  AddressRangeFn range = address_range_fn();
  if (range == nullptr) return MEP_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  const CUdeviceptr p = reinterpret_cast<CUdeviceptr>(ptr);
  if (range(&base, &size, p) != CUDA_SUCCESS) return MEP_ERR_INVALID_ARG;
  const uint64_t offset = p - base;
  if (offset > size || bytes > size - offset) return MEP_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return MEP_ERR_CUDA;
  std::memcpy(out->handle, &h, sizeof h);
  out->offset = offset;
  out->bytes = bytes;
  return MEP_OK;
}

mep_status_t mep_ipc_open(const mep_ipc_handle_t *handle, void **ptr) {
  if (handle == nullptr || ptr == nullptr) return MEP_ERR_INVALID_ARG;
  MapKey key;
  if (!map_key(handle, &key)) return MEP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_map_mu);
  Mapping &m = g_maps[key];
  if (m.users == 0) {
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle->handle, sizeof h);
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
      g_maps.erase(key);
      return MEP_ERR_CUDA;
    }
    m.base = base;
  }
  ++m.users;
  *ptr = static_cast<char *>(m.base) + handle->offset;
  return MEP_OK;
}

mep_status_t mep_ipc_close(const mep_ipc_handle_t *handle, void *ptr) {
  if (handle == nullptr || ptr == nullptr) return MEP_ERR_INVALID_ARG;
  MapKey key;
  if (!map_key(handle, &key)) return MEP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_map_mu);
  auto it = g_maps.find(key);
  if (it == g_maps.end() || static_cast<char *>(it->second.base) + handle->offset != ptr)
    return MEP_ERR_INVALID_ARG;
  if (--it->second.users > 0) return MEP_OK;
  void *base = it->second.base;
  g_maps.erase(it);
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? MEP_OK : MEP_ERR_CUDA;
}

}  // extern "C"
