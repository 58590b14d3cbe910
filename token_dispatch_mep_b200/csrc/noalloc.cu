// mep_plan_noalloc: the plan call for callers that cannot allocate device
// memory.
//
// Some callers have no way to obtain a device buffer for the workspace: code
// running under an allocator-less runtime, a host thread that must not call
// cudaMalloc while another component owns the device memory pool, or a plugin
// whose host framework forbids allocation after start-up.  This entry point
// gives them the plan without a caller-supplied workspace.  Its scratch is a
// file-scope device array compiled into the library, of a fixed size that
// covers every shape the library accepts (the plan workspace of
// MEP_MAX_EXPERTS experts).  Every GPU that loads the library holds this
// array until the process exits.
//
// In host code, `g_plan_scratch` names a host-side shadow, not device memory:
// passing it to a kernel would fault or read the wrong memory.  The device
// address is looked up once per device, with that device current, by
// cudaGetSymbolAddress, and that address is what the plan kernel receives.
//
// The array is shared by every call on the device and keeps the last call's
// contents.  The grid-barrier words at its start must be zero when the plan
// kernel starts, so each call clears them (a 256-byte cudaMemsetAsync on the
// caller's stream) before the launch; the rest is fully written before it is
// read.  Two calls that overlap on the GPU (different streams, no ordering
// between them) race on the array and give undefined plans.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "mep.h"
#include "mep_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = MEP_NOALLOC_SCRATCH_BYTES;
static_assert(kStaticScratchBytes == mep::kPlanWsHeader + (size_t)MEP_MAX_EXPERTS *
                                         mep::kPlanMaxBlocks * sizeof(int32_t),
              "the static scratch must hold the plan workspace of MEP_MAX_EXPERTS experts");

static __device__ __align__(256) unsigned char g_plan_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_plan_scratch on the current device (looked up on the
// first call for that device).
mep_status_t scratch_on_current_device(void **addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MEP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || p == nullptr)
      return MEP_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return MEP_OK;
}

}  // namespace

extern "C" {

MEP_API mep_status_t mep_plan_noalloc(mep_shape_t shape, const int32_t *topk_idx,
                                      const mep_plan_t *plan, void *stream) {
  const size_t need = mep_plan_workspace_bytes(shape);
  if (need == 0) return MEP_ERR_INVALID_ARG;         // shape outside the library's rules
  if (need > kStaticScratchBytes) return MEP_ERR_WORKSPACE;
  if (topk_idx == nullptr || plan == nullptr) return MEP_ERR_INVALID_ARG;
  void *scratch = nullptr;
  mep_status_t st = scratch_on_current_device(&scratch);
  if (st != MEP_OK) return st;
  if (cudaMemsetAsync(scratch, 0, mep::kPlanWsHeader, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MEP_ERR_CUDA;
  return mep_plan(shape, topk_idx, plan, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
