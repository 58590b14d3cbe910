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
// address is looked up by cudaGetSymbolAddress, with the device current, the
// first time a call runs in a CUDA context of that device, and cached with the
// context's ID.  A later call in a different context of the same device (after
// cudaDeviceReset, the module holding the array is loaded afresh, possibly at
// another address) looks it up again, so a reset never leaves a stale address
// behind.  The lookup may load the module, so the first call in a context
// should come before any stream capture on that device.
//
// The array is shared by every call on the device and keeps the last call's
// contents.  The grid-barrier words at its start must be zero when the plan
// kernel starts, so each call clears them (a 256-byte cudaMemsetAsync on the
// caller's stream, issued only after every argument has been checked) before
// the launch; the rest is fully written before it is read.  Two calls that
// overlap on the GPU (different streams, no ordering between them) race on
// the array and give undefined plans.
#include <cstdint>
#include <mutex>

#include <cuda.h>
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

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name) {
  void *f = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPointByVersion(name, &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(f);
}

// Unique ID of the current CUDA context (IDs are never reused within a
// process), 0 if it cannot be read.
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct ScratchAddr {
  unsigned long long ctx_id = 0;  // context the address belongs to (0: none yet)
  void *addr = nullptr;
};

std::mutex g_mu;
ScratchAddr g_scratch[kMaxDevices];

// Device address of g_plan_scratch in the current context of the current
// device: looked up once per context, again whenever the context changes.
mep_status_t scratch_on_current_device(void **addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MEP_ERR_CUDA;
  // 0 if no context is current yet (the runtime makes the device's primary
  // context current on its first call that needs one, the lookup below).
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  ScratchAddr &c = g_scratch[dev];
  if (c.addr == nullptr || ctx == 0 || c.ctx_id != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || p == nullptr)
      return MEP_ERR_CUDA;
    c.addr = p;
    c.ctx_id = current_context_id();
  }
  *addr = c.addr;
  return MEP_OK;
}

}  // namespace

extern "C" {

MEP_API mep_status_t mep_plan_noalloc(mep_shape_t shape, const int32_t *topk_idx,
                                      const mep_plan_t *plan, void *stream) {
  // Every argument is checked before anything is queued on the stream.
  mep_status_t st = mep::check_plan_args(shape, topk_idx, plan);
  if (st != MEP_OK) return st;
  if (mep_plan_workspace_bytes(shape) > kStaticScratchBytes) return MEP_ERR_WORKSPACE;
  void *scratch = nullptr;
  if ((st = scratch_on_current_device(&scratch)) != MEP_OK) return st;
  if (cudaMemsetAsync(scratch, 0, mep::kPlanWsHeader, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MEP_ERR_CUDA;
  return mep_plan(shape, topk_idx, plan, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
