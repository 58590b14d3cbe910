// A barrier between EP ranks on the device, in place of a host round trip
// (MoonEP release page, "Why this matters to engineers": static buffer shapes
// remove the per-layer host synchronisation).  Every rank owns R flag words
// (uint32, one per rank) in its own memory, mapped into every peer's address
// space.  Arriving at epoch n, rank r makes everything its stream wrote
// before visible system-wide and stores n into word r of every rank's flag
// array (release, system scope); it then waits until all R words of its own
// array have reached n (acquire, system scope).  After the barrier kernel
// returns, later work on the stream sees every rank's writes from before its
// arrival.
//
// Every wait is bounded by the GPU global timer (mep_set_wait_limit_ns): a
// word that does not reach the epoch in time records MEP_ERR_TIMEOUT in the
// caller's status word and the kernel returns, leaving the context usable.
// Epochs compare modulo 2^32 (a word w has reached n when (int32)(w - n) >= 0),
// so a counter that wraps keeps working.  A NULL or misaligned peer pointer
// is reported (MEP_ERR_DEVICE_DATA) and never stored through.
#include <cstdint>

#include <cuda_runtime.h>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_sys(uint32_t *p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__global__ void rank_barrier_kernel(uint32_t *const *peer_flags, const uint32_t *my_flags,
                                    int32_t R, int32_t rank, uint32_t epoch, int32_t *status,
                                    uint64_t limit_ns) {
  const int t = threadIdx.x;
  // arrive: word `rank` of every rank's array, after a system-wide fence that
  // orders this stream's earlier writes (earlier kernels) before the flags
  if (t < R) {
    uint32_t *f = peer_flags[t];
    if (f == nullptr || (reinterpret_cast<uintptr_t>(f) & 3) != 0) {
      set_status(status, MEP_ERR_DEVICE_DATA);
    } else {
      __threadfence_system();
      st_release_sys(f + rank, epoch);
    }
  }
  // wait: every rank's word in this rank's own array
  if (t < R) {
    const uint64_t t0 = global_timer_ns();
    while ((int32_t)(ld_acquire_sys(my_flags + t) - epoch) < 0) {
      if (global_timer_ns() - t0 > limit_ns) {
        set_status(status, MEP_ERR_TIMEOUT);
        break;
      }
      __nanosleep(256);
    }
  }
}

}  // namespace

cudaError_t launch_rank_barrier(uint32_t *const *peer_flags, const uint32_t *my_flags, int32_t R,
                                int32_t rank, uint32_t epoch, int32_t *status, uint64_t limit_ns,
                                cudaStream_t stream) {
  const int threads = ((R + 31) / 32) * 32;
  rank_barrier_kernel<<<1, threads, 0, stream>>>(peer_flags, my_flags, R, rank, epoch, status,
                                                 limit_ns);
  return cudaGetLastError();
}

}  // namespace mep
