// Device-side helpers shared by the libmep kernels: the status word, the
// global timer, acquire/release accesses and the bounded grid barrier of the
// plan kernel.
//
// Every wait in this library is bounded by the GPU global timer; a wait that
// runs out records MEP_ERR_TIMEOUT in the caller's status word and returns
// false so the kernel can wind down.  No kernel traps or asserts.
#pragma once

#include <cstdint>

#include "mep.h"

namespace mep {

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch: a kernel launched with launch_pdl may start
// (launch, block scheduling, prologue) while the previous kernel on its stream
// drains; every such kernel calls griddep_wait() before its first global
// memory access, which returns once the previous kernel has completed and its
// writes are visible -- so results are exactly those of plain stream order.
// Without the launch attribute the wait is a no-op.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// First error wins.
__device__ __forceinline__ void set_status(int32_t *status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ uint32_t lanemask_gt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_gt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ void red_release_add_gpu(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier for a cooperative launch (all blocks co-resident).
// bar[0] counts arrivals over the whole launch: the k-th barrier of a launch
// opens when it reaches k * nblocks.  Thread 0 of each block adds its arrival
// with release semantics (publishing the block's earlier writes, ordered by
// __syncthreads) and polls with acquire loads for at most `limit_ns`; the
// count is compared as a signed value.  Returns false (and records
// MEP_ERR_TIMEOUT) if the wait ran out.
__device__ __forceinline__ bool grid_barrier(uint32_t *bar, int target, uint64_t limit_ns,
                                             int32_t *status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    red_release_add_gpu(bar, 1u);
    if ((int)ld_acquire_gpu(bar) < target) {
      const uint64_t t0 = global_timer_ns();
      while ((int)ld_acquire_gpu(bar) < target) {
        if (global_timer_ns() - t0 > limit_ns) {
          ok = 0;
          set_status(status, MEP_ERR_TIMEOUT);
          break;
        }
      }
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// Called once by every block after its last barrier: bar[32] counts the
// blocks that are done; the last one puts both words back to zero, so a
// zero-filled workspace is zero again after every clean launch.
__device__ __forceinline__ void grid_barrier_exit(uint32_t *bar, uint32_t nblocks) {
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(bar + 32, 1u);
    if (prev == nblocks - 1) {
      atomicExch(bar, 0u);
      atomicExch(bar + 32, 0u);
    }
  }
}

}  // namespace mep
