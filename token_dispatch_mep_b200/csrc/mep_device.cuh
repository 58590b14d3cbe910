// Device-side helpers shared by the libmep kernels: status word, bounded
// waits, the grid barrier of the plan kernel, and thin inline-PTX wrappers for
// mbarriers and the sm_90+/sm_100a bulk-copy (TMA, non-tensor) engine.
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

// Grid-wide barrier for a cooperative launch (all blocks co-resident).
// bar[0] counts arrivals, bar[32] is the generation (a separate 128-byte
// line).  The last block to arrive resets the count and bumps the
// generation; the others poll the generation for at most `limit_ns`.  The
// count is back at zero after every completed barrier, so a zero-filled
// workspace stays valid from call to call.  Returns false (and records
// MEP_ERR_TIMEOUT) if the wait ran out.
__device__ __forceinline__ bool grid_barrier(uint32_t *bar, uint32_t nblocks,
                                             uint64_t limit_ns, int32_t *status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    uint32_t *count = bar;
    uint32_t *gen = bar + 32;
    const uint32_t g = ld_acquire_gpu(gen);
    __threadfence();
    const uint32_t prev = atomicAdd(count, 1u);
    if (prev == nblocks - 1) {
      atomicExch(count, 0u);
      __threadfence();
      st_release_gpu(gen, g + 1);
    } else {
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_gpu(gen) == g) {
        if (global_timer_ns() - t0 > limit_ns) {
          ok = 0;
          set_status(status, MEP_ERR_TIMEOUT);
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// ---- mbarrier and bulk copies ------------------------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// Bulk global -> shared copy (this CTA's shared memory; no multicast),
// completion signalled on `bar` as transaction bytes.  src, dst 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst_smem)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Bulk shared -> global copy tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_store(void *dst, const void *src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_addr(src_smem)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// All but the newest N committed groups have finished reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Every committed group has completed (writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace mep
