// Dispatch through the bulk-copy engine: buf[slot[g,k], :] = x[g, :], the
// same result as dispatch_kernel, with every row staged in shared memory.
//
// Method: each token row is copied once per routed expert straight into its
// final slot of the static, expert-ordered receive buffer (MoonEP release
// page, "Why this matters to engineers").  This form follows the staging
// recipe -- rows moved between HBM and shared memory by the bulk-copy (TMA)
// engine rather than by threads -- and is kept beside the register form for
// comparison: on B200 it moves 0.83-0.86 of the HBM copy bandwidth on the
// R=8/E=64, Kimi-shaped and R=32 skew workloads against 0.96-0.99 for the
// register form, so mep_dispatch uses the register form.
//
// Each warp is a pipeline of kStages shared-memory row buffers; its lane 0
// issues, per token, one bulk load of the row into a stage (completion on the
// stage's mbarrier, transaction-counted) and, once the row has landed, K bulk
// stores of that stage to the token's slots, committed as one bulk group.
// Before a stage is loaded again, the group that last read it must have
// finished reading (cp.async.bulk.wait_group.read).  Plain (non-tensor) bulk
// copies: 16-byte aligned addresses and row sizes, no multicast.
//
// Every mbarrier wait is bounded by the GPU global timer; a wait that runs out
// records MEP_ERR_TIMEOUT and the warp stops issuing work, then drains its
// outstanding bulk stores and waits (bounded) for its outstanding row load
// before returning.  A slot outside [0, N*K) records MEP_ERR_DEVICE_DATA and
// is skipped.
#include <algorithm>
#include <cstdint>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

constexpr int kStages = 2;
constexpr int kMaxWarps = 8;
constexpr int kSmemBudget = 200 * 1024;  // stage buffers per block

struct BulkParams {
  const uint8_t *x;
  uint8_t *buf;
  const int32_t *slot;
  int32_t *status;
  int64_t N, NK;
  int32_t K;
  int32_t rowbytes;
  uint64_t wait_ns;
};

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Waits (bounded) for phase `parity` of the mbarrier at `mb`; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t mb, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(mb), "r"(parity)
        : "memory");
    if (done) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

__global__ void __launch_bounds__(kMaxWarps * 32) dispatch_bulk_kernel(BulkParams p) {
  griddep_wait();  // the previous kernel on the stream is complete and visible
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t mbar[kMaxWarps][kStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  if (lane != 0) return;  // one issuing thread per pipeline
  uint8_t *stages = stage_mem + (size_t)warp * kStages * p.rowbytes;
  for (int s = 0; s < kStages; ++s)
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&mbar[warp][s])));
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // inits visible to the copy engine

  uint32_t parity[kStages] = {};
  bool pending_load = false;  // a load whose completion was not observed
  uint32_t pending_mb = 0, pending_parity = 0;
  int64_t it = 0;
  const int64_t nw = (int64_t)gridDim.x * W;
  for (int64_t g = (int64_t)blockIdx.x * W + warp; g < p.N; g += nw, ++it) {
    const int s = (int)(it % kStages);
    uint8_t *st = stages + (size_t)s * p.rowbytes;
    const uint32_t mb = smem_u32(&mbar[warp][s]);
    // the stores that read this stage kStages tokens ago are done reading it
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kStages - 1) : "memory");
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mb),
                 "r"(p.rowbytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(st)),
        "l"(p.x + g * (int64_t)p.rowbytes), "r"(p.rowbytes), "r"(mb)
        : "memory");
    if (!mbar_wait(mb, parity[s], p.wait_ns)) {
      set_status(p.status, MEP_ERR_TIMEOUT);
      pending_load = true;
      pending_mb = mb;
      pending_parity = parity[s];
      break;
    }
    parity[s] ^= 1u;
    for (int k = 0; k < p.K; ++k) {
      const int q = __ldg(p.slot + g * p.K + k);
      if ((unsigned)q >= (unsigned)p.NK) {
        set_status(p.status, MEP_ERR_DEVICE_DATA);
        continue;
      }
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                       p.buf + (int64_t)q * p.rowbytes),
                   "r"(smem_u32(st)), "r"(p.rowbytes)
                   : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores issued are complete
  if (pending_load) mbar_wait(pending_mb, pending_parity, p.wait_ns);
}

}  // namespace

cudaError_t launch_dispatch_bulk(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                                 const uint16_t *x, uint16_t *buf, uint64_t wait_ns,
                                 cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  BulkParams p{};
  p.x = reinterpret_cast<const uint8_t *>(x);
  p.buf = reinterpret_cast<uint8_t *>(buf);
  p.slot = pl.slot;
  p.status = pl.status;
  p.N = (int64_t)s.R * s.S;
  p.NK = p.N * s.K;
  p.K = s.K;
  p.rowbytes = H * 2;  // a multiple of 16 (H % 8 == 0)
  p.wait_ns = wait_ns;
  // 8 pipelines of 2 stages per block, fewer when long rows would not fit;
  // one block per SM (the measured best of 1-16 pipelines and 2-4 stages)
  const int warps = std::max(1, std::min(kMaxWarps, kSmemBudget / (kStages * p.rowbytes)));
  const size_t smem = (size_t)warps * kStages * p.rowbytes;
  if ((err = cudaFuncSetAttribute(dispatch_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
    return err;
  return launch_pdl(dispatch_bulk_kernel, dim3(sms), dim3(warps * 32), smem, stream, p);
}

}  // namespace mep
