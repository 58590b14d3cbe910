// Zero-copy dispatch: buf[slot[g,k], :] = x[g, :] for every (token, k) pair.
//
// Method: each token row is copied once per routed expert, directly into its
// final slot of an expert-ordered receive buffer whose shape never changes
// (MoonEP release page, "Why this matters to engineers"; "How MoonEP works":
// a fixed S*K slots per rank).
//
// Token-major, so each hidden row crosses HBM once on the way in and K times
// on the way out (the algorithmic minimum).  Each warp runs its own pipeline
// over a contiguous token range: lane 0 streams rows into a ring of
// shared-memory stages with bulk (TMA) loads completed on per-stage
// mbarriers, and issues the K bulk stores of each row from its stage into
// the K destination slots.  A stage is refilled once the bulk group that
// reads it has finished reading.  The slot indices of the next 32 tokens are
// prefetched into registers by all 32 lanes and broadcast with shuffles, so
// the issuing lane never waits on a slot load.  Every slot is bounds-checked
// against [0, N*K) before it is used.
#include <algorithm>
#include <cstdint>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

#ifndef MEP_DISPATCH_WARPS
#define MEP_DISPATCH_WARPS 4  // independent pipelines (warps) per block
#endif
#ifndef MEP_DISPATCH_STAGES
#define MEP_DISPATCH_STAGES 16  // shared-memory stages per pipeline, at most
#endif

constexpr int kMaxWarps = MEP_DISPATCH_WARPS;
constexpr int kMaxStages = MEP_DISPATCH_STAGES;
constexpr int kMaxK = 16;

struct DispatchParams {
  const uint16_t *x;
  uint16_t *buf;
  const int32_t *slot;
  int32_t *status;
  int64_t N, NK;
  int32_t K, H;
  uint32_t row_bytes;
  int32_t stages;
  int64_t tokens_per_warp;
  uint64_t wait_ns;
};

template <int KC>
__device__ __forceinline__ void load_slots(int (&r)[KC], const int32_t *slot, int64_t g, int64_t t1,
                                           int K) {
#pragma unroll
  for (int k = 0; k < KC; ++k) r[k] = (g < t1 && k < K) ? __ldg(slot + g * K + k) : -1;
}

template <int KC>
__global__ void __launch_bounds__(kMaxWarps * 32) dispatch_kernel(DispatchParams p) {
  extern __shared__ __align__(128) unsigned char stage_mem[];
  __shared__ __align__(8) uint64_t full_bar[kMaxWarps][kMaxStages];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  const int64_t t0 = gw * p.tokens_per_warp;
  const int64_t t1 = std::min(t0 + p.tokens_per_warp, p.N);
  if (t0 >= t1) return;  // warp-uniform; no block-wide sync below
  const int64_t n = t1 - t0;
  const int S = p.stages;
  const uint32_t rb = p.row_bytes;
  unsigned char *stages = stage_mem + (size_t)warp * S * rb;
  uint64_t *full = full_bar[warp];

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
    const int64_t pro = std::min<int64_t>(S, n);
    for (int64_t i = 0; i < pro; ++i) {
      mbar_arrive_expect_tx(&full[i], rb);
      bulk_load(stages + i * rb, p.x + (t0 + i) * p.H, rb, &full[i]);
    }
  }
  __syncwarp();

  int cur[KC], nxt[KC];
  load_slots<KC>(cur, p.slot, t0 + lane, t1, p.K);
  bool bad = false, timed_out = false;
  int64_t issued_loads = std::min<int64_t>(S, n);  // loads issued so far
  int64_t consumed = 0;                           // loads waited for

  for (int64_t g0 = 0; g0 < n && !timed_out; g0 += 32) {
    load_slots<KC>(nxt, p.slot, t0 + g0 + 32 + lane, t1, p.K);
    const int jn = (int)std::min<int64_t>(32, n - g0);
    for (int j = 0; j < jn; ++j) {
      const int64_t i = g0 + j;
      const int s = (int)(i % S);
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&full[s], (uint32_t)((i / S) & 1), p.wait_ns);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        timed_out = true;
        break;
      }
      consumed = i + 1;
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        if (k < p.K) {
          const int pk = __shfl_sync(0xffffffffu, cur[k], j);
          if (lane == 0) {
            if ((unsigned)pk < (unsigned)p.NK)
              bulk_store(p.buf + (int64_t)pk * p.H, stages + (size_t)s * rb, rb);
            else
              bad = true;
          }
        }
      }
      if (lane == 0) {
        bulk_commit();
        const int64_t next = i - 1 + S;  // refill the stage of token i-1
        if (i >= 1 && next < n) {
          bulk_wait_read<1>();
          const int sp = (int)((i - 1) % S);
          mbar_arrive_expect_tx(&full[sp], rb);
          bulk_load(stages + (size_t)sp * rb, p.x + (t0 + next) * p.H, rb, &full[sp]);
          issued_loads = next + 1;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < KC; ++k) cur[k] = nxt[k];
  }

  if (lane == 0) {
    if (timed_out) {
      set_status(p.status, MEP_ERR_TIMEOUT);
      // Give the loads still in flight a bounded chance to land before the
      // shared memory they target goes away.
      for (int64_t i = consumed; i < issued_loads; ++i)
        (void)mbar_wait_bounded(&full[i % S], (uint32_t)((i / S) & 1), p.wait_ns);
    }
    bulk_wait_all();
    if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
  }
}

template <int KC>
cudaError_t launch_kc(const DispatchParams &p, int warps, int blocks, size_t smem,
                      cudaStream_t stream) {
  cudaError_t err = cudaFuncSetAttribute(dispatch_kernel<KC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dispatch_kernel<KC><<<blocks, warps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                            const uint16_t *x, uint16_t *buf, uint64_t wait_ns,
                            cudaStream_t stream) {
  int dev = 0, sms = 0, smem_max = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  if ((err = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
      cudaSuccess)
    return err;
  DispatchParams p{};
  p.x = x;
  p.buf = buf;
  p.slot = pl.slot;
  p.status = pl.status;
  p.N = (int64_t)s.R * s.S;
  p.NK = p.N * s.K;
  p.K = s.K;
  p.H = H;
  p.row_bytes = (uint32_t)H * 2u;
  p.wait_ns = wait_ns;

  // Shared-memory budget: leave room for the static mbarriers.
  const size_t budget = (size_t)std::max(0, smem_max - 4096);
  int warps = (int)std::min<size_t>(kMaxWarps, budget / (2 * (size_t)p.row_bytes));
  if (warps < 1) return cudaErrorInvalidValue;
  int stages = (int)std::min<size_t>(kMaxStages, budget / ((size_t)warps * p.row_bytes));
  stages = std::max(stages, 2);
  p.stages = stages;
  const size_t smem = (size_t)warps * stages * p.row_bytes;

  const int64_t total_warps = std::min<int64_t>(p.N, (int64_t)sms * warps);
  p.tokens_per_warp = (p.N + total_warps - 1) / total_warps;
  const int64_t used_warps = (p.N + p.tokens_per_warp - 1) / p.tokens_per_warp;
  const int blocks = (int)((used_warps + warps - 1) / warps);

  if (s.K <= 2) return launch_kc<2>(p, warps, blocks, smem, stream);
  if (s.K <= 4) return launch_kc<4>(p, warps, blocks, smem, stream);
  if (s.K <= 8) return launch_kc<8>(p, warps, blocks, smem, stream);
  return launch_kc<kMaxK>(p, warps, blocks, smem, stream);
}

}  // namespace mep
