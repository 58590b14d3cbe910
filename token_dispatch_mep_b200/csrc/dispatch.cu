// Zero-copy dispatch: buf[slot[g,k], :] = x[g, :] for every (token, k) pair.
//
// Method: each token row is copied once per routed expert, directly into its
// final slot of an expert-ordered receive buffer whose shape never changes
// (MoonEP release page, "Why this matters to engineers"; "How MoonEP works":
// a fixed S*K slots per rank).
//
// Token-major, so each hidden row is read from HBM once and written K times
// (the algorithmic minimum).  A warp task is one token and a run of 32 x kU
// 16-byte chunks of its row (lane l owns chunks l, l+32, ...).  Lanes k < K
// fetch the token's slot ids, which the warp broadcasts with shuffles; the
// next task's ids are fetched before the current task's row, so consecutive
// tasks' dependent loads overlap.  Each lane loads its kU chunks once
// (streaming loads) and stores them to the K slots (streaming stores), so a
// warp writes 512-byte contiguous runs.  The grid is several times the
// resident capacity, so blocks that finish early are replaced by new ones
// (uneven destination rows balance out).  Every slot is bounds-checked
// against [0, N*K) before it is used.
//
// Occupancy: one block of 24 warps per SM.  Measured over block sizes and
// residencies (16, 24, 32, 40 warps per SM), 24 resident warps moved the
// most bytes on every workload (1-2.5 % over 40): more concurrent store
// streams only queue behind one another.  The block asks for more than half
// an SM's shared memory (unused) so that a second block cannot be resident.
//
// Rank-addressed form (mep_dispatch_ranked): rank r's S*K slots live in
// their own buffer rank_bufs[r] (on a multi-GPU system a peer buffer mapped
// into this GPU's address space), so slot p is row p % SK of rank_bufs[p / SK]
// and each store goes straight to the rank that owns the slot; a NULL or
// misaligned rank pointer is reported, never used.  A token range [g0, g0 +
// N) restricts the kernel to one rank's own tokens (mep_dispatch_ranked_tokens).
//
// A bulk-copy (TMA) design -- rows staged in shared memory by bulk loads on
// mbarriers, K bulk stores per row -- measured 0.82-0.87 of the HBM copy
// peak on this path against 0.89-0.94 for the register path at the time
// (0.99-1.03 now), so it is not used.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_DISPATCH_U
#define MEP_DISPATCH_U 4  // 16-byte chunks per lane per task
#endif
#ifndef MEP_DISPATCH_BLOCKS_PER_SM
#define MEP_DISPATCH_BLOCKS_PER_SM 1024  // grid cap in multiples of the SM count
#endif
#ifndef MEP_DISPATCH_THREADS
#define MEP_DISPATCH_THREADS 768  // threads per block, one block resident per SM
#endif

namespace mep {

namespace {

constexpr int kThreads = MEP_DISPATCH_THREADS;
constexpr int kWarps = kThreads / 32;
constexpr int kU = MEP_DISPATCH_U;

struct DispatchParams {
  const uint16_t *x;
  uint16_t *buf;
  uint16_t *const *rank_bufs;  // ranked form: R row buffers of SK rows
  int64_t SK;
  const int32_t *slot;
  int32_t *status;
  int64_t g0;     // first token (global order); x row i is token g0 + i
  int64_t N, NK;  // tokens processed, slots of the plan
  int32_t K, H;
  int32_t chunks;  // 16-byte chunks per row = H / 8
  int32_t parts;   // warp tasks per token
};

template <int KC, bool kRanked>
__global__ void __launch_bounds__(kThreads) dispatch_kernel(DispatchParams p) {
  griddep_wait();  // the previous kernel on the stream is complete and visible
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  const int64_t ntask = p.N * p.parts;
  int64_t task = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  bool bad = false;
  auto fetch = [&](int64_t t) -> int {
    return (t < ntask && lane < p.K) ? __ldg(p.slot + (p.g0 + t / p.parts) * p.K + lane) : -1;
  };
  int sl = fetch(task);
  for (; task < ntask; task += nwarps) {
    const int nsl = fetch(task + nwarps);
    const int64_t g = task / p.parts;
    const int cbase = (int)(task - g * p.parts) * 32 * kU + lane;
    const uint4 *xrow = reinterpret_cast<const uint4 *>(p.x + g * p.H);
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = cbase + u * 32;
      if (c < p.chunks) v[u] = __ldcs(xrow + c);
    }
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int pk = __shfl_sync(0xffffffffu, sl, k);
      if (k < p.K) {
        uint16_t *row = nullptr;
        if ((unsigned)pk < (unsigned)p.NK) {
          if (kRanked) {
            // a rank buffer must be present and 16-byte aligned
            const int64_t r = pk / p.SK;
            uint16_t *base = p.rank_bufs[r];
            if (base != nullptr && (reinterpret_cast<uintptr_t>(base) & 15) == 0)
              row = base + (pk - r * p.SK) * p.H;
          } else {
            row = p.buf + (int64_t)pk * p.H;
          }
        }
        if (row != nullptr) {
          uint4 *brow = reinterpret_cast<uint4 *>(row);
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int c = cbase + u * 32;
            if (c < p.chunks) __stcs(brow + c, v[u]);
          }
        } else {
          bad = true;
        }
      }
    }
    sl = nsl;
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

// Per-device launch constants: SM count and the shared-memory request that
// keeps one dispatch block per SM, set up once per device under the mutex and
// published by the release store of smem.
struct DispatchDev {
  std::mutex mu;
  int sms = 0;
  std::atomic<int> smem{-1};
};
DispatchDev g_dispatch_dev[64];

template <int KC>
cudaError_t set_smem_attr(int smem) {
  cudaError_t err = cudaFuncSetAttribute(dispatch_kernel<KC, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  return cudaFuncSetAttribute(dispatch_kernel<KC, false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t dispatch_dev(DispatchDev *&out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DispatchDev &d = g_dispatch_dev[dev];
  if (d.smem.load(std::memory_order_acquire) < 0) {
    std::lock_guard<std::mutex> lock(d.mu);
    if (d.smem.load(std::memory_order_acquire) >= 0) {
      out = &d;
      return cudaSuccess;
    }
    int sms = 0, per_sm = 0, per_block = 0;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return err;
    if ((err = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                      dev)) != cudaSuccess)
      return err;
    if ((err = cudaDeviceGetAttribute(&per_block, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                                      dev)) != cudaSuccess)
      return err;
    // Just over half of the SM's shared memory: a second block never fits.
    const int smem = std::min(per_block, per_sm / 2 + 1024);
    if ((err = set_smem_attr<2>(smem)) != cudaSuccess) return err;
    if ((err = set_smem_attr<4>(smem)) != cudaSuccess) return err;
    if ((err = set_smem_attr<8>(smem)) != cudaSuccess) return err;
    if ((err = set_smem_attr<16>(smem)) != cudaSuccess) return err;
    d.sms = sms;
    d.smem.store(smem, std::memory_order_release);
  }
  out = &d;
  return cudaSuccess;
}

template <int KC>
cudaError_t launch_kc(const DispatchParams &p, const DispatchDev &d, cudaStream_t stream) {
  const int64_t want = (p.N * p.parts + kWarps - 1) / kWarps;
  const int blocks = (int)std::max<int64_t>(
      1, std::min<int64_t>(want, (int64_t)d.sms * MEP_DISPATCH_BLOCKS_PER_SM));
  const int smem = d.smem.load(std::memory_order_relaxed);
  if (p.rank_bufs != nullptr)
    return launch_pdl(dispatch_kernel<KC, true>, dim3(blocks), dim3(kThreads), (size_t)smem, stream, p);
  return launch_pdl(dispatch_kernel<KC, false>, dim3(blocks), dim3(kThreads), (size_t)smem, stream, p);
}

}  // namespace

cudaError_t launch_dispatch(const mep_shape_t &s, int32_t H, const mep_plan_t &pl, int64_t g0,
                            int64_t count, const uint16_t *x, uint16_t *buf,
                            uint16_t *const *rank_bufs, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
  DispatchDev *d = nullptr;
  const cudaError_t err = dispatch_dev(d);
  if (err != cudaSuccess) return err;
  DispatchParams p{};
  p.x = x;
  p.buf = buf;
  p.rank_bufs = rank_bufs;
  p.SK = (int64_t)s.S * s.K;
  p.slot = pl.slot;
  p.status = pl.status;
  p.g0 = g0;
  p.N = count;
  p.NK = (int64_t)s.R * s.S * s.K;
  p.K = s.K;
  p.H = H;
  p.chunks = H / 8;
  p.parts = (p.chunks + 32 * kU - 1) / (32 * kU);
  if (s.K <= 2) return launch_kc<2>(p, *d, stream);
  if (s.K <= 4) return launch_kc<4>(p, *d, stream);
  if (s.K <= 8) return launch_kc<8>(p, *d, stream);
  return launch_kc<16>(p, *d, stream);
}

}  // namespace mep
