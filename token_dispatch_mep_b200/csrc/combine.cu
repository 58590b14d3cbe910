// Weighted combine back to token order:
//   out[g, :] = bf16_rne( sum_{k=0..K-1} w[g,k] * y[slot[g,k], :] )
// accumulated in float32 with one fused multiply-add per term, k ascending.
//
// Method: a router assigns every token to K experts (MoonEP release page,
// "Why expert parallelism is needed"); the K expert outputs return to the
// token's position, weighted by the router weights.
//
// Work unit: a warp task = one token and a run of 32 x kU 16-byte column
// chunks of its row (lane l owns chunks l, l+32, ...).  Lanes k < K load the
// token's slot id and weight once and the warp broadcasts them with
// shuffles; the next task's slot ids and weights are fetched before the
// current task's rows, so the two dependent loads of consecutive tasks
// overlap.  Each lane then issues all K x kU independent 16-byte streaming
// loads before it touches any of them, adds them in k order with float32
// FMAs, rounds to bf16 and writes 16 bytes per chunk (streaming store).
//
// Rank-addressed form (mep_combine_ranked): expert outputs are read from R
// separate rank buffers, slot p being row p % SK of rank_ys[p / SK].
//
// With no weights (w == nullptr) every weight is 1 and the kernel is the
// backward of dispatch: grad_x[g] = bf16(sum_k grad_buf[slot[g,k]]) (an FMA
// with weight 1 rounds exactly like an addition).
#include <algorithm>
#include <cstdint>

#include <cuda_bf16.h>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_COMBINE_LOADS
#define MEP_COMBINE_LOADS 16  // 16-byte row loads in flight per lane (K x kU)
#endif
#ifndef MEP_COMBINE_MAX_U
#define MEP_COMBINE_MAX_U 2  // 16-byte chunks per lane per task, at most
#endif
#ifndef MEP_COMBINE_BLOCKS_PER_SM
#define MEP_COMBINE_BLOCKS_PER_SM 4
#endif
#ifndef MEP_COMBINE_MIN_BLOCKS
#define MEP_COMBINE_MIN_BLOCKS 2  // launch bound: resident blocks per SM
#endif

namespace mep {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct CombineParams {
  const uint16_t *y;
  const uint16_t *const *rank_ys;  // ranked form: R row buffers of SK rows
  int64_t SK;
  const float *w;
  const int32_t *slot;
  uint16_t *out;
  int32_t *status;
  int64_t N, NK;
  int32_t K, H;
  int32_t chunks;      // 16-byte chunks per row = H / 8
  int32_t parts;       // warp tasks per token
};

__device__ __forceinline__ void fma8(float (&acc)[8], float wk, const uint4 &v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = __uint_as_float(u[j] << 16);
    const float hi = __uint_as_float(u[j] & 0xffff0000u);
    acc[2 * j] = __fmaf_rn(wk, lo, acc[2 * j]);
    acc[2 * j + 1] = __fmaf_rn(wk, hi, acc[2 * j + 1]);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
  uint32_t u[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * j], acc[2 * j + 1]);
    u[j] = *reinterpret_cast<const uint32_t *>(&b);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

template <int KC, int U, bool kRanked>
__global__ void __launch_bounds__(kThreads, MEP_COMBINE_MIN_BLOCKS) combine_kernel(CombineParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  const int64_t ntask = p.N * p.parts;
  int64_t task = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  bool bad = false;

  // slot id and weight of (token of `task`, k = lane) for lanes < K
  auto fetch = [&](int64_t t, int &sl, float &wt) {
    sl = -1;
    wt = 0.f;
    if (t < ntask && lane < p.K) {
      const int64_t g = t / p.parts;
      sl = __ldg(p.slot + g * p.K + lane);
      wt = p.w != nullptr ? __ldg(p.w + g * p.K + lane) : 1.f;
    }
  };
  int sl, nsl;
  float wt, nwt;
  fetch(task, sl, wt);

  for (; task < ntask; task += nwarps) {
    fetch(task + nwarps, nsl, nwt);
    const int64_t g = task / p.parts;
    const int cbase = (int)(task - g * p.parts) * 32 * U + lane;
    uint4 v[KC][U];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int pk = __shfl_sync(0xffffffffu, sl, k);
      if (k < p.K) {
        const bool ok = (unsigned)pk < (unsigned)p.NK;
        bad |= !ok;
        const int64_t pp = ok ? pk : 0;
        const uint16_t *yrow;
        if (kRanked) {
          const int64_t r = pp / p.SK;
          yrow = p.rank_ys[r] + (pp - r * p.SK) * p.H;
        } else {
          yrow = p.y + pp * p.H;
        }
        const uint4 *row = reinterpret_cast<const uint4 *>(yrow);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = cbase + u * 32;
          v[k][u] = (ok && c < p.chunks) ? __ldcs(row + c) : make_uint4(0, 0, 0, 0);
        }
      }
    }
    float acc[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[u][j] = 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const float wk = __shfl_sync(0xffffffffu, wt, k);
      if (k < p.K) {
#pragma unroll
        for (int u = 0; u < U; ++u) fma8(acc[u], wk, v[k][u]);
      }
    }
    uint4 *orow = reinterpret_cast<uint4 *>(p.out + g * p.H);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = cbase + u * 32;
      if (c < p.chunks) __stcs(orow + c, pack8(acc[u]));
    }
    sl = nsl;
    wt = nwt;
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

template <int KC>
cudaError_t launch_kc(CombineParams p, int sms, cudaStream_t stream) {
  constexpr int U0 = (MEP_COMBINE_LOADS / KC) > 0 ? (MEP_COMBINE_LOADS / KC) : 1;
  constexpr int U = U0 < MEP_COMBINE_MAX_U ? U0 : MEP_COMBINE_MAX_U;
  p.parts = (p.chunks + 32 * U - 1) / (32 * U);
  const int64_t ntask = p.N * p.parts;
  const int64_t want = (ntask + kWarps - 1) / kWarps;
  const int blocks = (int)std::max<int64_t>(
      1, std::min<int64_t>(want, (int64_t)sms * MEP_COMBINE_BLOCKS_PER_SM));
  if (p.rank_ys != nullptr)
    combine_kernel<KC, U, true><<<blocks, kThreads, 0, stream>>>(p);
  else
    combine_kernel<KC, U, false><<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                           const uint16_t *y, const uint16_t *const *rank_ys, const float *w,
                           uint16_t *out, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  CombineParams p{};
  p.y = y;
  p.rank_ys = rank_ys;
  p.SK = (int64_t)s.S * s.K;
  p.w = w;
  p.slot = pl.slot;
  p.out = out;
  p.status = pl.status;
  p.N = (int64_t)s.R * s.S;
  p.NK = p.N * s.K;
  p.K = s.K;
  p.H = H;
  p.chunks = H / 8;
  if (s.K <= 2) return launch_kc<2>(p, sms, stream);
  if (s.K <= 4) return launch_kc<4>(p, sms, stream);
  if (s.K <= 8) return launch_kc<8>(p, sms, stream);
  return launch_kc<16>(p, sms, stream);
}

}  // namespace mep
