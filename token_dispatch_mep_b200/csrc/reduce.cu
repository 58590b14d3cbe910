// Backward reduction of replica weight-gradients into their home expert:
//   home[e, :] = sum over expert e's segments s (ascending) of G[s, :]
// in float32, zero for an expert with no segment.
//
// Method: during the backward pass the gradients of an expert's duplicates are
// summed into the copy on its home rank (MoonEP release page, "How MoonEP
// works").  The plan lists an expert's segments contiguously
// (expert_seg_ptr), so the reduction is a segmented sum over contiguous rows
// of G.
//
// A task is one (expert, column tile) pair; a tile is kThreads x kU vectors
// of one row, so each thread owns kU vectors spaced kThreads apart (every
// warp access is a contiguous 512-byte run).  Blocks stride over tasks,
// expert-major; the segment range is read once per task.  A thread issues
// the kU loads of kSU segment rows before adding them, in segment order.  G is read once and home written once,
// both with streaming (evict-first) accesses.  The segment pointers are read
// on the device and bounds-checked; nothing is sized from a host copy of the
// plan.
#include <algorithm>
#include <cstdint>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_REDUCE_U
#define MEP_REDUCE_U 4
#endif
#ifndef MEP_REDUCE_BLOCKS_PER_SM
#define MEP_REDUCE_BLOCKS_PER_SM 1024
#endif
#ifndef MEP_REDUCE_MIN_BLOCKS
#define MEP_REDUCE_MIN_BLOCKS 3  // launch bound: resident blocks per SM
#endif
#ifndef MEP_REDUCE_SEG_UNROLL
#define MEP_REDUCE_SEG_UNROLL 2  // segment rows in flight per thread
#endif

namespace mep {

namespace {

constexpr int kThreads = 256;
constexpr int kU = MEP_REDUCE_U;
constexpr int kSU = MEP_REDUCE_SEG_UNROLL;

struct ReduceParams {
  const float *G;
  float *home;
  const int32_t *eptr;
  int32_t *status;
  int32_t E;
  int32_t rows;   // E + R - 1
  int64_t cols;   // P / 4 (vector path) or P (scalar path)
};

template <typename V>
__device__ __forceinline__ V zero_v();
template <>
__device__ __forceinline__ float4 zero_v<float4>() { return make_float4(0.f, 0.f, 0.f, 0.f); }
template <>
__device__ __forceinline__ float zero_v<float>() { return 0.f; }

__device__ __forceinline__ float4 addv(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float addv(float a, float b) { return a + b; }

template <typename V>
__global__ void __launch_bounds__(kThreads, MEP_REDUCE_MIN_BLOCKS) reduce_kernel(ReduceParams p) {
  const V *G = reinterpret_cast<const V *>(p.G);
  V *home = reinterpret_cast<V *>(p.home);
  const int64_t tile = (int64_t)kThreads * kU;
  const int64_t tiles_per_e = (p.cols + tile - 1) / tile;
  const int64_t ntask = (int64_t)p.E * tiles_per_e;
  bool bad = false;
  for (int64_t task = blockIdx.x; task < ntask; task += gridDim.x) {
    const int e = (int)(task / tiles_per_e);
    const int64_t c0 = (task - (int64_t)e * tiles_per_e) * tile + threadIdx.x;
    int s0 = __ldg(p.eptr + e), s1 = __ldg(p.eptr + e + 1);
    if (s0 < 0 || s1 < s0 || s1 > p.rows) {
      bad = true;
      s0 = s1 = 0;
    }
    V acc[kU];
#pragma unroll
    for (int j = 0; j < kU; ++j) acc[j] = zero_v<V>();
    int s = s0;
    for (; s + kSU <= s1; s += kSU) {
      V a[kSU][kU];
#pragma unroll
      for (int q = 0; q < kSU; ++q) {
        const V *row = G + (int64_t)(s + q) * p.cols;
#pragma unroll
        for (int j = 0; j < kU; ++j) {
          const int64_t c = c0 + (int64_t)j * kThreads;
          if (c < p.cols) a[q][j] = __ldcs(row + c);
        }
      }
#pragma unroll
      for (int q = 0; q < kSU; ++q)
#pragma unroll
        for (int j = 0; j < kU; ++j)
          if (c0 + (int64_t)j * kThreads < p.cols) acc[j] = addv(acc[j], a[q][j]);
    }
    for (; s < s1; ++s) {
      const V *row = G + (int64_t)s * p.cols;
      V a[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int64_t c = c0 + (int64_t)j * kThreads;
        if (c < p.cols) a[j] = __ldcs(row + c);
      }
#pragma unroll
      for (int j = 0; j < kU; ++j)
        if (c0 + (int64_t)j * kThreads < p.cols) acc[j] = addv(acc[j], a[j]);
    }
    V *hrow = home + (int64_t)e * p.cols;
#pragma unroll
    for (int j = 0; j < kU; ++j) {
      const int64_t c = c0 + (int64_t)j * kThreads;
      if (c < p.cols) __stcs(hrow + c, acc[j]);
    }
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

}  // namespace

cudaError_t launch_reduce(const mep_shape_t &s, const mep_plan_t &pl, int64_t P,
                          const float *G, float *home, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  ReduceParams p{};
  p.G = G;
  p.home = home;
  p.eptr = pl.expert_seg_ptr;
  p.status = pl.status;
  p.E = s.E;
  p.rows = s.E + s.R - 1;
  const bool vec = (P % 4) == 0;
  p.cols = vec ? P / 4 : P;
  const int64_t tile = (int64_t)kThreads * kU;
  const int64_t ntask = (int64_t)s.E * ((p.cols + tile - 1) / tile);
  const int blocks =
      (int)std::max<int64_t>(1, std::min<int64_t>(ntask, (int64_t)sms * MEP_REDUCE_BLOCKS_PER_SM));
  if (vec)
    reduce_kernel<float4><<<blocks, kThreads, 0, stream>>>(p);
  else
    reduce_kernel<float><<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mep
