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
// Flat grid-stride over (expert, column) items, expert-major, so consecutive
// threads read consecutive 16-byte columns.  Each thread issues up to eight
// segment-row loads before adding them, in segment order.  G is read once and
// home written once, both streaming.  The segment pointers are read on the
// device and bounds-checked; nothing is sized from a host copy of the plan.
#include <algorithm>
#include <cstdint>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

constexpr int kThreads = 256;
constexpr int kBatch = 8;

struct ReduceParams {
  const float *G;
  float *home;
  const int32_t *eptr;
  int32_t *status;
  int32_t E;
  int32_t rows;   // E + R - 1
  int64_t cols;   // P / 4 (vector path) or P (scalar path)
};

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

template <typename V>
__device__ __forceinline__ V zero_v();
template <>
__device__ __forceinline__ float4 zero_v<float4>() { return make_float4(0.f, 0.f, 0.f, 0.f); }
template <>
__device__ __forceinline__ float zero_v<float>() { return 0.f; }

__device__ __forceinline__ float4 addv(float4 a, float4 b) { return add4(a, b); }
__device__ __forceinline__ float addv(float a, float b) { return a + b; }

template <typename V>
__global__ void __launch_bounds__(kThreads) reduce_kernel(ReduceParams p) {
  const V *G = reinterpret_cast<const V *>(p.G);
  V *home = reinterpret_cast<V *>(p.home);
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  int64_t start = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  int e = (int)(start / p.cols);
  int64_t i = start - (int64_t)e * p.cols;
  const int64_t step_e = stride / p.cols, step_i = stride - step_e * p.cols;
  bool bad = false;
  while (e < p.E) {
    int s0 = __ldg(p.eptr + e), s1 = __ldg(p.eptr + e + 1);
    if (s0 < 0 || s1 < s0 || s1 > p.rows) {
      bad = true;
      s0 = s1 = 0;
    }
    V acc = zero_v<V>();
    for (int s = s0; s < s1; s += kBatch) {
      V v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (s + u < s1) v[u] = __ldcs(G + (int64_t)(s + u) * p.cols + i);
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (s + u < s1) acc = addv(acc, v[u]);
    }
    __stcs(home + (int64_t)e * p.cols + i, acc);
    e += (int)step_e;
    i += step_i;
    if (i >= p.cols) {
      i -= p.cols;
      e += 1;
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
  const int64_t items = (int64_t)s.E * p.cols;
  const int64_t want = (items + kThreads - 1) / kThreads;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
  if (vec)
    reduce_kernel<float4><<<blocks, kThreads, 0, stream>>>(p);
  else
    reduce_kernel<float><<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mep
