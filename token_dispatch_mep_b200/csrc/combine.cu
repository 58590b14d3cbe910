// Weighted combine back to token order:
//   out[g, :] = bf16_rne( sum_{k=0..K-1} w[g,k] * y[slot[g,k], :] )
// accumulated in float32 with one fused multiply-add per term, k ascending.
//
// Method: a router assigns every token to K experts (MoonEP release page,
// "Why expert parallelism is needed"); the K expert outputs return to the
// token's position, weighted by the router weights.
//
// Each thread owns one 16-byte column chunk (8 bf16) of one token: it loads
// the token's K slot ids and weights (shared by the warp, served by L1), then
// issues the K independent 16-byte row loads before it touches any of them,
// so K x 16 bytes per thread are in flight.  Expert outputs are read once
// (streaming loads); the output row is written once (streaming stores).
#include <algorithm>
#include <cstdint>

#include <cuda_bf16.h>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

constexpr int kThreads = 256;

struct CombineParams {
  const uint16_t *y;
  const float *w;
  const int32_t *slot;
  uint16_t *out;
  int32_t *status;
  int64_t NK;
  int32_t K, H;
  uint32_t chunks_per_row;  // H / 8
  uint64_t items;           // N * H / 8
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

template <int KC>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineParams p) {
  const uint64_t stride = (uint64_t)gridDim.x * kThreads;
  bool bad = false;
  for (uint64_t it = (uint64_t)blockIdx.x * kThreads + threadIdx.x; it < p.items; it += stride) {
    const uint64_t g = it / p.chunks_per_row;
    const uint32_t c = (uint32_t)(it - g * p.chunks_per_row);
    int pk[KC];
    float wk[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      if (k < p.K) {
        pk[k] = __ldg(p.slot + g * p.K + k);
        wk[k] = __ldg(p.w + g * p.K + k);
      }
    }
    uint4 v[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      if (k < p.K) {
        if ((unsigned)pk[k] < (unsigned)p.NK) {
          v[k] = __ldcs(reinterpret_cast<const uint4 *>(p.y + (int64_t)pk[k] * p.H) + c);
        } else {
          v[k] = make_uint4(0, 0, 0, 0);
          bad = true;
        }
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < KC; ++k)
      if (k < p.K) fma8(acc, wk[k], v[k]);
    __stcs(reinterpret_cast<uint4 *>(p.out + g * p.H) + c, pack8(acc));
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

template <int KC>
cudaError_t launch_kc(const CombineParams &p, int blocks, cudaStream_t stream) {
  combine_kernel<KC><<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                           const uint16_t *y, const float *w, uint16_t *out,
                           cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  CombineParams p{};
  p.y = y;
  p.w = w;
  p.slot = pl.slot;
  p.out = out;
  p.status = pl.status;
  const int64_t N = (int64_t)s.R * s.S;
  p.NK = N * s.K;
  p.K = s.K;
  p.H = H;
  p.chunks_per_row = (uint32_t)(H / 8);
  p.items = (uint64_t)N * p.chunks_per_row;
  const uint64_t want = (p.items + kThreads - 1) / kThreads;
  const int blocks = (int)std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)sms * 8));
  if (s.K <= 2) return launch_kc<2>(p, blocks, stream);
  if (s.K <= 4) return launch_kc<4>(p, blocks, stream);
  if (s.K <= 8) return launch_kc<8>(p, blocks, stream);
  return launch_kc<16>(p, blocks, stream);
}

}  // namespace mep
