// Backward of combine: the adjoint of out[g] = sum_k w[g,k] * y[slot[g,k]].
//   grad_y[slot[g,k], :] = bf16( w[g,k] * grad_out[g, :] )     correctly rounded
//   grad_w[g, k]         = sum_h grad_out[g, h] * y[slot[g,k], h]  (float32)
//
// Method: the training step has a backward pass (MoonEP release page, "How
// MoonEP works"); the gradient of the weighted combine goes to every slot
// scaled by its router weight and to every router weight as the dot product
// of the output gradient with the slot's expert output.
//
// One warp per token walks the row once, kU 16-byte chunks per lane per step
// (lane l owns chunks l, l+32, ...): it loads the output-gradient chunks and
// the K expert-output chunks (all issued before use), accumulates the K partial dot
// products in float32 FMAs, and stores the K scaled chunks.  The K partial
// dots are summed across the warp with a fixed butterfly, so runs are
// bit-identical.  The scaled gradient is rounded once: the float32 product is
// taken toward zero and its last bit set when inexact (round-to-odd, Boldo &
// Melquiond 2008), then rounded to nearest-even bf16; with 16 extra bits this
// equals rounding the exact product.
#include <algorithm>
#include <cstdint>

#include <cuda_bf16.h>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_COMBINE_BWD_BLOCKS_PER_SM
#define MEP_COMBINE_BWD_BLOCKS_PER_SM 1024  // grid cap in multiples of the SM count
#endif
#ifndef MEP_COMBINE_BWD_U
#define MEP_COMBINE_BWD_U 2  // 16-byte chunks per lane per iteration
#endif

namespace mep {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kU = MEP_COMBINE_BWD_U;

struct CombineBwdParams {
  const uint16_t *grad_out;
  const float *w;
  const uint16_t *y;
  const int32_t *slot;
  uint16_t *grad_y;
  float *grad_w;
  int32_t *status;
  int64_t N, NK;
  int32_t K, H;
  int32_t chunks;  // H / 8
};

// w * g rounded once to bf16 (round-to-odd float32 product, then RNE).
__device__ __forceinline__ float product_rto(float w, float g) {
  const float pz = __fmul_rz(w, g);
  const float r = __fmaf_rn(w, g, -pz);  // exact residual of the product
  return (r != 0.f && isfinite(pz)) ? __uint_as_float(__float_as_uint(pz) | 1u) : pz;
}

__device__ __forceinline__ uint4 scale8(float wk, const float (&gf)[8]) {
  uint32_t u[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const __nv_bfloat162 b =
        __floats2bfloat162_rn(product_rto(wk, gf[2 * j]), product_rto(wk, gf[2 * j + 1]));
    u[j] = *reinterpret_cast<const uint32_t *>(&b);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(u[j] << 16);
    f[2 * j + 1] = __uint_as_float(u[j] & 0xffff0000u);
  }
}

template <int KC>
__global__ void __launch_bounds__(kThreads) combine_bwd_kernel(CombineBwdParams p) {
  griddep_wait();  // the previous kernel on the stream is complete and visible
  constexpr int KG = KC < 8 ? KC : 8;  // expert-output chunks loaded together
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  bool bad = false;
  for (int64_t g = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); g < p.N; g += nwarps) {
    // lane k < K holds slot id and weight of (g, k)
    int sl = lane < p.K ? __ldg(p.slot + g * p.K + lane) : -1;
    const float wt = lane < p.K ? __ldg(p.w + g * p.K + lane) : 0.f;
    if (lane < p.K && (unsigned)sl >= (unsigned)p.NK) {
      bad = true;
      sl = -1;
    }
    const unsigned okmask = __ballot_sync(0xffffffffu, sl >= 0);
    float dot[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) dot[k] = 0.f;
    const uint4 *gorow = reinterpret_cast<const uint4 *>(p.grad_out + g * p.H);
    // Warp-uniform loop over the row (every lane runs every iteration, so the
    // shuffles below always see the full warp); memory accesses are
    // predicated on the lane's chunk being inside the row.
    for (int c0 = 0; c0 < p.chunks; c0 += 32 * kU) {
      float gf[kU][8];
      bool in_row[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * 32 + lane;
        in_row[u] = c < p.chunks;
        unpack8(in_row[u] ? __ldcs(gorow + c) : make_uint4(0, 0, 0, 0), gf[u]);
      }
#pragma unroll
      for (int kg = 0; kg < KC; kg += KG) {
        uint4 yv[KG][kU];
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          const int pk = __shfl_sync(0xffffffffu, sl, kg + j);
          const bool ok = ((okmask >> (kg + j)) & 1) && (unsigned)pk < (unsigned)p.NK;
          const uint4 *yrow = reinterpret_cast<const uint4 *>(p.y + (int64_t)(ok ? pk : 0) * p.H);
#pragma unroll
          for (int u = 0; u < kU; ++u)
            yv[j][u] = (ok && in_row[u]) ? __ldcs(yrow + c0 + u * 32 + lane) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          const int k = kg + j;
          const int pk = __shfl_sync(0xffffffffu, sl, k);
          const float wk = __shfl_sync(0xffffffffu, wt, k);
          if (((okmask >> k) & 1) && (unsigned)pk < (unsigned)p.NK) {
            uint4 *gyrow = reinterpret_cast<uint4 *>(p.grad_y + (int64_t)pk * p.H);
#pragma unroll
            for (int u = 0; u < kU; ++u) {
              if (in_row[u]) {
                float yf[8];
                unpack8(yv[j][u], yf);
#pragma unroll
                for (int e = 0; e < 8; ++e) dot[k] = __fmaf_rn(gf[u][e], yf[e], dot[k]);
                __stcs(gyrow + c0 + u * 32 + lane, scale8(wk, gf[u]));
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      float d = dot[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (k < p.K && lane == k) p.grad_w[g * p.K + k] = d;
    }
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

template <int KC>
cudaError_t launch_kc(const CombineBwdParams &p, int sms, cudaStream_t stream) {
  const int64_t want = (p.N + kWarps - 1) / kWarps;
  const int blocks = (int)std::max<int64_t>(
      1, std::min<int64_t>(want, (int64_t)sms * MEP_COMBINE_BWD_BLOCKS_PER_SM));
  return launch_pdl(combine_bwd_kernel<KC>, dim3(blocks), dim3(kThreads), 0, stream, p);
}

}  // namespace

cudaError_t launch_combine_backward(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                                    const uint16_t *grad_out, const float *w, const uint16_t *y,
                                    uint16_t *grad_y, float *grad_w, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  CombineBwdParams p{};
  p.grad_out = grad_out;
  p.w = w;
  p.y = y;
  p.slot = pl.slot;
  p.grad_y = grad_y;
  p.grad_w = grad_w;
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
