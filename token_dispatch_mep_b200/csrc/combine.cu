// Weighted combine back to token order:
//   out[g, :] = bf16_rne( sum_{k=0..K-1} w[g,k] * y[slot[g,k], :] )
// accumulated in float32 with one fused multiply-add per term, k ascending.
//
// Method: a router assigns every token to K experts (MoonEP release page,
// "Why expert parallelism is needed"); the K expert outputs return to the
// token's position, weighted by the router weights.
//
// One warp per token walks the row, kRU = 2 16-byte chunks (8 bf16 each) per
// lane per step.  Lanes k < K hold the token's slot id and weight, which the
// warp broadcasts with shuffles.  The K expert-output chunks are loaded in
// groups of 8 (all loads of a group issued before any use) and added in k
// order with one float32 FMA each, so every output is the same k-ordered
// float32 sum whatever the grouping; the sum is rounded to bf16 and written
// with a streaming 16-byte store.  Expert outputs are read once (streaming
// loads).  The grid has one warp per token, in blocks of two warps: small
// blocks keep the last wave short (1 % over blocks of eight warps).  A form
// with warp tasks over parts of rows and all K loads in flight measured
// 0.90-1.00 of the HBM copy peak against 0.96-1.04 for this one.
//
// Rank-addressed form (mep_combine_ranked): expert outputs are read from R
// separate rank buffers, slot p being row p % SK of rank_ys[p / SK]; a NULL
// or misaligned rank pointer is reported, never used.  A token range [g0, g0
// + N) restricts the kernel to one rank's own tokens (out and w rows are the
// range's; mep_combine_ranked_tokens).
//
// With no weights (w == nullptr) every weight is 1 and the kernel is the
// backward of dispatch: grad_x[g] = bf16(sum_k grad_buf[slot[g,k]]) (an FMA
// with weight 1 rounds exactly like an addition).
#include <algorithm>
#include <cstdint>

#include <cuda_bf16.h>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_COMBINE_MIN_BLOCKS
#define MEP_COMBINE_MIN_BLOCKS 8  // launch bound: resident blocks per SM
#endif
#ifndef MEP_COMBINE_ROW_U
#define MEP_COMBINE_ROW_U 2  // 16-byte chunks per lane per step
#endif

namespace mep {

namespace {

constexpr int kThreads = 64;  // two token rows per block
constexpr int kWarps = kThreads / 32;

struct CombineParams {
  const uint16_t *y;
  const uint16_t *const *rank_ys;  // ranked form: R row buffers of SK rows
  int64_t SK;
  const float *w;
  const int32_t *slot;
  uint16_t *out;
  int32_t *status;
  int64_t g0;     // first token (global order); out / w row i is token g0 + i
  int64_t N, NK;  // tokens processed, slots of the plan
  int32_t K, H;
  int32_t chunks;      // 16-byte chunks per row = H / 8
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

template <int KC, bool kRanked>
__global__ void __launch_bounds__(kThreads, MEP_COMBINE_MIN_BLOCKS) combine_row_kernel(CombineParams p) {
  constexpr int KG = KC < 8 ? KC : 8;
  constexpr int kRU = MEP_COMBINE_ROW_U;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  bool bad = false;
  for (int64_t g = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); g < p.N; g += nwarps) {
    int sl = lane < p.K ? __ldg(p.slot + (p.g0 + g) * p.K + lane) : -1;
    const float wt = lane < p.K ? (p.w != nullptr ? __ldg(p.w + g * p.K + lane) : 1.f) : 0.f;
    if (lane < p.K && (unsigned)sl >= (unsigned)p.NK) {
      bad = true;
      sl = -1;
    }
    const unsigned okmask = __ballot_sync(0xffffffffu, sl >= 0);
    uint4 *orow = reinterpret_cast<uint4 *>(p.out + g * p.H);
    for (int c0 = 0; c0 < p.chunks; c0 += 32 * kRU) {
      float acc[kRU][8];
#pragma unroll
      for (int u = 0; u < kRU; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
#pragma unroll
      for (int kg = 0; kg < KC; kg += KG) {
        uint4 v[KG][kRU];
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          const int pk = __shfl_sync(0xffffffffu, sl, kg + j);
          bool ok = ((okmask >> (kg + j)) & 1) && (unsigned)pk < (unsigned)p.NK;
          const int64_t pp = ok ? pk : 0;
          const uint16_t *yrow;
          if (kRanked) {
            // a rank buffer must be present and 16-byte aligned
            const int64_t r = pp / p.SK;
            const uint16_t *base = p.rank_ys[r];
            if (base == nullptr || (reinterpret_cast<uintptr_t>(base) & 15) != 0) {
              if (ok) bad = true;
              ok = false;
            }
            yrow = base + (pp - r * p.SK) * p.H;
          } else {
            yrow = p.y + pp * p.H;
          }
#pragma unroll
          for (int u = 0; u < kRU; ++u) {
            const int c = c0 + u * 32 + lane;
            v[j][u] = (ok && c < p.chunks) ? __ldcs(reinterpret_cast<const uint4 *>(yrow) + c)
                                           : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          const float wk = __shfl_sync(0xffffffffu, wt, kg + j);
          if ((okmask >> (kg + j)) & 1) {
#pragma unroll
            for (int u = 0; u < kRU; ++u) fma8(acc[u], wk, v[j][u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kRU; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < p.chunks) __stcs(orow + c, pack8(acc[u]));
      }
    }
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

template <int KC>
cudaError_t launch_kc(const CombineParams &p, int sms, cudaStream_t stream) {
  const int64_t want = (p.N + kWarps - 1) / kWarps;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 1024));
  if (p.rank_ys != nullptr)
    combine_row_kernel<KC, true><<<blocks, kThreads, 0, stream>>>(p);
  else
    combine_row_kernel<KC, false><<<blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const mep_shape_t &s, int32_t H, const mep_plan_t &pl, int64_t g0,
                           int64_t count, const uint16_t *y, const uint16_t *const *rank_ys,
                           const float *w, uint16_t *out, cudaStream_t stream) {
  if (count <= 0) return cudaSuccess;
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
  p.g0 = g0;
  p.N = count;
  p.NK = (int64_t)s.R * s.S * s.K;
  p.K = s.K;
  p.H = H;
  p.chunks = H / 8;
  if (s.K <= 2) return launch_kc<2>(p, sms, stream);
  if (s.K <= 4) return launch_kc<4>(p, sms, stream);
  if (s.K <= 8) return launch_kc<8>(p, sms, stream);
  return launch_kc<16>(p, sms, stream);
}

}  // namespace mep
