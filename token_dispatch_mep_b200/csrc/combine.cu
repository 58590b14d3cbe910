// Weighted combine back to token order:
//   out[g, :] = bf16_rne( sum_{k=0..K-1} w[g,k] * y[slot[g,k], :] )
// with the K terms added in binary64, k ascending, and the sum rounded once.
//
// Method: a router assigns every token to K experts (MoonEP release page,
// "Why expert parallelism is needed"); the K expert outputs return to the
// token's position, weighted by the router weights.
//
// Arithmetic.  A float32 weight times a bf16 value has at most 24 + 8
// significant bits, so every product is exact in binary64, and a chain of
// binary64 fused multiply-adds in k order, acc = fma(w_k, y_k, acc), rounds
// exactly like adding the exact products one by one.  The sum is then
// rounded once to bf16 (round to nearest, ties to even), so the result is the
// correctly rounded value of the k-ordered binary64 sum -- whatever the
// cancellation between terms.  A float32 accumulator could not promise that:
// under cancellation its rounding errors can move the result by several bf16
// units.  The kernel stays bound by HBM bandwidth: about five integer or FP64
// instructions per 2-byte element read.
//   bf16 -> binary64 without a conversion instruction: the bf16 bits b placed
//   as the top of a binary64 word -- sign to bit 63, the 8 exponent bits to
//   the low end of the 11-bit exponent field, the 7 fraction bits to the top
//   of the fraction -- give exactly y * 2^-896 for every finite y (zero and
//   subnormals included: the two formats' subnormal scales differ by the same
//   2^-896), and the weight is scaled by 2^896 once per term (exact: a float32
//   times 2^896 stays below 2^1024).  Infinities and NaNs do not survive this
//   mapping, so every loaded word's exponent fields are folded into a running
//   16x2 maximum (one instruction per two elements; an all-ones exponent is
//   the largest); a chunk that held one is summed again with exact
//   conversions (the oracle's arithmetic: inf and NaN propagate).  Measured
//   against the alternatives (float32 -> binary64 conversion instructions;
//   one chunk per lane with more resident warps), this form moved the most
//   bytes on every workload.
//
// One warp per token walks the row, kRU = 2 16-byte chunks (8 bf16 each) per
// lane per step.  Lanes k < K hold the token's slot id and weight, which the
// warp broadcasts with shuffles.  The K expert-output chunks are loaded in
// groups of 8 (all loads of a group issued before any use) and accumulated in
// k order; the sum is rounded to bf16 and written with a streaming 16-byte
// store.  Expert outputs are read once (streaming loads).  The kernel is
// instantiated for K up to 2, 4, 6, 8 and 16 terms: a warp's loads in flight
// are held in registers, so an instantiation no wider than K leaves room for
// more resident warps (for K = 6: a launch bound of 9 blocks per SM, which
// the compiler meets with 96 registers -- 10 resident blocks, against 8 for
// the K = 8 form -- measured 0.96 of the copy peak against 0.92; bounds of 8
// and 10 measured 0.93 and 0.95).  The grid has one
// warp per token, in blocks of two warps: small blocks keep the last wave
// short (1 % over blocks of eight warps).  A form with warp tasks over parts
// of rows and all K loads in flight measured 0.90-1.00 of the HBM copy peak
// against 0.96-1.04 for this one.
//
// Rank-addressed form (mep_combine_ranked): expert outputs are read from R
// separate rank buffers, slot p being row p % SK of rank_ys[p / SK]; a NULL
// or misaligned rank pointer is reported, never used.  Each token's K row
// addresses are resolved once into shared memory and read there by
// broadcast (resolving them at every step, or holding them in registers,
// measured 0.77-0.82 of the copy peak against 0.96-1.01 this way).  A token range [g0, g0
// + N) restricts the kernel to one rank's own tokens (out and w rows are the
// range's; mep_combine_ranked_tokens).
//
// With no weights (w == nullptr) every weight is 1 and the kernel is the
// backward of dispatch: grad_x[g] = bf16(sum_k grad_buf[slot[g,k]]), the same
// binary64 sum rounded once.
#include <algorithm>
#include <cstdint>

#include <cuda_bf16.h>

#include "mep_device.cuh"
#include "mep_internal.h"

#ifndef MEP_COMBINE_MIN_BLOCKS
#define MEP_COMBINE_MIN_BLOCKS 8  // launch bound: resident blocks per SM
#endif
#ifndef MEP_COMBINE_K6
#define MEP_COMBINE_K6 1  // 1: a K <= 6 instantiation (loads and registers for 6 terms)
#endif
#ifndef MEP_COMBINE_MIN_BLOCKS_K6
#define MEP_COMBINE_MIN_BLOCKS_K6 9  // its launch bound (blocks per SM)
#endif
#ifndef MEP_COMBINE_ROW_U
#define MEP_COMBINE_ROW_U 2  // 16-byte chunks per lane per step
#endif
#ifndef MEP_COMBINE_GROUP
#define MEP_COMBINE_GROUP 8  // expert-output loads issued together (k values per group)
#endif
#ifndef MEP_COMBINE_NF_MAX
#define MEP_COMBINE_NF_MAX 1  // 1: non-finite check by a 16x2 max of the exponents
#endif
#ifndef MEP_COMBINE_CVT
#define MEP_COMBINE_CVT 0  // 1: bf16 -> float32 -> binary64 by conversion instructions
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

constexpr double kTwo896 = 0x1p896;  // scale of the integer bf16 -> binary64 mapping

// Binary64 word whose value is y * 2^-896 for the bf16 y held in the top half
// of `x` (the low 16 bits of x are ignored): the sign stays at bit 31 of the
// high word, the arithmetic shift moves the exponent to bits 20..27 and the
// fraction to bits 13..19, and the mask clears the sign copies in bits 28..30
// and the low bits.
__device__ __forceinline__ double bf16_hi_to_scaled_f64(uint32_t x) {
  return __hiloint2double((int)(((int32_t)x >> 3) & (int32_t)0x8fffe000u), 0);
}

#if !MEP_COMBINE_NF_MAX
// Nonzero in bit 15 or 31 if a bf16 half of u has an all-ones exponent
// (infinity or NaN): the masked, inverted exponent of such a half is zero, and
// subtracting 1 from it sets the half's top bit (no other half value, all
// multiples of 0x80 below 0x8000, reaches it).
__device__ __forceinline__ uint32_t nonfinite_bits(uint32_t u) {
  return ((~u) & 0x7f807f80u) - 0x00010001u;
}
#endif

#if MEP_COMBINE_NF_MAX
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
#endif

// acc[j] = fma(ws, y_j * 2^-896, acc[j]) for the 8 bf16 of v (ws = w * 2^896),
// in element order; *nf collects the non-finite check of the loaded words.
__device__ __forceinline__ void fma8(double (&acc)[8], double ws, const uint4 &v, uint32_t *nf) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#if MEP_COMBINE_CVT
    (void)nf;
    acc[2 * j] = __fma_rn(ws, (double)__uint_as_float(u[j] << 16), acc[2 * j]);
    acc[2 * j + 1] = __fma_rn(ws, (double)__uint_as_float(u[j] & 0xffff0000u), acc[2 * j + 1]);
#else
#if MEP_COMBINE_NF_MAX
    *nf = max_u16x2(*nf, u[j] & 0x7f807f80u);
#else
    *nf |= nonfinite_bits(u[j]);
#endif
    acc[2 * j] = __fma_rn(ws, bf16_hi_to_scaled_f64(u[j] << 16), acc[2 * j]);
    acc[2 * j + 1] = __fma_rn(ws, bf16_hi_to_scaled_f64(u[j]), acc[2 * j + 1]);
#endif
  }
}

// Nonzero if the collected check saw an infinity or NaN.
__device__ __forceinline__ bool saw_nonfinite(uint32_t nf) {
#if MEP_COMBINE_CVT
  (void)nf;
  return false;
#elif MEP_COMBINE_NF_MAX
  return (nf & 0xffffu) == 0x7f80u || (nf >> 16) == 0x7f80u;
#else
  return (nf & 0x80008000u) != 0;
#endif
}

// The same sum with exact conversions (no scaling): infinities and NaNs
// propagate as in binary64 arithmetic.
__device__ __forceinline__ void fma8_exact(double (&acc)[8], double w, const uint4 &v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc[2 * j] = __fma_rn(w, (double)__uint_as_float(u[j] << 16), acc[2 * j]);
    acc[2 * j + 1] = __fma_rn(w, (double)__uint_as_float(u[j] & 0xffff0000u), acc[2 * j + 1]);
  }
}

__device__ __forceinline__ uint4 pack8(const double (&acc)[8]) {
  uint32_t u[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = __bfloat16_as_ushort(__double2bfloat16(acc[2 * j]));
    const uint32_t hi = __bfloat16_as_ushort(__double2bfloat16(acc[2 * j + 1]));
    u[j] = lo | (hi << 16);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

// Row address of slot pp (ranked form: row pp % SK of rank pp / SK's buffer);
// clears *ok (and flags *bad if *ok was set) when a rank buffer is missing or
// misaligned.
template <bool kRanked>
__device__ __forceinline__ const uint16_t *slot_row(const CombineParams &p, int64_t pp, bool *ok,
                                                    bool *bad) {
  if (kRanked) {
    const int64_t r = pp / p.SK;
    const uint16_t *base = p.rank_ys[r];
    if (base == nullptr || (reinterpret_cast<uintptr_t>(base) & 15) != 0) {
      if (*ok) *bad = true;
      *ok = false;
    }
    return base + (pp - r * p.SK) * p.H;
  }
  return p.y + pp * p.H;
}

template <int KC, bool kRanked>
__global__ void __launch_bounds__(kThreads, KC == 6 ? MEP_COMBINE_MIN_BLOCKS_K6 : MEP_COMBINE_MIN_BLOCKS)
    combine_row_kernel(CombineParams p) {
  griddep_wait();  // the previous kernel on the stream is complete and visible
  __shared__ const uint16_t *s_rows[kRanked ? kWarps : 1][kRanked ? KC : 1];  // ranked: the K rows
  constexpr int KG = KC < MEP_COMBINE_GROUP ? KC : MEP_COMBINE_GROUP;
  // Groups tile the K terms exactly: a partial last group would read row
  // pointers past the token's KC entries.
  static_assert(KC % KG == 0, "load groups must divide the instantiated term count");
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
#if MEP_COMBINE_CVT
    const double wts = (double)wt;
#else
    const double wts = (double)wt * kTwo896;  // exact
#endif
    const unsigned okmask = __ballot_sync(0xffffffffu, sl >= 0);
    // Ranked form: lane k < K resolves its slot's rank buffer and row once
    // per token (a division and the pointer checks) into shared memory, which
    // the warp reads by broadcast at every step (NULL: no row to read).
    if (kRanked) {
      __syncwarp();  // the previous token's rows are no longer read
      if (lane < KC) {
        bool ok = sl >= 0;
        const uint16_t *row = ok ? slot_row<true>(p, sl, &ok, &bad) : nullptr;
        s_rows[threadIdx.x >> 5][lane] = ok ? row : nullptr;
      }
      __syncwarp();
    }
    uint4 *orow = reinterpret_cast<uint4 *>(p.out + g * p.H);
    for (int c0 = 0; c0 < p.chunks; c0 += 32 * kRU) {
      double acc[kRU][8];
#pragma unroll
      for (int u = 0; u < kRU; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[u][e] = 0.0;
      uint32_t nf = 0;
#pragma unroll
      for (int kg = 0; kg < KC; kg += KG) {
        uint4 v[KG][kRU];
#pragma unroll
        for (int j = 0; j < KG; ++j) {
          bool ok;
          const uint16_t *yrow;
          if (kRanked) {
            yrow = s_rows[threadIdx.x >> 5][kg + j];
            ok = yrow != nullptr;
          } else {
            const int pk = __shfl_sync(0xffffffffu, sl, kg + j);
            ok = ((okmask >> (kg + j)) & 1) && (unsigned)pk < (unsigned)p.NK;
            yrow = slot_row<false>(p, ok ? pk : 0, &ok, &bad);
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
          const double wk = __shfl_sync(0xffffffffu, wts, kg + j);
          if ((okmask >> (kg + j)) & 1) {
#pragma unroll
            for (int u = 0; u < kRU; ++u) fma8(acc[u], wk, v[j][u], &nf);
          }
        }
      }
      // A chunk with an infinity or NaN among its inputs: sum it again with
      // exact conversions (rare; warp-uniform branch, the shuffles need every
      // lane).
      const bool redo = saw_nonfinite(nf);
      if (__any_sync(0xffffffffu, redo)) {
#pragma unroll
        for (int u = 0; u < kRU; ++u)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (redo) acc[u][e] = 0.0;
        for (int k = 0; k < KC; ++k) {
          const int pk = __shfl_sync(0xffffffffu, sl, k);
          const double wk = (double)__shfl_sync(0xffffffffu, wt, k);
          bool ok = redo && k < p.K && ((okmask >> k) & 1) && (unsigned)pk < (unsigned)p.NK;
          const uint16_t *yrow;
          if (kRanked) {
            yrow = s_rows[threadIdx.x >> 5][k];
            ok = ok && yrow != nullptr;
          } else {
            bool ignored = false;
            yrow = slot_row<false>(p, ok ? pk : 0, &ok, &ignored);
          }
#pragma unroll
          for (int u = 0; u < kRU; ++u) {
            const int c = c0 + u * 32 + lane;
            if (ok && c < p.chunks)
              fma8_exact(acc[u], wk, __ldcs(reinterpret_cast<const uint4 *>(yrow) + c));
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
    return launch_pdl(combine_row_kernel<KC, true>, dim3(blocks), dim3(kThreads), 0, stream, p);
  return launch_pdl(combine_row_kernel<KC, false>, dim3(blocks), dim3(kThreads), 0, stream, p);
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
#if MEP_COMBINE_K6
  if (s.K <= 6) return launch_kc<6>(p, sms, stream);
#endif
  if (s.K <= 8) return launch_kc<8>(p, sms, stream);
  return launch_kc<16>(p, sms, stream);
}

}  // namespace mep
