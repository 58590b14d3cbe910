// Backward reduction of replica weight-gradients into their home expert:
//   home[e, :] = float32( sum over expert e's segments s (ascending) of G[s, :] )
// with the sum taken in binary64 and rounded once to float32 (nearest-even);
// zero for an expert with no segment.  Every float32 is exact in binary64, so
// the result is the correctly rounded value of the ascending binary64 sum,
// whatever the cancellation between rows (a float32 running sum can be far
// off its relative bound there).  The kernel stays bound by HBM bandwidth:
// one conversion and one FP64 add per float read.
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
// the kU loads of kSU segment rows before adding them, in segment order.
// kU = 4, kSU = 1 and a launch bound of 4 blocks per SM (64 registers, 32
// resident warps) measured best on every workload (1.01-1.09 of the HBM copy
// peak), against 2 rows in flight with 3 blocks (80 registers: 0.97-1.01),
// 8 vectors per thread, and 5 or 6 blocks (which spill).  G
// is read once and home written once, both with streaming (evict-first)
// accesses.  The segment pointers are read on the device and bounds-checked;
// nothing is sized from a host copy of the plan.
//
// Rank-addressed form (mep_reduce_replica_grads_ranked): the gradients of a
// rank's segments live in that rank's own buffer (on a multi-GPU system, a
// peer buffer mapped into this GPU's address space), row j of rank r's
// buffer holding the j-th segment of rank r's list in slot order.  One home
// rank reduces its own E/R experts: for each task the block first resolves
// the expert's segments to row addresses (segment -> rank -> position in
// that rank's list, into shared memory), then sums exactly as above.
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
#define MEP_REDUCE_MIN_BLOCKS 4  // launch bound: resident blocks per SM
#endif
#ifndef MEP_REDUCE_SEG_UNROLL
#define MEP_REDUCE_SEG_UNROLL 1  // segment rows in flight per thread
#endif
#ifndef MEP_REDUCE_IMAP
#define MEP_REDUCE_IMAP 0  // 1: float32 -> binary64 by integer ops (x * 2^-896), one conversion per output
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
  // ranked form
  const float *const *rank_G;   // [R] rank gradient buffers
  const int4 *seg;              // segments {expert, rank, start, count}
  const int32_t *rank_seg_ptr;  // [R+1]
  const int32_t *rank_seg_idx;  // [E+R-1] segment indices, rank by rank, slot order
  int64_t rank_rows;            // rows of every rank gradient buffer
  int32_t R;
  int32_t e0;                   // first expert reduced (home rank * E/R)
  int32_t ne;                   // experts reduced
};

constexpr int kMaxSegPerExpert = MEP_MAX_RANKS;  // an expert has at most one segment per rank

template <typename V>
__device__ __forceinline__ V zero_v();
template <>
__device__ __forceinline__ float4 zero_v<float4>() { return make_float4(0.f, 0.f, 0.f, 0.f); }
template <>
__device__ __forceinline__ float zero_v<float>() { return 0.f; }

// Binary64 accumulator of one vector of G.
struct double4_t {
  double x, y, z, w;
};
template <typename V>
struct Acc;
template <>
struct Acc<float4> {
  using T = double4_t;
};
template <>
struct Acc<float> {
  using T = double;
};

__device__ __forceinline__ void zero_acc(double4_t &a) { a.x = a.y = a.z = a.w = 0.0; }
__device__ __forceinline__ void zero_acc(double &a) { a = 0.0; }

#if MEP_REDUCE_IMAP
// The float32 bits u placed at the top of a binary64 word (sign to bit 63,
// exponent to the low end of the exponent field, fraction to the top of the
// fraction) give exactly x * 2^-896 for every finite x, subnormals included.
// Sums of such values round exactly like the unscaled sums: a partial sum
// below 2^-1022 is a multiple of 2^-1045 (2^-896 times float32's finest
// step), hence exact in both.  Infinities and NaNs do not survive the
// mapping: *nf keeps the smallest inverted exponent seen (zero for an
// all-ones exponent), and such a column is summed again exactly.
__device__ __forceinline__ double f32_scaled_f64(float f, uint32_t *nf) {
  const uint32_t u = __float_as_uint(f);
  *nf = min(*nf, (~u) & 0x7f800000u);
  return __hiloint2double((int)(((int32_t)u >> 3) & (int32_t)0x8fffffffu), (int)(u << 29));
}
__device__ __forceinline__ void add_acc(double4_t &a, const float4 &b, uint32_t *nf) {
  a.x = __dadd_rn(a.x, f32_scaled_f64(b.x, nf));
  a.y = __dadd_rn(a.y, f32_scaled_f64(b.y, nf));
  a.z = __dadd_rn(a.z, f32_scaled_f64(b.z, nf));
  a.w = __dadd_rn(a.w, f32_scaled_f64(b.w, nf));
}
__device__ __forceinline__ void add_acc(double &a, float b, uint32_t *nf) {
  a = __dadd_rn(a, f32_scaled_f64(b, nf));
}
__device__ __forceinline__ float4 round_acc(const double4_t &a) {
  return make_float4(__double2float_rn(a.x * 0x1p896), __double2float_rn(a.y * 0x1p896),
                     __double2float_rn(a.z * 0x1p896), __double2float_rn(a.w * 0x1p896));
}
__device__ __forceinline__ float round_acc(double a) { return __double2float_rn(a * 0x1p896); }
#else
__device__ __forceinline__ void add_acc(double4_t &a, const float4 &b, uint32_t *) {
  a.x = __dadd_rn(a.x, (double)b.x);
  a.y = __dadd_rn(a.y, (double)b.y);
  a.z = __dadd_rn(a.z, (double)b.z);
  a.w = __dadd_rn(a.w, (double)b.w);
}
__device__ __forceinline__ void add_acc(double &a, float b, uint32_t *) {
  a = __dadd_rn(a, (double)b);
}
__device__ __forceinline__ float4 round_acc(const double4_t &a) {
  return make_float4(__double2float_rn(a.x), __double2float_rn(a.y), __double2float_rn(a.z),
                     __double2float_rn(a.w));
}
__device__ __forceinline__ float round_acc(double a) { return __double2float_rn(a); }
#endif

// Exact (conversion) forms, for a column that held an infinity or NaN.
__device__ __forceinline__ void add_exact(double4_t &a, const float4 &b) {
  a.x = __dadd_rn(a.x, (double)b.x);
  a.y = __dadd_rn(a.y, (double)b.y);
  a.z = __dadd_rn(a.z, (double)b.z);
  a.w = __dadd_rn(a.w, (double)b.w);
}
__device__ __forceinline__ void add_exact(double &a, float b) { a = __dadd_rn(a, (double)b); }
__device__ __forceinline__ float4 round_exact(const double4_t &a) {
  return make_float4(__double2float_rn(a.x), __double2float_rn(a.y), __double2float_rn(a.z),
                     __double2float_rn(a.w));
}
__device__ __forceinline__ float round_exact(double a) { return __double2float_rn(a); }

// Address of segment s's gradient row: row s of G, or (ranked form) the row
// resolved into s_rows for this task (nullptr if it could not be resolved).
template <typename V, bool kRanked>
__device__ __forceinline__ const V *seg_row(const ReduceParams &p, const V *G,
                                            const V *const *s_rows, int s, int s0) {
  if (kRanked) return s_rows[s - s0];
  return G + (int64_t)s * p.cols;
}

// Ranked form: threads t < s1 - s0 resolve segment s0 + t to its row in its
// rank's buffer.  Returns false if any segment's data was out of range.
// Ranked form: each segment's place in its rank's slot-ordered list (the
// row of the rank's gradient buffer that holds it), built once per block
// from rank_seg_ptr and rank_seg_idx: s_pos[s] = j - rank_seg_ptr[r] for the
// entry j of rank r listing segment s (r its own rank), -1 for a segment its
// rank does not list.  (Searching the rank's list for every segment of every
// task instead measured 0.22-0.77 of the copy peak on the per-home-rank calls.)
// Every thread of the block calls it.
__device__ void build_seg_pos(const ReduceParams &p, int *s_pos, int *s_ptr) {
  const int nrows = p.rows;  // E + R - 1 segment slots
  for (int i = threadIdx.x; i < nrows; i += blockDim.x) s_pos[i] = -1;
  for (int r = threadIdx.x; r <= p.R; r += blockDim.x) s_ptr[r] = __ldg(p.rank_seg_ptr + r);
  __syncthreads();
  const int total = s_ptr[p.R];
  if (total >= 0 && total <= nrows) {
    for (int j = threadIdx.x; j < total; j += blockDim.x) {
      int lo = 0, hi = p.R;  // the rank r with s_ptr[r] <= j < s_ptr[r + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_ptr[mid] <= j) lo = mid; else hi = mid;
      }
      const int sidx = __ldg(p.rank_seg_idx + j);
      // kept only where the listing rank is the segment's own rank
      if (sidx >= 0 && sidx < nrows && s_ptr[lo] <= j && __ldg(&p.seg[sidx].y) == lo)
        s_pos[sidx] = j - s_ptr[lo];
    }
  }
  __syncthreads();
}

// Ranked form: the rows of segments [s0, s1) into s_rows (NULL where a rank
// buffer is missing, misaligned or too short, or the segment is not listed
// by its rank); false if any row is NULL.
template <typename V>
__device__ bool resolve_rows(const ReduceParams &p, int s0, int s1, const int *s_pos,
                             const V **s_rows) {
  bool ok = true;
  for (int t = threadIdx.x; t < s1 - s0; t += blockDim.x) {
    const int s = s0 + t;
    const V *row = nullptr;
    const int r = __ldg(&p.seg[s].y);
    const int j = s_pos[s];
    if (r >= 0 && r < p.R && j >= 0) {
      // a rank buffer must be present, aligned to the vector type and long
      // enough
      const float *base = p.rank_G[r];
      if (base != nullptr && (reinterpret_cast<uintptr_t>(base) % sizeof(V)) == 0 && j < p.rank_rows)
        row = reinterpret_cast<const V *>(base) + (int64_t)j * p.cols;
    }
    if (row == nullptr) ok = false;
    s_rows[t] = row;
  }
  return ok;
}

template <typename V, bool kRanked>
__global__ void __launch_bounds__(kThreads, MEP_REDUCE_MIN_BLOCKS) reduce_kernel(ReduceParams p) {
  griddep_wait();  // the previous kernel on the stream is complete and visible
  __shared__ const V *s_rows[kRanked ? kMaxSegPerExpert : 1];
  __shared__ int s_pos[kRanked ? MEP_MAX_EXPERTS + MEP_MAX_RANKS - 1 : 1];
  __shared__ int s_ptr[kRanked ? MEP_MAX_RANKS + 1 : 1];
  if (kRanked) build_seg_pos(p, s_pos, s_ptr);
  const V *G = reinterpret_cast<const V *>(p.G);
  V *home = reinterpret_cast<V *>(p.home);
  const int64_t tile = (int64_t)kThreads * kU;
  const int64_t tiles_per_e = (p.cols + tile - 1) / tile;
  const int64_t ntask = (int64_t)p.ne * tiles_per_e;
  bool bad = false;
  for (int64_t task = blockIdx.x; task < ntask; task += gridDim.x) {
    const int el = (int)(task / tiles_per_e);  // expert index within the reduced range
    const int e = p.e0 + el;
    const int64_t c0 = (task - (int64_t)el * tiles_per_e) * tile + threadIdx.x;
    int s0 = __ldg(p.eptr + e), s1 = __ldg(p.eptr + e + 1);
    if (s0 < 0 || s1 < s0 || s1 > p.rows || (kRanked && s1 - s0 > kMaxSegPerExpert)) {
      bad = true;
      s0 = s1 = 0;
    }
    if (kRanked) {
      __syncthreads();  // the previous task's rows are no longer read
      if (!resolve_rows<V>(p, s0, s1, s_pos, s_rows)) bad = true;
      __syncthreads();
    }
    typename Acc<V>::T acc[kU];
#pragma unroll
    for (int j = 0; j < kU; ++j) zero_acc(acc[j]);
    uint32_t nf = 0xffffffffu;
    int s = s0;
    for (; s + kSU <= s1; s += kSU) {
      V a[kSU][kU];
#pragma unroll
      for (int q = 0; q < kSU; ++q) {
        const V *row = seg_row<V, kRanked>(p, G, s_rows, s + q, s0);
#pragma unroll
        for (int j = 0; j < kU; ++j) {
          const int64_t c = c0 + (int64_t)j * kThreads;
          a[q][j] = (row != nullptr && c < p.cols) ? __ldcs(row + c) : zero_v<V>();
        }
      }
#pragma unroll
      for (int q = 0; q < kSU; ++q)
#pragma unroll
        for (int j = 0; j < kU; ++j)
          if (c0 + (int64_t)j * kThreads < p.cols) add_acc(acc[j], a[q][j], &nf);
    }
    for (; s < s1; ++s) {
      const V *row = seg_row<V, kRanked>(p, G, s_rows, s, s0);
      V a[kU];
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int64_t c = c0 + (int64_t)j * kThreads;
        a[j] = (row != nullptr && c < p.cols) ? __ldcs(row + c) : zero_v<V>();
      }
#pragma unroll
      for (int j = 0; j < kU; ++j)
        if (c0 + (int64_t)j * kThreads < p.cols) add_acc(acc[j], a[j], &nf);
    }
    V *hrow = home + (int64_t)el * p.cols;
    if (MEP_REDUCE_IMAP && nf == 0) {
      // an infinity or NaN among this thread's inputs: sum its columns again
      // with exact conversions (rare; no cross-thread work involved)
#pragma unroll
      for (int j = 0; j < kU; ++j) zero_acc(acc[j]);
      for (int s2 = s0; s2 < s1; ++s2) {
        const V *row = seg_row<V, kRanked>(p, G, s_rows, s2, s0);
#pragma unroll
        for (int j = 0; j < kU; ++j) {
          const int64_t c = c0 + (int64_t)j * kThreads;
          if (row != nullptr && c < p.cols) add_exact(acc[j], __ldcs(row + c));
        }
      }
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int64_t c = c0 + (int64_t)j * kThreads;
        if (c < p.cols) __stcs(hrow + c, round_exact(acc[j]));
      }
    } else {
#pragma unroll
      for (int j = 0; j < kU; ++j) {
        const int64_t c = c0 + (int64_t)j * kThreads;
        if (c < p.cols) __stcs(hrow + c, round_acc(acc[j]));
      }
    }
  }
  if (bad) set_status(p.status, MEP_ERR_DEVICE_DATA);
}

template <bool kRanked>
cudaError_t launch(ReduceParams &p, int64_t P, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  const bool vec = (P % 4) == 0;
  p.cols = vec ? P / 4 : P;
  const int64_t tile = (int64_t)kThreads * kU;
  const int64_t ntask = (int64_t)p.ne * ((p.cols + tile - 1) / tile);
  if (ntask == 0) return cudaSuccess;
  // the ranked form builds its segment map once per block: a resident-size
  // grid, each block striding over many tasks
  const int64_t cap = kRanked ? (int64_t)sms * MEP_REDUCE_MIN_BLOCKS : (int64_t)sms * MEP_REDUCE_BLOCKS_PER_SM;
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ntask, cap));
  if (vec)
    return launch_pdl(reduce_kernel<float4, kRanked>, dim3(blocks), dim3(kThreads), 0, stream, p);
  return launch_pdl(reduce_kernel<float, kRanked>, dim3(blocks), dim3(kThreads), 0, stream, p);
}

}  // namespace

cudaError_t launch_reduce(const mep_shape_t &s, const mep_plan_t &pl, int64_t P,
                          const float *G, float *home, cudaStream_t stream) {
  ReduceParams p{};
  p.G = G;
  p.home = home;
  p.eptr = pl.expert_seg_ptr;
  p.status = pl.status;
  p.E = s.E;
  p.rows = s.E + s.R - 1;
  p.R = s.R;
  p.e0 = 0;
  p.ne = s.E;
  return launch<false>(p, P, stream);
}

cudaError_t launch_reduce_ranked(const mep_shape_t &s, const mep_plan_t &pl, int64_t P,
                                 int32_t home_rank, const float *const *rank_G,
                                 int64_t rank_rows, float *home, cudaStream_t stream) {
  ReduceParams p{};
  p.home = home;
  p.eptr = pl.expert_seg_ptr;
  p.status = pl.status;
  p.E = s.E;
  p.rows = s.E + s.R - 1;
  p.rank_G = rank_G;
  p.rank_rows = rank_rows;
  p.seg = reinterpret_cast<const int4 *>(pl.seg);
  p.rank_seg_ptr = pl.rank_seg_ptr;
  p.rank_seg_idx = pl.rank_seg_idx;
  p.R = s.R;
  p.ne = s.E / s.R;
  p.e0 = home_rank * p.ne;
  return launch<true>(p, P, stream);
}

}  // namespace mep
