// Internal launch entry points of libmep (host side, not part of the ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "mep.h"

namespace mep {

// Launches `kernel` on `stream` with programmatic stream serialisation
// allowed (see griddep_wait in mep_device.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

constexpr int kPlanThreads = 1024;
constexpr int kPlanMaxBlocks = 1024;          // bound used to size the workspace
constexpr int kPlanIdsPerWarp = 448;          // expert ids a plan warp keeps in shared memory
constexpr int kPlanContiguous = 0;            // plan kinds
constexpr int kPlanHomeFirst = 1;
constexpr int kPlanCapped = 2;
// Workspace rows (of E ints) the capped plan keeps for its published tables
// (3 E + 1 + 2 (E + R) <= 7 E + 1 ints, R <= E), at the end of the tile matrix.
constexpr int kPlanCappedTabRows = 16;
#ifndef MEP_PLAN_MIN_PAIRS_PER_TILE
#define MEP_PLAN_MIN_PAIRS_PER_TILE 2048
#endif
constexpr int64_t kPlanMinPairsPerBlock = MEP_PLAN_MIN_PAIRS_PER_TILE;
constexpr size_t kPlanWsHeader = 256;         // grid-barrier words

size_t plan_workspace_bytes(const mep_shape_t &s);

// Host-side checks of a full plan call's shape, ids pointer and plan struct
// (every field present and aligned); the workspace is checked separately.
mep_status_t check_plan_args(const mep_shape_t &shape, const int32_t *topk_idx,
                             const mep_plan_t *plan);

// Options of a plan launch beyond the whole-range contiguous plan.
struct PlanExtra {
  int B = 0;                              // kPlanCapped: replica experts per rank
  int32_t *max_rank_replicas = nullptr;   // kPlanCapped: [1] out
  // one rank's share (mep_plan_rank): idx holds only rank `rank`'s S*K pairs;
  // rank_counts [R][E] holds every rank's histogram
  const int32_t *rank_counts = nullptr;
  int rank = 0;
};

// Workspace rows (of E ints) at the end of the tile matrix that hold the
// tile totals of one rank's share (phase 2 must not write them to counts,
// which then receives the global T_e).
constexpr int kPlanTotalsRow = kPlanMaxBlocks - kPlanCappedTabRows - 1;

// full = 1: the whole plan; full = 0: counts, max_count, maxvio, status only.
// kind: kPlanContiguous (the sorted pairs cut into R chunks), kPlanHomeFirst
// or kPlanCapped (at most B replica experts per rank when every filler is
// placed; *max_rank_replicas receives the most replica segments on a rank).
cudaError_t launch_plan(const mep_shape_t &s, const int32_t *idx, const mep_plan_t &pl,
                        int full, int kind, void *ws, uint64_t wait_ns, cudaStream_t stream,
                        const PlanExtra *extra = nullptr);

// rank_bufs / rank_ys: nullptr for one [R, S*K, H] buffer, else a device array
// of R row buffers of S*K rows each.  Tokens [g0, g0 + count) of the global
// order are processed; row i of x / out and of w belongs to token g0 + i.
cudaError_t launch_dispatch(const mep_shape_t &s, int32_t H, const mep_plan_t &pl, int64_t g0,
                            int64_t count, const uint16_t *x, uint16_t *buf,
                            uint16_t *const *rank_bufs, cudaStream_t stream);

// The bulk-copy (TMA engine) form of dispatch, same results as launch_dispatch
// over all tokens; waits bounded by wait_ns.
cudaError_t launch_dispatch_bulk(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                                 const uint16_t *x, uint16_t *buf, uint64_t wait_ns,
                                 cudaStream_t stream);

cudaError_t launch_combine(const mep_shape_t &s, int32_t H, const mep_plan_t &pl, int64_t g0,
                           int64_t count, const uint16_t *y, const uint16_t *const *rank_ys,
                           const float *w, uint16_t *out, cudaStream_t stream);

cudaError_t launch_reduce(const mep_shape_t &s, const mep_plan_t &pl, int64_t P,
                          const float *G, float *home, cudaStream_t stream);

// Home rank `home_rank`'s experts only: segment s is row j of rank_G[r], r its
// rank and j its position in r's segment list (rank_seg_idx), j < rank_rows;
// home holds the E/R rows of experts home_rank*E/R ...
cudaError_t launch_reduce_ranked(const mep_shape_t &s, const mep_plan_t &pl, int64_t P,
                                 int32_t home_rank, const float *const *rank_G,
                                 int64_t rank_rows, float *home, cudaStream_t stream);

// The barrier between ranks: arrive at `epoch` in every rank's flag array
// (word `rank`), then wait, bounded by limit_ns, for all R words of my_flags.
cudaError_t launch_rank_barrier(uint32_t *const *peer_flags, const uint32_t *my_flags, int32_t R,
                                int32_t rank, uint32_t epoch, int32_t *status, uint64_t limit_ns,
                                cudaStream_t stream);

cudaError_t launch_prefetch(const mep_shape_t &s, const mep_plan_t &pl, int64_t row_bytes,
                            const void *w_home, void *w_rep, cudaStream_t stream);

cudaError_t launch_combine_backward(const mep_shape_t &s, int32_t H, const mep_plan_t &pl,
                                    const uint16_t *grad_out, const float *w, const uint16_t *y,
                                    uint16_t *grad_y, float *grad_w, cudaStream_t stream);

}  // namespace mep
