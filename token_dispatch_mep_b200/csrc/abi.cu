// The C ABI of libmep (declared in include/mep.h): argument checks, then one
// kernel launch per call.  Nothing here allocates, frees or synchronises,
// except mep_read_status.
#include <atomic>
#include <cstdint>

#include <cuda_runtime.h>

#include "mep.h"
#include "mep_internal.h"

namespace {

std::atomic<uint64_t> g_wait_ns{1000000000ull};

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

mep_status_t check_shape(const mep_shape_t &s) {
  if (s.R < 1 || s.S < 1 || s.E < 1 || s.K < 1) return MEP_ERR_INVALID_ARG;
  if (s.K > s.E || s.K > MEP_MAX_TOPK) return MEP_ERR_INVALID_ARG;
  if (s.E % s.R != 0) return MEP_ERR_INVALID_ARG;
  if (s.E > MEP_MAX_EXPERTS || s.R > MEP_MAX_RANKS) return MEP_ERR_INVALID_ARG;
  if ((int64_t)s.R * s.S * s.K > INT32_MAX) return MEP_ERR_INVALID_ARG;
  return MEP_OK;
}

mep_status_t check_hidden(int32_t H) {
  if (H < 8 || H > MEP_MAX_HIDDEN) return MEP_ERR_INVALID_ARG;
  if (H % 8 != 0) return MEP_ERR_MISALIGNED;
  return MEP_OK;
}

mep_status_t check_ws(const mep_shape_t &s, const void *ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, 256)) return MEP_ERR_WORKSPACE;
  if (ws_bytes < mep::plan_workspace_bytes(s)) return MEP_ERR_WORKSPACE;
  return MEP_OK;
}

mep_status_t check_tokens(const mep_shape_t &s, int64_t begin, int64_t count) {
  const int64_t N = (int64_t)s.R * s.S;
  if (begin < 0 || count < 0 || begin > N || count > N - begin) return MEP_ERR_INVALID_ARG;
  return MEP_OK;
}

mep_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MEP_OK : MEP_ERR_CUDA; }

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

}  // namespace

namespace mep {

mep_status_t check_plan_args(const mep_shape_t &shape, const int32_t *topk_idx,
                             const mep_plan_t *plan) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (!topk_idx || !plan) return MEP_ERR_INVALID_ARG;
  const mep_plan_t &p = *plan;
  if (!p.counts || !p.expert_offset || !p.slot || !p.src_pair || !p.seg || !p.rank_seg_ptr ||
      !p.expert_seg_ptr || !p.replica_seg || !p.num_seg || !p.num_replicas || !p.max_count ||
      !p.status || !p.maxvio || !p.rank_seg_idx)
    return MEP_ERR_INVALID_ARG;
  const void *i32s[] = {topk_idx, p.counts, p.expert_offset, p.slot, p.src_pair, p.rank_seg_ptr,
                        p.expert_seg_ptr, p.replica_seg, p.num_seg, p.num_replicas,
                        p.max_count, p.status, p.rank_seg_idx};
  for (const void *q : i32s)
    if (!aligned(q, 4)) return MEP_ERR_MISALIGNED;
  if (!aligned(p.seg, 16) || !aligned(p.maxvio, 8)) return MEP_ERR_MISALIGNED;
  return MEP_OK;
}

}  // namespace mep

extern "C" {

size_t mep_plan_workspace_bytes(mep_shape_t shape) {
  if (check_shape(shape) != MEP_OK) return 0;
  return mep::plan_workspace_bytes(shape);
}

mep_status_t mep_maxvio(mep_shape_t shape, const int32_t *topk_idx, int32_t *counts,
                        int32_t *max_count, double *maxvio, int32_t *status, void *ws,
                        size_t ws_bytes, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (!topk_idx || !counts || !max_count || !maxvio || !status) return MEP_ERR_INVALID_ARG;
  if (!aligned(topk_idx, 4) || !aligned(counts, 4) || !aligned(max_count, 4) ||
      !aligned(status, 4) || !aligned(maxvio, 8))
    return MEP_ERR_MISALIGNED;
  if ((st = check_ws(shape, ws, ws_bytes)) != MEP_OK) return st;
  mep_plan_t pl{};
  pl.counts = counts;
  pl.max_count = max_count;
  pl.maxvio = maxvio;
  pl.status = status;
  return from_cuda(
      mep::launch_plan(shape, topk_idx, pl, 0, mep::kPlanContiguous, ws, g_wait_ns.load(), as_stream(stream)));
}

namespace {

mep_status_t plan_common(mep_shape_t shape, const int32_t *topk_idx, const mep_plan_t *plan,
                         void *ws, size_t ws_bytes, void *stream, int kind) {
  mep_status_t st = mep::check_plan_args(shape, topk_idx, plan);
  if (st != MEP_OK) return st;
  if ((st = check_ws(shape, ws, ws_bytes)) != MEP_OK) return st;
  return from_cuda(mep::launch_plan(shape, topk_idx, *plan, 1, kind, ws, g_wait_ns.load(), as_stream(stream)));
}

}  // namespace

mep_status_t mep_plan(mep_shape_t shape, const int32_t *topk_idx, const mep_plan_t *plan, void *ws,
                      size_t ws_bytes, void *stream) {
  return plan_common(shape, topk_idx, plan, ws, ws_bytes, stream, mep::kPlanContiguous);
}

mep_status_t mep_plan_home_first(mep_shape_t shape, const int32_t *topk_idx,
                                 const mep_plan_t *plan, void *ws, size_t ws_bytes, void *stream) {
  return plan_common(shape, topk_idx, plan, ws, ws_bytes, stream, mep::kPlanHomeFirst);
}

mep_status_t mep_plan_capped(mep_shape_t shape, int32_t B, const int32_t *topk_idx,
                             const mep_plan_t *plan, int32_t *max_rank_replicas, void *ws,
                             size_t ws_bytes, void *stream) {
  mep_status_t st = mep::check_plan_args(shape, topk_idx, plan);
  if (st != MEP_OK) return st;
  if (B < 1 || !max_rank_replicas) return MEP_ERR_INVALID_ARG;
  if (!aligned(max_rank_replicas, 4)) return MEP_ERR_MISALIGNED;
  if ((st = check_ws(shape, ws, ws_bytes)) != MEP_OK) return st;
  // rounds of fillers beyond E can never be used: keep B - 2 in range
  mep::PlanExtra x;
  x.B = B > shape.E + 2 ? shape.E + 2 : B;
  x.max_rank_replicas = max_rank_replicas;
  return from_cuda(mep::launch_plan(shape, topk_idx, *plan, 1, mep::kPlanCapped, ws,
                                    g_wait_ns.load(), as_stream(stream), &x));
}

mep_status_t mep_rank_histogram(mep_shape_t shape, const int32_t *local_idx, int32_t *counts,
                                int32_t *status, void *ws, size_t ws_bytes, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (!local_idx || !counts || !status) return MEP_ERR_INVALID_ARG;
  if (!aligned(local_idx, 4) || !aligned(counts, 4) || !aligned(status, 4))
    return MEP_ERR_MISALIGNED;
  if ((st = check_ws(shape, ws, ws_bytes)) != MEP_OK) return st;
  // the histogram of one rank's S*K pairs: the counting pass over a
  // one-rank shape (max_count and maxvio are not wanted)
  const mep_shape_t one{1, shape.S, shape.E, shape.K};
  mep_plan_t pl{};
  pl.counts = counts;
  pl.status = status;
  return from_cuda(mep::launch_plan(one, local_idx, pl, 0, mep::kPlanContiguous, ws,
                                    g_wait_ns.load(), as_stream(stream)));
}

mep_status_t mep_plan_rank(mep_shape_t shape, int32_t schedule, int32_t B, int32_t rank,
                           const int32_t *local_idx, const int32_t *rank_counts,
                           const mep_plan_t *plan, int32_t *max_rank_replicas, void *ws,
                           size_t ws_bytes, void *stream) {
  mep_status_t st = mep::check_plan_args(shape, local_idx, plan);
  if (st != MEP_OK) return st;
  if (rank < 0 || rank >= shape.R || !rank_counts) return MEP_ERR_INVALID_ARG;
  if (schedule != MEP_SCHEDULE_CONTIGUOUS && schedule != MEP_SCHEDULE_HOME_FIRST &&
      schedule != MEP_SCHEDULE_CAPPED)
    return MEP_ERR_INVALID_ARG;
  if (schedule == MEP_SCHEDULE_CAPPED && (B < 1 || !max_rank_replicas)) return MEP_ERR_INVALID_ARG;
  if (!aligned(rank_counts, 4) || (max_rank_replicas && !aligned(max_rank_replicas, 4)))
    return MEP_ERR_MISALIGNED;
  if ((st = check_ws(shape, ws, ws_bytes)) != MEP_OK) return st;
  mep::PlanExtra x;
  x.rank_counts = rank_counts;
  x.rank = rank;
  int kind = mep::kPlanContiguous;
  if (schedule == MEP_SCHEDULE_HOME_FIRST) kind = mep::kPlanHomeFirst;
  if (schedule == MEP_SCHEDULE_CAPPED) {
    kind = mep::kPlanCapped;
    x.B = B > shape.E + 2 ? shape.E + 2 : B;
    x.max_rank_replicas = max_rank_replicas;
  }
  return from_cuda(mep::launch_plan(shape, local_idx, *plan, 1, kind, ws, g_wait_ns.load(),
                                    as_stream(stream), &x));
}

mep_status_t mep_dispatch(mep_shape_t shape, int32_t H, const mep_plan_t *plan, const uint16_t *x,
                          uint16_t *buf, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !x || !buf) return MEP_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(buf, 16) || !aligned(plan->slot, 4)) return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_dispatch(shape, H, *plan, 0, (int64_t)shape.R * shape.S, x, buf,
                                        nullptr, as_stream(stream)));
}

mep_status_t mep_dispatch_bulk(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                               const uint16_t *x, uint16_t *buf, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !x || !buf) return MEP_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(buf, 16) || !aligned(plan->slot, 4)) return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_dispatch_bulk(shape, H, *plan, x, buf, g_wait_ns.load(),
                                             as_stream(stream)));
}

mep_status_t mep_combine(mep_shape_t shape, int32_t H, const mep_plan_t *plan, const uint16_t *y,
                         const float *topk_w, uint16_t *out, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !y || !topk_w || !out) return MEP_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(topk_w, 4) || !aligned(plan->slot, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_combine(shape, H, *plan, 0, (int64_t)shape.R * shape.S, y, nullptr,
                                       topk_w, out, as_stream(stream)));
}

mep_status_t mep_reduce_replica_grads(mep_shape_t shape, const mep_plan_t *plan, int64_t P,
                                      const float *seg_grads, float *home_grads, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (P < 0 || !plan) return MEP_ERR_INVALID_ARG;
  if (P == 0) return MEP_OK;
  if (!plan->expert_seg_ptr || !plan->status || !seg_grads || !home_grads)
    return MEP_ERR_INVALID_ARG;
  if ((int64_t)shape.E * P > ((int64_t)1 << 46)) return MEP_ERR_INVALID_ARG;
  const size_t a = (P % 4 == 0) ? 16 : 4;
  if (!aligned(seg_grads, a) || !aligned(home_grads, a) || !aligned(plan->expert_seg_ptr, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_reduce(shape, *plan, P, seg_grads, home_grads, as_stream(stream)));
}

mep_status_t mep_combine_backward(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                  const uint16_t *grad_out, const float *topk_w, const uint16_t *y,
                                  uint16_t *grad_y, float *grad_w, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !grad_out || !topk_w || !y || !grad_y || !grad_w)
    return MEP_ERR_INVALID_ARG;
  if (!aligned(grad_out, 16) || !aligned(y, 16) || !aligned(grad_y, 16) || !aligned(topk_w, 4) ||
      !aligned(grad_w, 4) || !aligned(plan->slot, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_combine_backward(shape, H, *plan, grad_out, topk_w, y, grad_y,
                                                grad_w, as_stream(stream)));
}

mep_status_t mep_dispatch_backward(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                   const uint16_t *grad_buf, uint16_t *grad_x, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !grad_buf || !grad_x) return MEP_ERR_INVALID_ARG;
  if (!aligned(grad_buf, 16) || !aligned(grad_x, 16) || !aligned(plan->slot, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(
      mep::launch_combine(shape, H, *plan, 0, (int64_t)shape.R * shape.S, grad_buf, nullptr, nullptr,
                          grad_x, as_stream(stream)));
}

mep_status_t mep_prefetch_replica_weights(mep_shape_t shape, const mep_plan_t *plan,
                                          int64_t row_bytes, const void *w_home, void *w_rep,
                                          void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (row_bytes < 0 || !plan) return MEP_ERR_INVALID_ARG;
  if (row_bytes == 0) return MEP_OK;
  if (!plan->replica_seg || !plan->seg || !plan->num_replicas || !plan->status || !w_home ||
      !w_rep)
    return MEP_ERR_INVALID_ARG;
  if (row_bytes % 16 != 0 || !aligned(w_home, 16) || !aligned(w_rep, 16) ||
      !aligned(plan->seg, 16) || !aligned(plan->replica_seg, 4) || !aligned(plan->num_replicas, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_prefetch(shape, *plan, row_bytes, w_home, w_rep, as_stream(stream)));
}

mep_status_t mep_dispatch_ranked(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                 const uint16_t *x, uint16_t *const *rank_bufs, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !x || !rank_bufs) return MEP_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rank_bufs, 8) || !aligned(plan->slot, 4)) return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_dispatch(shape, H, *plan, 0, (int64_t)shape.R * shape.S, x, nullptr,
                                        rank_bufs, as_stream(stream)));
}

mep_status_t mep_dispatch_ranked_tokens(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                        int64_t token_begin, int64_t token_count,
                                        const uint16_t *x, uint16_t *const *rank_bufs,
                                        void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if ((st = check_tokens(shape, token_begin, token_count)) != MEP_OK) return st;
  if (token_count == 0) return MEP_OK;
  if (!plan || !plan->slot || !plan->status || !x || !rank_bufs) return MEP_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rank_bufs, 8) || !aligned(plan->slot, 4)) return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_dispatch(shape, H, *plan, token_begin, token_count, x, nullptr,
                                        rank_bufs, as_stream(stream)));
}

mep_status_t mep_combine_ranked(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                const uint16_t *const *rank_ys, const float *topk_w, uint16_t *out,
                                void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if (!plan || !plan->slot || !plan->status || !rank_ys || !topk_w || !out)
    return MEP_ERR_INVALID_ARG;
  if (!aligned(rank_ys, 8) || !aligned(out, 16) || !aligned(topk_w, 4) || !aligned(plan->slot, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_combine(shape, H, *plan, 0, (int64_t)shape.R * shape.S, nullptr,
                                       rank_ys, topk_w, out, as_stream(stream)));
}

mep_status_t mep_combine_ranked_tokens(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                       int64_t token_begin, int64_t token_count,
                                       const uint16_t *const *rank_ys, const float *topk_w,
                                       uint16_t *out, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if ((st = check_hidden(H)) != MEP_OK) return st;
  if ((st = check_tokens(shape, token_begin, token_count)) != MEP_OK) return st;
  if (token_count == 0) return MEP_OK;
  if (!plan || !plan->slot || !plan->status || !rank_ys || !topk_w || !out)
    return MEP_ERR_INVALID_ARG;
  if (!aligned(rank_ys, 8) || !aligned(out, 16) || !aligned(topk_w, 4) || !aligned(plan->slot, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_combine(shape, H, *plan, token_begin, token_count, nullptr, rank_ys,
                                       topk_w, out, as_stream(stream)));
}

mep_status_t mep_reduce_replica_grads_ranked(mep_shape_t shape, const mep_plan_t *plan, int64_t P,
                                             int32_t home_rank, const float *const *rank_grads,
                                             int64_t rank_rows, float *home_grads, void *stream) {
  mep_status_t st = check_shape(shape);
  if (st != MEP_OK) return st;
  if (P < 0 || !plan || home_rank < 0 || home_rank >= shape.R || rank_rows < 1)
    return MEP_ERR_INVALID_ARG;
  if (P == 0) return MEP_OK;
  if (!plan->expert_seg_ptr || !plan->seg || !plan->rank_seg_ptr || !plan->rank_seg_idx ||
      !plan->status || !rank_grads || !home_grads)
    return MEP_ERR_INVALID_ARG;
  if ((int64_t)shape.E * P > ((int64_t)1 << 46)) return MEP_ERR_INVALID_ARG;
  const size_t a = (P % 4 == 0) ? 16 : 4;
  if (!aligned(home_grads, a) || !aligned(rank_grads, 8) || !aligned(plan->expert_seg_ptr, 4) ||
      !aligned(plan->seg, 16) || !aligned(plan->rank_seg_ptr, 4) || !aligned(plan->rank_seg_idx, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_reduce_ranked(shape, *plan, P, home_rank, rank_grads, rank_rows,
                                             home_grads, as_stream(stream)));
}

mep_status_t mep_rank_barrier(uint32_t *const *peer_flags, uint32_t *my_flags, int32_t R,
                              int32_t rank, uint32_t epoch, int32_t *status, void *stream) {
  if (R < 1 || R > MEP_MAX_RANKS || rank < 0 || rank >= R) return MEP_ERR_INVALID_ARG;
  if (!peer_flags || !my_flags || !status) return MEP_ERR_INVALID_ARG;
  if (!aligned(peer_flags, 8) || !aligned(my_flags, 4) || !aligned(status, 4))
    return MEP_ERR_MISALIGNED;
  return from_cuda(mep::launch_rank_barrier(peer_flags, my_flags, R, rank, epoch, status,
                                            g_wait_ns.load(), as_stream(stream)));
}

mep_status_t mep_read_status(const mep_plan_t *plan, void *stream) {
  if (!plan || !plan->status) return MEP_ERR_INVALID_ARG;
  int32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, plan->status, sizeof host, cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e != cudaSuccess) return MEP_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MEP_ERR_CUDA;
  return static_cast<mep_status_t>(host);
}

const char *mep_status_string(mep_status_t s) {
  switch (s) {
    case MEP_OK: return "ok";
    case MEP_ERR_INVALID_ARG: return "invalid argument";
    case MEP_ERR_MISALIGNED: return "misaligned pointer or hidden size";
    case MEP_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MEP_ERR_CUDA: return "CUDA error";
    case MEP_ERR_DEVICE_DATA: return "out-of-range data seen on the device";
    case MEP_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

void mep_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns < 1000 ? 1000 : ns); }

uint64_t mep_get_wait_limit_ns(void) { return g_wait_ns.load(); }

int32_t mep_version(void) { return MEP_VERSION; }

}  // extern "C"
