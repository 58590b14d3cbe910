/*
 * mep.h -- C ABI of libmep: MoonEP's balanced expert-parallel token plan and
 * its data movement, as hand-written CUDA kernels for one B200 (sm_100a).
 *
 * What the library computes (sources named by page title and section):
 *
 *   "Moonshot AI Open-Sources MoonEP, the Library Used to Train the MoE Model
 *   Kimi K3" (below: the MoonEP release page)
 *     - "Why expert parallelism is needed": a router assigns each token to K
 *       experts; imbalance is measured by maxvio = max_e(T_e / T-bar) - 1,
 *       which is 0 for a perfectly even load.
 *     - "How MoonEP works": the number of token slots per EP rank is pinned
 *       at S x K whatever the routing; a few duplicate (replica) experts are
 *       placed each step from that step's routing, and in the backward pass
 *       the duplicates' gradients are summed into the home copy.
 *     - "Why this matters to engineers": fixed buffer shapes, no staging
 *       copy -- each row goes directly to its final expert-ordered slot --
 *       and no host round trip per layer.
 *   "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert Parallelism
 *   Library for MoE Training", "The problem MoonEP targets": T_e counts the
 *   tokens routed to expert e; T-bar is the count expected under perfect
 *   balance.
 *
 * The pages give no scheduling algorithm.  This library fixes one: the stable
 * sort of all (token, k) pairs by (expert, global token g, k), cut into R
 * contiguous chunks of S*K slots.  Chunk r is rank r's static receive buffer;
 * a (rank, expert) run inside it is a segment; a segment on a rank other
 * than home(e) = e / (E/R) hosts a replica of expert e.
 *
 * Notation.  R simulated ranks, S tokens per rank, E experts, K experts per
 * token, H hidden size.  N = R*S tokens, global token g = r*S + s (rank-major),
 * pair (g, k) has flat index g*K + k, NK = N*K pairs = slots, SK = S*K slots per
 * rank, global slot p in [0, NK), rank(p) = p / SK.
 *
 * Conventions for every call.
 *   - All buffers are caller-owned device memory; the library never allocates
 *     or frees.  Scratch comes from a caller-supplied workspace.
 *   - Every call is asynchronous and stream-ordered on `stream` (a
 *     cudaStream_t; NULL is the legacy default stream).  No call synchronises
 *     the host except mep_read_status.
 *   - Host-detected errors (bad shape, NULL or misaligned pointer, small
 *     workspace) return immediately and launch nothing.
 *   - Device-detected errors (an expert id outside [0, E), a slot or segment
 *     pointer outside its range, a wait that timed out) are written into the
 *     plan's device status word; the first error wins.  Outputs are undefined
 *     when the status is not MEP_OK, but no kernel ever reads or writes
 *     outside the buffers described here.
 *   - bf16 buffers are typed uint16_t (raw bf16 bit patterns) so that C callers
 *     need no CUDA headers.
 *   - The current CUDA device is the one the buffers live on.
 */
#ifndef MEP_H
#define MEP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MEP_API __attribute__((visibility("default")))
#else
#define MEP_API
#endif

#define MEP_VERSION 4
#define MEP_MAX_EXPERTS 1024      /* E <= 1024 */
#define MEP_MAX_RANKS 1024        /* R <= 1024 */
#define MEP_MAX_HIDDEN 32768      /* H <= 32768 bf16 elements per row */
#define MEP_MAX_TOPK 16           /* K <= 16 */

typedef enum {
    MEP_OK = 0,
    MEP_ERR_INVALID_ARG = 1,  /* shape rule broken or NULL pointer */
    MEP_ERR_MISALIGNED = 2,   /* row buffers need 16-byte alignment and H % 8 == 0 */
    MEP_ERR_WORKSPACE = 3,    /* workspace NULL, not 256-byte aligned, or too small */
    MEP_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    MEP_ERR_DEVICE_DATA = 5,  /* device saw an expert id / slot / segment pointer out of range */
    MEP_ERR_TIMEOUT = 6       /* a bounded device-side wait ran out */
} mep_status_t;

/* Shape rules: R, S, E, K >= 1; K <= E; K <= MEP_MAX_TOPK; E % R == 0
 * (home(e) = e / (E/R)); E <= MEP_MAX_EXPERTS; R <= MEP_MAX_RANKS;
 * R*S*K < 2^31. */
typedef struct {
    int32_t R, S, E, K;
} mep_shape_t;

/* One (rank, expert) run of slots: slots [rank*SK + start, rank*SK + start +
 * count) all hold pairs routed to `expert`.  16 bytes. */
typedef struct {
    int32_t expert, rank, start, count;
} mep_segment_t;

/* The plan: device pointers, caller-owned, sized from the shape alone.
 * Segments are listed by (expert, rank); at most E + R - 1 exist.  In the
 * contiguous plan (mep_plan) that is also slot order; in the home-first plan
 * (mep_plan_home_first) each rank's segments in slot order are listed by
 * rank_seg_idx. */
typedef struct {
    int32_t *counts;          /* [E]     T_e                                    */
    int32_t *expert_offset;   /* [E+1]   first slot of expert e; [E] = NK        */
    int32_t *slot;            /* [N*K]   pair (g,k) -> global slot p             */
    int32_t *src_pair;        /* [N*K]   slot p -> pair index g*K + k            */
    mep_segment_t *seg;       /* [E+R-1] segments in slot order                  */
    int32_t *rank_seg_ptr;    /* [R+1]   rank r owns entries [ptr[r], ptr[r+1]) of rank_seg_idx */
    int32_t *expert_seg_ptr;  /* [E+1]   expert e owns segments [ptr[e], ptr[e+1]) */
    int32_t *replica_seg;     /* [E+R-1] indices of replica segments, ascending  */
    int32_t *num_seg;         /* [1]                                             */
    int32_t *num_replicas;    /* [1]     segments with rank != home(expert)      */
    int32_t *max_count;       /* [1]     max_e T_e                               */
    int32_t *status;          /* [1]     device error word (mep_status_t)        */
    double *maxvio;           /* [1]     max_e(T_e / T-bar) - 1, T-bar = NK / E  */
    int32_t *rank_seg_idx;    /* [E+R-1] segment indices, rank by rank, slot order */
} mep_plan_t;

/* Bytes of workspace mep_plan and mep_maxvio need for this shape.  The
 * workspace must be zero-filled once before its first use (e.g. by
 * cudaMemsetAsync); every call that returns MEP_OK and ends with device
 * status MEP_OK leaves it ready for the next call.  After MEP_ERR_TIMEOUT or
 * MEP_ERR_CUDA, zero it again.  One workspace serves one stream at a time. */
MEP_API size_t mep_plan_workspace_bytes(mep_shape_t shape);

/* T_e and maxvio only ("Why expert parallelism is needed", release page).
 *   topk_idx  int32 [N, K] row-major, expert ids of each token's top-K.
 *   counts    int32 [E] out: T_e.
 *   max_count int32 [1] out: max_e T_e.
 *   maxvio    double [1] out: (double)(max_count * E) / (double)(N*K) - 1.0,
 *             one IEEE binary64 division of two exact integers.
 *   status    int32 [1] out: device error word, cleared by this call.
 *   ws        workspace of mep_plan_workspace_bytes(shape) bytes, 256-byte aligned. */
MEP_API mep_status_t mep_maxvio(mep_shape_t shape, const int32_t *topk_idx,
                        int32_t *counts, int32_t *max_count, double *maxvio,
                        int32_t *status, void *ws, size_t ws_bytes, void *stream);

/* The balanced plan ("How MoonEP works"; "Why this matters to engineers").
 *   topk_idx  int32 [N, K] row-major.
 *   plan      every field written: counts, maxvio and max_count as in
 *             mep_maxvio; expert_offset = exclusive prefix sum of counts;
 *             slot[g*K+k] = expert_offset[e] + #{(g',k') before (g,k) in
 *             (g, k) order with the same expert e}; src_pair its inverse;
 *             the segments, CSR pointers and replica list of the R-way cut;
 *             rank_seg_idx[i] = i (segments are already in slot order).
 *             plan->status is cleared at the start of the call.
 * Rank r holds exactly the SK slots [r*SK, (r+1)*SK), in expert order. */
MEP_API mep_status_t mep_plan(mep_shape_t shape, const int32_t *topk_idx,
                      const mep_plan_t *plan, void *ws, size_t ws_bytes,
                      void *stream);

/* The home-first plan: the same outputs as mep_plan (and the same workspace),
 * for a schedule that keeps experts home whenever their home rank has room
 * -- the pages' "small number" of duplicates ("How MoonEP works"); the pages
 * fix no algorithm, this is the reading this library takes:
 *   1. rank r fills its S*K slots with its home experts first, in ascending
 *      expert order: expert e keeps h_e = min(T_e, room left) pairs home;
 *   2. the overflow T_e - h_e of all experts, in ascending expert order, is
 *      cut contiguously over the spare room of the ranks in ascending rank
 *      order; every (expert, rank) piece of overflow is a replica;
 *   3. rank r's slots hold its home pieces, then its replica pieces, each in
 *      expert order; inside a piece pairs keep (g, k) order, and an expert's
 *      first h_e pairs are the ones kept home.
 * Every rank still receives exactly S*K slots.  Segments are listed by
 * (expert, rank) (so mep_reduce_replica_grads works unchanged);
 * rank_seg_idx[rank_seg_ptr[r] .. rank_seg_ptr[r+1]) lists rank r's segments
 * in slot order.  expert_offset is the exclusive prefix sum of counts (not a
 * slot position in this plan).  At most E + R - 1 segments, and at most
 * (overflowing experts) + (ranks with room) - 1 replicas. */
MEP_API mep_status_t mep_plan_home_first(mep_shape_t shape, const int32_t *topk_idx,
                                         const mep_plan_t *plan, void *ws, size_t ws_bytes,
                                         void *stream);

/* The capped plan: at most B replica experts per rank ("How MoonEP works": a
 * small number of duplicate experts; "Key facts about the release": B = E/R
 * for training, 3-4 recommended for inference).  The pages do not define B;
 * this library reads it as the number of replica (duplicate) experts a rank
 * may host besides its home experts -- the slots of its buffer for
 * duplicates' weights.  Same outputs as mep_plan (and the same workspace);
 * the pages fix no algorithm, this is the one this library takes:
 *   1. rank r keeps its home experts' pairs, smallest expert (by T_e, ties to
 *      the lower id) first: expert e keeps h_e = min(T_e, room left);
 *   2. items = experts that overflow, by overflow descending (ties: lower
 *      id); rooms = ranks with spare room, by room descending (ties: lower
 *      rank); Dmax = the largest room;
 *   3. items with overflow below Dmax are fillers: filler f (in item order)
 *      is offered to room f mod Y (Y rooms) in round f / Y and placed whole,
 *      as one replica piece, if the round is below B - 2 and the room's space
 *      left holds it;
 *   4. the other items, in item order, are cut contiguously over the rooms'
 *      space left, in room order;
 *   5. rank r's slots hold its home pieces (ascending expert), then its
 *      fillers (by round), then its stream pieces (stream order); expert e's
 *      pairs in (g, k) order fill its home piece (the first h_e), then its
 *      replica pieces in the order they were made.
 * Every rank receives exactly S*K slots.  When every filler is placed and
 * B >= 3, no rank hosts more than B replicas (a room takes at most B - 2
 * fillers, and the stream items are all at least Dmax, so a room's space
 * left meets at most two of them); otherwise the cap may be exceeded.
 *   B                  >= 1 (values above E + 2 act as E + 2).
 *   max_rank_replicas  int32 [1] device out: the most replica segments on
 *                      one rank; compare it with B.
 * Segments are listed by (expert, rank); rank_seg_idx lists each rank's
 * segments in slot order; expert_offset is the exclusive prefix sum of
 * counts.  At most E + R - 1 segments. */
MEP_API mep_status_t mep_plan_capped(mep_shape_t shape, int32_t B, const int32_t *topk_idx,
                                     const mep_plan_t *plan, int32_t *max_rank_replicas,
                                     void *ws, size_t ws_bytes, void *stream);

/* The schedules a plan can follow (mep_plan_rank). */
typedef enum {
    MEP_SCHEDULE_CONTIGUOUS = 0,  /* mep_plan */
    MEP_SCHEDULE_HOME_FIRST = 1,  /* mep_plan_home_first */
    MEP_SCHEDULE_CAPPED = 2       /* mep_plan_capped */
} mep_schedule_t;

/* One rank's histogram, the input of the plan's one exchange between ranks
 * ("The problem MoonEP targets": T_e counts the tokens routed to expert e).
 *   local_idx  int32 [S, K], the rank's own top-K expert ids.
 *   counts     int32 [E] out: how many of those S*K pairs go to each expert.
 *   status     int32 [1] out: device error word, cleared by this call
 *              (MEP_ERR_DEVICE_DATA for an id outside [0, E)).
 *   ws         workspace of mep_plan_workspace_bytes(shape) bytes.
 * On a multi-GPU system every rank all-gathers these E-vectors (R x E int32:
 * 229 KB on the R = 64, E = 896 shape) and calls mep_plan_rank. */
MEP_API mep_status_t mep_rank_histogram(mep_shape_t shape, const int32_t *local_idx,
                                        int32_t *counts, int32_t *status, void *ws,
                                        size_t ws_bytes, void *stream);

/* One rank's share of the plan, from the gathered histograms ("How MoonEP
 * works": every rank computes the same schedule from the current routing).
 *   schedule       a mep_schedule_t; B and max_rank_replicas as in
 *                  mep_plan_capped (ignored, may be 0 / NULL, otherwise).
 *   rank           0 <= rank < R: the rank whose tokens local_idx holds
 *                  (global tokens rank*S .. rank*S + S - 1).
 *   local_idx      int32 [S, K].
 *   rank_counts    int32 [R, E] device: row r = mep_rank_histogram of rank
 *                  r's ids.  Row `rank` must equal this rank's own histogram
 *                  (checked on the device: MEP_ERR_DEVICE_DATA otherwise).
 *   plan           written exactly as the whole-range call of the same
 *                  schedule writes it, except slot and src_pair: slot rows
 *                  rank*S .. rank*S + S - 1 (this rank's pairs) and src_pair
 *                  at those pairs' slots; other entries are not touched.
 * A pair's place among its expert's pairs is the number of pairs of that
 * expert on lower ranks (a prefix of the gathered columns; tokens are
 * numbered rank-major) plus its place among the rank's own, so every rank's
 * tables equal the whole-range plan's bit for bit. */
MEP_API mep_status_t mep_plan_rank(mep_shape_t shape, int32_t schedule, int32_t B, int32_t rank,
                                   const int32_t *local_idx, const int32_t *rank_counts,
                                   const mep_plan_t *plan, int32_t *max_rank_replicas,
                                   void *ws, size_t ws_bytes, void *stream);

/* Zero-copy dispatch into the static receive buffer ("Why this matters to
 * engineers": each row is copied directly to its final expert-ordered slot).
 *   x    bf16 [N, H], 16-byte aligned; H % 8 == 0, 8 <= H <= MEP_MAX_HIDDEN.
 *   buf  bf16 [R, S*K, H] out, 16-byte aligned: buf[slot[g,k], :] = x[g, :]
 *        for every pair; a token routed to several experts is copied once
 *        per slot.  Bit-exact copies. */
MEP_API mep_status_t mep_dispatch(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                          const uint16_t *x, uint16_t *buf, void *stream);

/* mep_dispatch through the bulk-copy (TMA) engine: the same arguments and the
 * same bytes in buf, with every row staged in shared memory -- one bulk load
 * of the token's row, then K bulk stores of it to the token's slots, per
 * pipeline of two shared-memory stages.  Kept for comparison with
 * mep_dispatch, which moves the rows through registers and is faster on B200
 * (0.96-0.99 of the HBM copy bandwidth against 0.83-0.86 for this form on
 * the R=8/E=64, Kimi-shaped and R=32 skew workloads).  Its waits on row
 * arrival are bounded by mep_get_wait_limit_ns (MEP_ERR_TIMEOUT in
 * plan->status); a slot outside [0, N*K) records MEP_ERR_DEVICE_DATA. */
MEP_API mep_status_t mep_dispatch_bulk(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                       const uint16_t *x, uint16_t *buf, void *stream);

/* Weighted combine back to token order (the return leg of the top-K routing
 * in "Why expert parallelism is needed").
 *   y      bf16 [R, S*K, H] expert outputs in slot order, 16-byte aligned.
 *   topk_w float32 [N, K] router weights.
 *   out    bf16 [N, H] out: out[g,:] = bf16_rne(sum over k = 0..K-1, in that
 *          order, of w[g,k] * y[slot[g,k], :]), accumulated in float32 with a
 *          fused multiply-add per term. */
MEP_API mep_status_t mep_combine(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                         const uint16_t *y, const float *topk_w, uint16_t *out,
                         void *stream);

/* Backward reduction of replica weight-gradients into their home expert
 * ("How MoonEP works": duplicates' gradients summed into the home copy).
 *   seg_grads  float32 [E+R-1, P]: row s is the gradient computed by segment
 *              s of the plan (its rank's copy of expert seg[s].expert); rows
 *              s >= num_seg are ignored.  16-byte aligned when P % 4 == 0.
 *   home_grads float32 [E, P] out: home_grads[e,:] = sum of rows
 *              expert_seg_ptr[e] .. expert_seg_ptr[e+1]-1, ascending, in
 *              float32; zero for an expert with no segment.
 *   P >= 0; P == 0 is a no-op. */
MEP_API mep_status_t mep_reduce_replica_grads(mep_shape_t shape, const mep_plan_t *plan,
                                      int64_t P, const float *seg_grads,
                                      float *home_grads, void *stream);

/* Rank-addressed dispatch and combine: the same operations with every rank's
 * S*K slots in a buffer of its own.  This is the form the exchange between
 * GPUs takes: on a multi-GPU system rank r's receive buffer lives on GPU r
 * and is mapped into this GPU's address space (CUDA IPC or symmetric memory
 * over NVLink), so each 16-byte store of dispatch is a peer write straight
 * into the slot that rank owns and combine reads its rows back the same way
 * -- the all-to-all is fused into the copy, with no staging buffer.  The
 * caller orders the exchange (every rank's buffer free before dispatch, every
 * rank's expert outputs written before combine).
 *   rank_bufs / rank_ys  device array of R device pointers (8-byte aligned);
 *            pointer r addresses rank r's [S*K, H] bf16 rows, 16-byte aligned.
 *   Slot p is row p % (S*K) of buffer p / (S*K).  Results are bit-identical
 *   to mep_dispatch / mep_combine on the concatenated buffer. */
MEP_API mep_status_t mep_dispatch_ranked(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                         const uint16_t *x, uint16_t *const *rank_bufs,
                                         void *stream);
MEP_API mep_status_t mep_combine_ranked(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                        const uint16_t *const *rank_ys, const float *topk_w,
                                        uint16_t *out, void *stream);

/* One rank's share of the exchange: the rank-addressed dispatch and combine
 * restricted to the tokens [token_begin, token_begin + token_count) of the
 * global order -- on a multi-GPU system, the tokens this GPU holds (rank r:
 * token_begin = r*S, token_count = S), after every rank has computed the same
 * plan from the gathered router ids.  Row i of x, out and topk_w belongs to
 * global token token_begin + i:
 *   x       bf16 [token_count, H]   the local hidden rows (dispatch input).
 *   topk_w  float32 [token_count, K] the local router weights (combine).
 *   out     bf16 [token_count, H] out: the local combine output.
 * rank_bufs / rank_ys as in mep_dispatch_ranked / mep_combine_ranked; every
 * pointer in them must be non-NULL and 16-byte aligned (checked on the
 * device: a bad one records MEP_ERR_DEVICE_DATA and is not dereferenced).
 * 0 <= token_begin, 0 <= token_count, token_begin + token_count <= N, else
 * MEP_ERR_INVALID_ARG; token_count == 0 is a no-op.  Calls over disjoint
 * token ranges that cover [0, N) give exactly the results of the whole-range
 * calls. */
MEP_API mep_status_t mep_dispatch_ranked_tokens(mep_shape_t shape, int32_t H,
                                                const mep_plan_t *plan, int64_t token_begin,
                                                int64_t token_count, const uint16_t *x,
                                                uint16_t *const *rank_bufs, void *stream);
MEP_API mep_status_t mep_combine_ranked_tokens(mep_shape_t shape, int32_t H,
                                               const mep_plan_t *plan, int64_t token_begin,
                                               int64_t token_count,
                                               const uint16_t *const *rank_ys,
                                               const float *topk_w, uint16_t *out, void *stream);

/* One home rank's share of the backward reduction ("How MoonEP works": the
 * duplicates' gradients are summed into the home copy), with every rank's
 * segment gradients in a buffer of its own.
 *   home_rank   0 <= home_rank < R; its experts are e = home_rank*E/R ...
 *               (home_rank+1)*E/R - 1.
 *   rank_grads  device array of R device pointers (8-byte aligned); pointer r
 *               addresses rank r's float32 rows [rank_rows, P], row j holding
 *               the gradient of rank r's j-th segment in slot order, i.e.
 *               segment rank_seg_idx[rank_seg_ptr[r] + j].  A rank holds at
 *               most min(E, S*K) segments, so rank_rows = min(E, S*K) always
 *               suffices.  Each pointer 16-byte aligned when P % 4 == 0 (else
 *               4).  A NULL or misaligned pointer, or a segment at j >=
 *               rank_rows, is detected on the device, records
 *               MEP_ERR_DEVICE_DATA and contributes nothing.  Only the pointers
 *               of ranks that hold a segment of a home expert are read.
 *   rank_rows   rows of every rank's gradient buffer, >= 1.
 *   home_grads  float32 [E/R, P] out: row i = sum over the segments of expert
 *               home_rank*E/R + i, ascending segment index, in float32 (the
 *               same sums, bit for bit, as rows of mep_reduce_replica_grads);
 *               zero for an expert with no segment.
 *   P >= 0; P == 0 is a no-op. */
MEP_API mep_status_t mep_reduce_replica_grads_ranked(mep_shape_t shape, const mep_plan_t *plan,
                                                     int64_t P, int32_t home_rank,
                                                     const float *const *rank_grads,
                                                     int64_t rank_rows, float *home_grads,
                                                     void *stream);

/* Buffer sharing between processes (one process per GPU): rank r exports its
 * receive, expert-output and gradient buffers, the others map them and put
 * the mapped addresses into the device pointer arrays above.  Host calls,
 * synchronous, no kernel; CUDA IPC underneath, so the memory must come from
 * cudaMalloc (directly or through a caching allocator of cudaMalloc
 * segments).  Mapping and unmapping a peer's allocation is the only memory
 * management in the library; it never allocates.
 *   mep_ipc_export  describes [ptr, ptr + bytes) of the current device:
 *                   `out` receives the allocation's IPC handle, the offset of
 *                   ptr inside it and `bytes`.  MEP_ERR_INVALID_ARG if the
 *                   range is not inside one allocation, MEP_ERR_CUDA if CUDA
 *                   refuses the handle.
 *   mep_ipc_open    in another process: maps the allocation (peer access
 *                   enabled lazily) and returns the exported address in
 *                   *ptr.  A process may not open its own export.
 *   mep_ipc_close   unmaps what mep_ipc_open returned for the same handle;
 *                   call after the last kernel that reads or writes it has
 *                   finished. */
typedef struct {
    unsigned char handle[64];   /* cudaIpcMemHandle_t of the allocation */
    uint64_t offset;            /* byte offset of the exported range in it */
    uint64_t bytes;             /* length of the exported range */
} mep_ipc_handle_t;
MEP_API mep_status_t mep_ipc_export(const void *ptr, uint64_t bytes, mep_ipc_handle_t *out);
MEP_API mep_status_t mep_ipc_open(const mep_ipc_handle_t *handle, void **ptr);
MEP_API mep_status_t mep_ipc_close(const mep_ipc_handle_t *handle, void *ptr);

/* Replica weight prefetch: before the expert compute, every replica gets a
 * copy of its expert's home weights ("How MoonEP works": the duplicates are
 * fetched ahead of the main computation).  The forward mirror of
 * mep_reduce_replica_grads.
 *   row_bytes  bytes of one expert's weights (any element type), a multiple
 *              of 16; 0 is a no-op.
 *   w_home     [E, row_bytes] home weights, 16-byte aligned.
 *   w_rep      [E+R-1, row_bytes] out: row j < num_replicas receives
 *              w_home[seg[replica_seg[j]].expert]; rows j >= num_replicas are
 *              not touched.  num_replicas is read on the device.
 * Bit-exact copies. */
MEP_API mep_status_t mep_prefetch_replica_weights(mep_shape_t shape, const mep_plan_t *plan,
                                                  int64_t row_bytes, const void *w_home,
                                                  void *w_rep, void *stream);

/* Backward of mep_combine (the adjoint of the weighted combine; the backward
 * pass of "How MoonEP works").
 *   grad_out bf16 [N, H]        gradient of the combine output.
 *   topk_w   float32 [N, K]     router weights of the forward combine.
 *   y        bf16 [R, S*K, H]   expert outputs the forward combine read.
 *   grad_y   bf16 [R, S*K, H] out: grad_y[slot[g,k], :] = w[g,k] * grad_out[g, :],
 *            rounded once to nearest-even bf16 (every slot is written once).
 *   grad_w   float32 [N, K] out: grad_w[g,k] = sum_h grad_out[g,h] * y[slot[g,k],h],
 *            float32 FMAs per lane, then a fixed-order warp reduction.
 * Row buffers 16-byte aligned, H % 8 == 0. */
MEP_API mep_status_t mep_combine_backward(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                          const uint16_t *grad_out, const float *topk_w,
                                          const uint16_t *y, uint16_t *grad_y, float *grad_w,
                                          void *stream);

/* Backward of mep_dispatch (the adjoint of the copy into the slots).
 *   grad_buf bf16 [R, S*K, H]   gradient of the dispatch buffer.
 *   grad_x   bf16 [N, H] out: grad_x[g,:] = bf16_rne(sum over k = 0..K-1, in
 *            that order, of grad_buf[slot[g,k], :]), accumulated in float32.
 * Row buffers 16-byte aligned, H % 8 == 0. */
MEP_API mep_status_t mep_dispatch_backward(mep_shape_t shape, int32_t H, const mep_plan_t *plan,
                                           const uint16_t *grad_buf, uint16_t *grad_x,
                                           void *stream);

/* mep_plan without a caller-supplied workspace, for callers that cannot
 * allocate device memory (no allocator in their runtime, or a host framework
 * that owns the device memory pool and forbids allocation after start-up).
 * The paper (the MoonEP release pages) has no counterpart to this call.
 * Same arguments and results as mep_plan.  Its scratch is a device array of
 * MEP_NOALLOC_SCRATCH_BYTES compiled into the library, held by every GPU that
 * loads the library until the process exits.  It holds the workspace of
 * the largest shape the library accepts (E = MEP_MAX_EXPERTS); a shape beyond
 * the shape rules is rejected with MEP_ERR_INVALID_ARG, and a workspace that
 * would not fit the array with MEP_ERR_WORKSPACE, before anything runs; every
 * argument check of mep_plan also runs before anything is queued.  The first
 * call in a CUDA context of a device looks up that array's device address in
 * that context (make that call before any stream capture on the device); a
 * call in a new context of the device, e.g. after cudaDeviceReset, looks it up
 * again.  Each call clears the array's barrier words with a 256-byte memset on
 * `stream`, then launches the plan.
 * The array is shared by all calls on a device: calls that overlap on the GPU
 * (e.g. on two streams with no ordering between them) race and give
 * undefined plans.  Allocates nothing and frees nothing. */
#define MEP_NOALLOC_SCRATCH_BYTES (256u + 1024u * 1024u * 4u)
MEP_API mep_status_t mep_plan_noalloc(mep_shape_t shape, const int32_t *topk_idx,
                                      const mep_plan_t *plan, void *stream);

/* A barrier between the ranks of an expert-parallel group, on the device, in
 * place of a host round trip between the exchange's phases ("Why this
 * matters to engineers": no per-layer host synchronisation).
 *   peer_flags  device array of R device pointers (8-byte aligned); pointer p
 *               addresses rank p's R flag words (uint32, 4-byte aligned), in
 *               rank p's memory and mapped into this process (mep_ipc_open),
 *               or any device-visible memory.
 *   my_flags    this rank's own R flag words (the array peer_flags[rank]
 *               addresses, as this process sees it).
 *   rank        0 <= rank < R <= MEP_MAX_RANKS.
 *   epoch       this crossing's number; use 1, 2, 3, ... on every rank (the
 *               words start at 0; comparisons are modulo 2^32).
 *   status      int32 [1] device word: MEP_ERR_TIMEOUT if some rank's word did
 *               not reach `epoch` within mep_get_wait_limit_ns, and
 *               MEP_ERR_DEVICE_DATA for a NULL or misaligned peer pointer
 *               (first error wins; the word is not cleared).
 * One kernel: after every earlier write of `stream` is made visible system-
 * wide, it stores `epoch` into word `rank` of every rank's array (release,
 * system scope), then waits until all R words of my_flags have reached
 * `epoch` (acquire, system scope).  Later work on `stream` then sees every
 * rank's writes from before its own arrival.  Every rank must call it with
 * the same epochs, in the same order. */
MEP_API mep_status_t mep_rank_barrier(uint32_t *const *peer_flags, uint32_t *my_flags, int32_t R,
                                      int32_t rank, uint32_t epoch, int32_t *status,
                                      void *stream);

/* Synchronises `stream` and returns the plan's device status word (MEP_OK if
 * every call so far on this plan ran clean), or MEP_ERR_CUDA if the copy
 * itself fails.  The only call that blocks the host. */
MEP_API mep_status_t mep_read_status(const mep_plan_t *plan, void *stream);

/* Static, human-readable name of a status code. */
MEP_API const char *mep_status_string(mep_status_t status);

/* Upper bound, in nanoseconds of the GPU global timer, on every device-side
 * wait (the grid barriers of the plan calls and the waits of
 * mep_rank_barrier).  A wait that runs out
 * records MEP_ERR_TIMEOUT and the kernel returns.  Process-wide; default 1e9
 * (one second); values below 1000 are raised to 1000. */
MEP_API void mep_set_wait_limit_ns(uint64_t ns);
MEP_API uint64_t mep_get_wait_limit_ns(void);

/* MEP_VERSION of the built library. */
MEP_API int32_t mep_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MEP_H */
