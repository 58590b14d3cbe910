// Plan kernel: T_e, maxvio, expert offsets, the stable counting-sort scatter
// and the R-way cut into (rank, expert) segments, in one cooperative launch.
//
// The method (MoonEP release page "Moonshot AI Open-Sources MoonEP, the
// Library Used to Train the MoE Model Kimi K3"):
//   * "Why expert parallelism is needed": the skew metric
//     maxvio = max_e(T_e / T-bar) - 1;
//   * "How MoonEP works": each rank's share is fixed at S*K slots, and a few
//     duplicate experts are placed per step from that step's routing;
//   * "Why this matters to engineers": each row goes directly to its final,
//     expert-ordered slot in a buffer of fixed shape, without a host round trip.
// The schedule is the stable sort of (token, k) pairs by (expert, g, k) cut
// into R chunks of S*K.
//
// Structure.  The pairs are split into nt contiguous tiles, each tile into
// 32 contiguous warp ranges.  With more than one tile the grid is nt + 1
// co-resident blocks: block 0 is a coordinator that owns no pairs and builds
// the plan's tables while the others scatter; with one tile a single block
// does everything and the grid barriers reduce to __syncthreads.
//   Phase 1  every warp counts its range into a warp-private histogram in
//            shared memory (shared-memory atomics: only the warp's own lanes
//            contend) and parks its ids in shared memory; the block turns the
//            32 warp histograms into per-warp exclusive offsets and publishes
//            its tile total per expert to tile[e][t].
//   -- grid barrier --
//   Phase 2  one warp per expert scans its row tile[e][0..nt) into exclusive
//            per-tile offsets and writes T_e.
//   -- grid barrier --
//            When the tile matrix is small (at most 8 entries per thread)
//            every block instead reads all of it and sums T_e and its own
//            tile offsets itself: no second grid barrier, no write-back of
//            the matrix.
//   Phase 3  every block scans T_e over experts (expert offsets); the
//            coordinator writes maxvio, the offsets, segments, CSR pointers
//            and replica list; every tile warp walks its ids again in (g, k)
//            order and gives each pair its position in the expert-sorted
//            order, off_e + tile offset + warp offset + rank among equal ids
//            earlier in the warp.  The rank comes from a peer mask (ballots
//            on the 11 id bits: the lanes holding the same id) and one
//            population count of the peers below the lane; the last peer
//            moves the warp's cursor.  The contiguous plan's slot is that
//            position; the home-first plan maps it through per-expert and
//            per-rank tables every block derives; the capped plan keeps it in
//            slot, and after one more grid barrier (while the coordinator,
//            which built the capped tables meanwhile, writes the segment
//            table) maps it through the tables the coordinator published.
//            This loop bounds phase 3 on large workloads (~0.8 us per 32-pair
//            step of the 32 warps on the Kimi shape); removing its scattered
//            src_pair stores saved ~2 of its ~11 us (measured in a timing
//            copy), and staging them through shared memory was slower.
// A warp whose range exceeds its shared-memory id buffer reads its ids again
// from global memory (L2 hits) in phase 3.
#include <atomic>
#include <climits>
#include <cstdint>
#include <mutex>

#include "mep_device.cuh"
#include "mep_internal.h"

namespace mep {

namespace {

constexpr int kThreads = kPlanThreads;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;          // 32-pair chunks a warp loads at once
constexpr int kTab = MEP_MAX_EXPERTS + 1;
constexpr int kDirectLoads = 8;  // tile-matrix entries per thread in the direct phase 2

#ifndef MEP_PLAN_PEERS_BALLOT
#define MEP_PLAN_PEERS_BALLOT 2  // 2: peer masks from ballots on all 11 id bits, unrolled;
                                 // 1: the same over the id's nbits, in a loop; 0: match.any
#endif

struct PlanParams {
  const int32_t *idx;
  int32_t R, S, E, K;
  int64_t NK, SK;
  int32_t nb;    // blocks
  int32_t nt;    // tiles (nb - 1 with a coordinator, else 1)
  int64_t ppb;   // pairs per tile
  int32_t full;  // 0: counts + maxvio only
  int32_t kind;  // kPlanContiguous, kPlanHomeFirst or kPlanCapped
  int32_t *counts, *expert_offset, *slot, *src_pair;
  int4 *seg;
  int32_t *rank_seg_ptr, *expert_seg_ptr, *replica_seg, *rank_seg_idx;
  int32_t *num_seg, *num_replicas, *max_count, *status;
  double *maxvio;
  int32_t *tile;   // workspace [E][nt]
  uint32_t *bar;   // workspace barrier words
  uint64_t wait_ns;
  // one rank's share (mep_plan_rank): the tiles cover that rank's own pairs,
  // global pairs [pair0, pair0 + NKt); T_e and the rank prefix come from the
  // gathered per-rank histograms
  int64_t pair0;               // global index of the first pair the tiles cover
  int64_t NKt;                 // pairs the tiles cover (NK for the whole range)
  const int32_t *rank_counts;  // [R][E] per-rank histograms, or nullptr
  int32_t rank;                // the rank whose pairs the tiles cover
  int32_t *totals;             // [E] tile totals of phase 2 (p.counts, or workspace)
  // capped plan
  int32_t B;                   // replica experts a rank may host
  int32_t *max_rank_replicas;  // [1] out
  int32_t *tab;                // workspace: the scatter tables the coordinator publishes
};

// Mask of the lanes whose key equals this lane's key; keys are < 2^nbits
// (nbits <= 11, E <= 1024).
__device__ __forceinline__ unsigned peers_of(int key, int nbits) {
#if MEP_PLAN_PEERS_BALLOT == 2
  // bits at and above nbits are zero in every key: their ballots change nothing
  (void)nbits;
  unsigned m = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < 11; ++b) {
    const unsigned bit = (unsigned)(key >> b) & 1u;
    const unsigned on = __ballot_sync(0xffffffffu, bit);
    m &= ~(on ^ (0u - bit));  // lanes whose bit b equals this lane's
  }
  return m;
#elif MEP_PLAN_PEERS_BALLOT
  unsigned m = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned on = __ballot_sync(0xffffffffu, bit);
    m &= bit ? on : ~on;
  }
  return m;
#else
  (void)nbits;
  return __match_any_sync(0xffffffffu, key);
#endif
}

// Exclusive prefix sum of one value per thread over the block; *total gets the
// block sum.  Uses s_w[32]; every thread of the block must call it.
__device__ __forceinline__ int block_excl_scan(int v, int *total, int *s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_w[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = s_w[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_w[lane] = w;
  }
  __syncthreads();
  const int before = warp ? s_w[warp - 1] : 0;
  *total = s_w[kWarps - 1];
  __syncthreads();
  return before + x - v;
}

// block_excl_scan for 64-bit values (two int-sized sums packed in one), with
// its own shared words.
__device__ __forceinline__ long long block_excl_scan64(long long v, long long *total) {
  __shared__ long long s_w64[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_w64[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = s_w64[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    s_w64[lane] = w;
  }
  __syncthreads();
  const long long before = warp ? s_w64[warp - 1] : 0;
  *total = s_w64[kWarps - 1];
  __syncthreads();
  return before + x - v;
}

__device__ __forceinline__ int block_max(int v, int *s_w) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) s_w[warp] = v;
  __syncthreads();
  int m = s_w[0];
  for (int w = 1; w < kWarps; ++w) m = max(m, s_w[w]);
  __syncthreads();
  return m;
}

// First index i in [0, n) with a[i] > x (n if none); a nondecreasing.
__device__ __forceinline__ int upper_bound_idx(const int *a, int n, int x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] <= x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Slot of the i-th pair (in (g,k) order) of expert e in the home-first plan.
// s_rf[e] is the first rank of e's overflow; the pair's rank, the first r
// with D[r+1] > q, is found by stepping from there (an expert's overflow
// spans few ranks).
__device__ __forceinline__ int home_first_slot(int e, int i, int Bx, int C, int R, const int *s_h,
                                               const int *s_off, const int *s_O, const int *s_F,
                                               const int *s_D, const int *s_rf) {
  const int h = s_h[e];
  const int home = e / Bx;
  if (i < h) return home * C + (s_off[e] - s_off[home * Bx]) + i;
  const int q = s_O[e] + (i - h);
  int r = s_rf[e];
  while (r < R - 1 && s_D[r + 1] <= q) ++r;
  return r * C + s_F[r] + (q - s_D[r]);
}

// Slot of the i-th pair (in (g,k) order) of expert e in the capped plan: the
// first h_e pairs go home, the others to the piece holding overflow index
// q = i - h_e (pieces of e in creation order, first overflow indices
// ascending: a binary search).
__device__ __forceinline__ int capped_slot(int e, int i, const int *s_h, const int *s_hb,
                                           const int *s_pb, const int *s_pq, const int *s_pbase) {
  const int h = s_h[e];
  if (i < h) return s_hb[e] + i;
  const int q = i - h;
  int lo = s_pb[e], hi = s_pb[e + 1];
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pq[mid] <= q) lo = mid; else hi = mid;
  }
  return s_pbase[lo] + q;
}

// One compare-exchange of a bitonic network, seen from position i: the key
// it keeps against its partner's key y at distance j in merge size k.
template <typename Key>
__device__ __forceinline__ Key bitonic_keep(Key x, Key y, int i, int j, int k) {
  const bool keep_min = ((i & k) == 0) == ((i & j) == 0);
  const bool lt = x < y;
  return keep_min == lt ? x : y;
}

// Ascending bitonic sort of n2 keys (n2 a power of two, n2 <= blockDim.x)
// held in registers, one per thread (position = thread index).  Steps with a
// partner inside the warp exchange by shuffle; longer ones go through shared
// memory (buf: 2 * n2 keys, double-buffered, one barrier per step).  Every
// thread of the block calls it; positions >= n2 are ignored.
template <typename Key>
__device__ void block_sort_regs(Key &x, int n2, Key *buf) {
  const int t = threadIdx.x;
  int cur = 0;
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      Key y;
      if (j >= 32) {
        Key *b = buf + cur * n2;
        if (t < n2) b[t] = x;
        __syncthreads();
        y = t < n2 ? b[t ^ j] : x;
        cur ^= 1;
      } else {
        y = __shfl_xor_sync(0xffffffffu, x, j);
      }
      x = bitonic_keep(x, y, t, j, k);
    }
  }
}

// Last index i in [0, n) with a[i] <= x (a nondecreasing, a[0] <= x).
__device__ __forceinline__ int last_le(const int *a, int n, int x) {
  return upper_bound_idx(a, n, x) - 1;
}

// Words of the capped plan's scatter tables in the workspace (published by
// the coordinator): per expert the pairs kept home h_e, the home slot base
// and the first of its replica pieces; per piece its first overflow index
// and its slot base (slot = base + overflow index).
__host__ __device__ __forceinline__ int64_t capped_tab_words(int E, int R) {
  return 3 * (int64_t)E + 1 + 2 * ((int64_t)E + R);
}

// Shared-memory ints the capped builder uses: 13 E + 9 R + 6 (E + R) + 8,
// plus two sort buffers of n2 8-byte keys (n2 the power of two at or above
// the items and rooms, who number at most E).  The coordinator's dynamic shared
// memory holds kWarps * (E + kPlanIdsPerWarp) ints, which is more for every
// E <= MEP_MAX_EXPERTS (R <= E); the launch checks it.
__host__ __device__ __forceinline__ int64_t capped_smem_ints(int E, int R) {
  int64_t n2 = 1;  // sort size bound: the power of two at or above E (items + rooms <= E)
  while (n2 < (int64_t)E) n2 <<= 1;
  return 13 * (int64_t)E + 9 * (int64_t)R + 6 * ((int64_t)E + R) + 8 + 4 * n2;
}

// The capped builder's arrays in the coordinator's shared memory.
struct CapMem {
  int *sT;        // [E] T_e
  int *sh;        // [E] h_e, pairs kept home
  int *shb;       // [E] home slot base of e
  int *shf;       // [E] home pieces of the experts before e
  int *spb;       // [E+1] first replica piece of e
  int *shl;       // [E] index of e's home piece among its rank's segments
  int *it_e;      // [E] expert of item i (items: overflow descending, expert ascending)
  int *it_O;      // [E] overflow of item i
  int *it_loc;    // [E] filler: start in its room's replica area, else -1
  int *it_P;      // [E] stream position of item i
  int *it_s;      // [E] stream index, or a filler's index in its room
  int *it_of;     // [E] item index of expert e, -1 if e has no overflow
  int *st_i;      // [E] item at stream index s
  int *rm_r;      // [R] rank of room j (rooms: spare room descending, rank ascending)
  int *rm_D;      // [R] spare room
  int *rm_left;   // [R] space left after the fillers
  int *rm_nf;     // [R] fillers placed
  int *rm_Q;      // [R] stream position of room j's space left; then rank_seg_ptr
  int *rm_first;  // [R] stream index of the first item meeting room j
  int *rm_nz;     // [R+1] rooms with space left before room j
  int *rk_nh;     // [R] home pieces of rank r
  int *rk_nr;     // [R] replica pieces of rank r
  int *pc_e, *pc_r, *pc_loc, *pc_n, *pc_q, *pc_li;  // [E+R] per piece: expert, rank,
                  // first slot within the rank, size, first overflow index, index
                  // among the rank's segments (slot order)
  int *misc;      // [4]: home pieces, replica pieces
  uint64_t *keys; // [n2] sorted items and rooms (aliases the piece arrays)
  uint64_t *sbuf; // [2 n2] sort exchange buffers
};

__device__ __forceinline__ CapMem cap_mem(int *sm, int E, int R) {
  CapMem m;
  const int NP = E + R;
  int *q = sm;
  m.sT = q; q += E;
  m.sh = q; q += E;
  m.shb = q; q += E;
  m.shf = q; q += E;
  m.spb = q; q += E + 1;
  m.shl = q; q += E;
  m.it_e = q; q += E;
  m.it_O = q; q += E;
  m.it_loc = q; q += E;
  m.it_P = q; q += E;
  m.it_s = q; q += E;
  m.it_of = q; q += E;
  m.st_i = q; q += E;
  m.rm_r = q; q += R;
  m.rm_D = q; q += R;
  m.rm_left = q; q += R;
  m.rm_nf = q; q += R;
  m.rm_Q = q; q += R;
  m.rm_first = q; q += R;
  m.rm_nz = q; q += R + 1;
  m.rk_nh = q; q += R;
  m.rk_nr = q; q += R;
  m.misc = q; q += 4;
  q = reinterpret_cast<int *>((reinterpret_cast<uintptr_t>(q) + 7) & ~static_cast<uintptr_t>(7));
  m.keys = reinterpret_cast<uint64_t *>(q);  // X + Y <= E keys: inside the 6 NP piece ints
  m.pc_e = q; q += NP;
  m.pc_r = q; q += NP;
  m.pc_loc = q; q += NP;
  m.pc_n = q; q += NP;
  m.pc_q = q; q += NP;
  m.pc_li = q; q += NP;
  m.sbuf = reinterpret_cast<uint64_t *>(q);  // even offset from the aligned base
  return m;
}

// Keys of the one sort of step 2: items (overflowing experts) first by
// overflow descending, then expert; rooms (ranks with spare room) after them
// by room descending, then rank.
__device__ __forceinline__ uint64_t item_key(int O, int e) {
  return ((uint64_t)(0x7fffffff - O) << 32) | (uint32_t)e;
}
__device__ __forceinline__ uint64_t room_key(int D, int r) {
  return (1ull << 63) | ((uint64_t)(0x7fffffff - D) << 32) | (uint32_t)r;
}

// Sorts the X items and Y rooms of keys[0, X + Y) (n2 >= X + Y, n2 <=
// blockDim.x) and writes the item and room tables.
__device__ __forceinline__ void capped_sort_and_decode(const CapMem &m, int n2, int X, int Y) {
  const int t = threadIdx.x;
  uint64_t x = t < X + Y ? m.keys[t] : ~0ull;
  block_sort_regs<uint64_t>(x, n2, m.sbuf);
  const int id = (int)(x & 0xffffffffu);
  const int v = 0x7fffffff - (int)((x >> 32) & 0x7fffffff);
  if (t < X) {
    m.it_e[t] = id;
    m.it_O[t] = v;
    m.it_of[id] = t;
    m.it_loc[t] = -1;
  } else if (t < X + Y) {
    m.rm_r[t - X] = id;
    m.rm_D[t - X] = v;
  }
}

// The capped schedule's scatter tables, built by the coordinator block (which
// owns no pairs, so its dynamic shared memory is free scratch).  T is this
// thread's expert count (t < E), s_off the expert offsets.  Writes
// max_rank_replicas and publishes the scatter tables to p.tab; the segment
// table follows in capped_segments, after the grid barrier that releases the
// tile blocks.
//   1. home fill, smallest home experts first (ties: lower id): each expert
//      sums the counts of the experts filled before it in its home block;
//   2. items (overflowing experts, overflow descending) and rooms (ranks with
//      spare room, room descending), compacted and sorted together;
//   3. fillers (items below the largest room): filler f is offered to room
//      f mod Y in round f / Y < B - 2, placed whole if it fits -- one thread
//      per room walks its candidates;
//   4. the stream: items not placed, cut over the rooms' space left, by
//      prefix sums and binary searches; the pieces, expert by expert.
__device__ void capped_tables(const PlanParams &p, int T, const int *s_off, int *sm, int *s_w) {
  const int t = threadIdx.x;
  const int E = p.E, R = p.R, C = (int)p.SK, Bh = E / R;
  const int NP = E + R;  // bound on replica pieces (at most E + R - 1)
  const CapMem m = cap_mem(sm, E, R);
  int tot;

  // ---- 1. home fill, smallest home experts first --------------------------
  if (t < E) {
    m.sT[t] = T;
    m.it_of[t] = -1;
  }
  __syncthreads();
  const int b0 = t < E ? (t / Bh) * Bh : 0;
  int h = 0;
  if (t < E) {
    int pre = 0;  // pairs of the home experts filled before e
    if (R > 1) {
      for (int e2 = b0; e2 < b0 + Bh; ++e2) {
        const int v = m.sT[e2];
        pre += (v < T || (v == T && e2 < t)) ? v : 0;
      }
    }
    // with one rank every pair fits at home
    h = R == 1 ? T : max(0, min(T, C - pre));
    m.sh[t] = h;
  }
  const int O = t < E ? T - h : 0;
  // spare room of rank t: its home load is s_off over its block
  const int Dr = t < R ? C - min(s_off[(t + 1) * Bh] - s_off[t * Bh], C) : 0;
  __syncthreads();
  if (t < E) {
    int hx = 0, hn = 0;  // home pairs and home pieces of the block's experts before e
    for (int e2 = b0; e2 < t; ++e2) {
      const int v = m.sh[e2];
      hx += v;
      hn += v > 0 ? 1 : 0;
    }
    m.shb[t] = (t / Bh) * C + hx;
    m.shl[t] = hn;
    if (t == b0 + Bh - 1) m.rk_nh[t / Bh] = hn + (h > 0 ? 1 : 0);
  }

  // ---- 2. items and rooms, compacted and sorted in one pass ----------------
  const int isx = (t < E && O > 0) ? 1 : 0, isy = (t < R && Dr > 0) ? 1 : 0;
  const int cpos = block_excl_scan(isx | (isy << 16), &tot, s_w);
  const int X = tot & 0xffff, Y = tot >> 16;
  if (isx) m.keys[cpos & 0xffff] = item_key(O, t);
  if (isy) m.keys[X + (cpos >> 16)] = room_key(Dr, t);
  __syncthreads();
  // X + Y <= E <= kThreads: an overflowing expert's home rank is full, so the
  // items come from full ranks (E/R experts each) and the rooms are the
  // other ranks -- X + Y <= (E/R) F + (R - F) <= E for F full ranks.
  int n2 = 1;
  while (n2 < X + Y) n2 <<= 1;
  if (n2 > kThreads) {  // unreachable by the bound above; never sorted partially
    if (t == 0) set_status(p.status, MEP_ERR_DEVICE_DATA);
    n2 = kThreads;
  }
  capped_sort_and_decode(m, n2, min(X, kThreads), min(Y, kThreads - min(X, kThreads)));
  __syncthreads();

  // ---- 3. fillers ----------------------------------------------------------
  const int dmax = Y > 0 ? m.rm_D[0] : 0;
  int i0 = 0;  // items at least dmax: the first index with it_O < dmax
  {
    int lo = 0, hi = X;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (m.it_O[mid] >= dmax) lo = mid + 1; else hi = mid;
    }
    i0 = lo;
  }
  const int nf = X - i0;
  if (t < Y) {
    int left = m.rm_D[t], cnt = 0;
    for (int round = 0; round < p.B - 2; ++round) {
      const int f = t + round * Y;
      if (f >= nf) break;
      const int i = i0 + f;
      if (m.it_O[i] <= left) {
        m.it_loc[i] = m.rm_D[t] - left;
        m.it_s[i] = cnt;  // index among the room's fillers
        left -= m.it_O[i];
        ++cnt;
      }
    }
    m.rm_left[t] = left;
    m.rm_nf[t] = cnt;
  }
  __syncthreads();

  // ---- 4. the stream -------------------------------------------------------
  // stream items: overflow prefix P and index; rooms: space-left prefix Q and
  // the count of rooms with space left before (each pair packed in one scan;
  // prefixes < 2^31, counts < 2^16)
  const bool ins = t < X && m.it_loc[t] < 0;
  const int left_t = t < Y ? m.rm_left[t] : 0;
  long long tot64;
  const long long pq = block_excl_scan64(
      (long long)(ins ? m.it_O[t] : 0) | ((long long)left_t << 32), &tot64);
  const int cnts = block_excl_scan((ins ? 1 : 0) | ((left_t > 0 ? 1 : 0) << 16), &tot, s_w);
  const int ns_items = tot & 0xffff;
  if (ins) {
    m.it_P[t] = (int)(pq & 0xffffffffll);
    m.it_s[t] = cnts & 0xffff;
    m.st_i[cnts & 0xffff] = t;
  }
  if (t < Y) {
    m.rm_Q[t] = (int)(pq >> 32);
    m.rm_nz[t] = cnts >> 16;
  }
  if (t == 0) m.rm_nz[Y] = tot >> 16;
  __syncthreads();
  // stream index of the first item meeting room j, and the stream items that
  // meet it
  int nrep_j = 0;
  if (t < Y) {
    int nst = 0;
    if (m.rm_left[t] > 0) {
      int lo = 0, hi = ns_items;  // last s with P(st_i[s]) <= Q
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (m.it_P[m.st_i[mid]] <= m.rm_Q[t]) lo = mid; else hi = mid;
      }
      m.rm_first[t] = lo;
      int lo2 = lo, hi2 = ns_items;  // last s with P(st_i[s]) <= Q + left - 1
      const int last = m.rm_Q[t] + m.rm_left[t] - 1;
      while (hi2 - lo2 > 1) {
        const int mid = (lo2 + hi2) >> 1;
        if (m.it_P[m.st_i[mid]] <= last) lo2 = mid; else hi2 = mid;
      }
      nst = lo2 - lo + 1;
    }
    nrep_j = m.rm_nf[t] + nst;
  }
  __syncthreads();
  // pieces of expert t: its filler, or its stream pieces
  int npc = 0, j0 = 0, j1 = -1;
  const int it = t < E ? m.it_of[t] : -1;
  if (it >= 0) {
    if (m.it_loc[it] >= 0) {
      npc = 1;
    } else {
      const int a = m.it_P[it], b = a + m.it_O[it];
      j0 = last_le(m.rm_Q, Y, a);
      j1 = last_le(m.rm_Q, Y, b - 1);
      npc = m.rm_nz[j1 + 1] - m.rm_nz[j0];
    }
  }
  // replica pieces before e, and home pieces before e (both < 2^16)
  const int pc = block_excl_scan(npc | ((t < E && h > 0 ? 1 : 0) << 16), &tot, s_w);
  const int pb = pc & 0xffff, npieces = tot & 0xffff;
  if (t < E) {
    m.spb[t] = pb;
    m.shf[t] = pc >> 16;
  }
  if (t == 0) {
    m.spb[E] = npieces;
    m.misc[0] = tot >> 16;  // home pieces
    m.misc[1] = npieces;
  }
  if (t < R) m.rk_nr[t] = 0;
  if (it >= 0 && pb + npc <= NP) {  // at most E + R - 1 pieces by construction
    const int e = t;
    if (m.it_loc[it] >= 0) {
      const int j = (it - i0) % Y;
      const int r = m.rm_r[j];
      m.pc_e[pb] = e;
      m.pc_r[pb] = r;
      m.pc_loc[pb] = (C - m.rm_D[j]) + m.it_loc[it];
      m.pc_n[pb] = m.it_O[it];
      m.pc_q[pb] = 0;
      m.pc_li[pb] = m.rk_nh[r] + m.it_s[it];
    } else {
      const int a = m.it_P[it], b = a + m.it_O[it];
      int q = pb;
      for (int j = j0; j <= j1; ++j) {
        if (m.rm_left[j] == 0) continue;
        const int r = m.rm_r[j];
        const int lo = max(a, m.rm_Q[j]), hi = min(b, m.rm_Q[j] + m.rm_left[j]);
        m.pc_e[q] = e;
        m.pc_r[q] = r;
        m.pc_loc[q] = (C - m.rm_D[j]) + (m.rm_D[j] - m.rm_left[j]) + (lo - m.rm_Q[j]);
        m.pc_n[q] = hi - lo;
        m.pc_q[q] = lo - a;
        m.pc_li[q] = m.rk_nh[r] + m.rm_nf[j] + (m.it_s[it] - m.rm_first[j]);
        ++q;
      }
    }
  }
  __syncthreads();
  if (t < Y) m.rk_nr[m.rm_r[t]] = nrep_j;
  const int mx = block_max(nrep_j, s_w);  // syncs
  if (t == 0 && p.max_rank_replicas != nullptr) *p.max_rank_replicas = mx;
  // publish the scatter tables
  int *tab_h = p.tab, *tab_hb = tab_h + E, *tab_pb = tab_hb + E;
  int *tab_pq = tab_pb + E + 1, *tab_pbase = tab_pq + NP;
  if (t < E) {
    __stcg(tab_h + t, m.sh[t]);
    __stcg(tab_hb + t, m.shb[t]);
    __stcg(tab_pb + t, pb);
  }
  if (t == 0) __stcg(tab_pb + E, npieces);
  for (int q = t; q < npieces; q += kThreads) {
    __stcg(tab_pq + q, m.pc_q[q]);
    __stcg(tab_pbase + q, m.pc_r[q] * C + m.pc_loc[q] - m.pc_q[q]);
  }
}

// The capped plan's segment table, by (expert, rank), from the builder's
// arrays (the coordinator, after the tables are published).  An expert's
// segments are its home piece and its replica pieces in rank order; a
// piece's place among them is the number of the expert's pieces on lower
// ranks.  Also writes rank_seg_ptr, rank_seg_idx, replica_seg,
// expert_seg_ptr, num_seg and num_replicas.
__device__ void capped_segments(const PlanParams &p, int *sm, int *s_w) {
  const int t = threadIdx.x;
  const int E = p.E, R = p.R, C = (int)p.SK, Bh = E / R;
  const CapMem m = cap_mem(sm, E, R);
  const int nhome = m.misc[0], npieces = m.misc[1];
  int rtot;
  const int rsp = block_excl_scan(t < R ? m.rk_nh[t] + m.rk_nr[t] : 0, &rtot, s_w);
  if (t < R) {
    p.rank_seg_ptr[t] = rsp;
    m.rm_Q[t] = rsp;  // rank_seg_ptr (rm_Q is no longer needed)
  }
  if (t == 0) p.rank_seg_ptr[R] = rtot;
  __syncthreads();
  const int lim = E + R - 1;  // rank_seg_idx entries
  for (int e = t; e < E; e += kThreads) {
    const int b = m.spb[e], n = m.spb[e + 1] - b;
    const int base = m.shf[e] + b;  // segments of the experts before e
    p.expert_seg_ptr[e] = base;
    const int h = m.sh[e];
    if (h > 0) {
      const int home = e / Bh;
      int lower = 0;
      for (int q = b; q < b + n; ++q) lower += m.pc_r[q] < home ? 1 : 0;
      const int a = base + lower;
      p.seg[a] = make_int4(e, home, m.shb[e] - home * C, h);
      const int at = m.rm_Q[home] + m.shl[e];
      if (at >= 0 && at < lim) p.rank_seg_idx[at] = a;
    }
  }
  for (int q = t; q < npieces; q += kThreads) {
    const int e = m.pc_e[q], r = m.pc_r[q];
    const int b = m.spb[e], n = m.spb[e + 1] - b;
    int lower = 0;
    for (int q2 = b; q2 < b + n; ++q2) lower += m.pc_r[q2] < r ? 1 : 0;
    const int a = m.shf[e] + b + lower + ((m.sh[e] > 0 && e / Bh < r) ? 1 : 0);
    p.seg[a] = make_int4(e, r, m.pc_loc[q], m.pc_n[q]);
    const int at = m.rm_Q[r] + m.pc_li[q];
    if (at >= 0 && at < lim) p.rank_seg_idx[at] = a;
    p.replica_seg[b + lower] = a;  // replicas in table order
  }
  if (t == 0) {
    p.expert_seg_ptr[E] = nhome + npieces;
    *p.num_seg = nhome + npieces;
    *p.num_replicas = npieces;
  }
}

__device__ __forceinline__ bool plan_sync(const PlanParams &p, int k) {
  if (p.nb == 1) {
    __syncthreads();
    return true;
  }
  return grid_barrier(p.bar, k * p.nb, p.wait_ns, p.status);
}

__global__ void __launch_bounds__(kThreads, 1) plan_kernel(PlanParams p) {
  extern __shared__ int smem[];  // [kWarps][E] histograms / cursors, then [kWarps][kPlanIdsPerWarp] ids
  __shared__ int s_w[32];
  // Tables over experts (or ranks), E + 1 <= kTab entries each.
  __shared__ int s_tab[8][kTab];
  __shared__ int s_rank[MEP_MAX_RANKS];  // home-first coordinator: per-rank index base
  __shared__ int s_rf[MEP_MAX_EXPERTS];  // home-first: first rank of each expert's overflow
  int *s_off = s_tab[0];   // expert offsets (exclusive prefix of T_e), [E] = total

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int E = p.E;
  const int nbits = 32 - __clz(E);          // 2^nbits > E
  const int sentinel = (1 << nbits) - 1;    // key of an empty or invalid lane
  const bool coord = p.nb > 1 && blockIdx.x == 0;
  const int tile = p.nb > 1 ? (int)blockIdx.x - 1 : 0;
  if (blockIdx.x == 0 && t == 0) *p.status = 0;

  int *wh_all = smem;
  int *wh = wh_all + warp * E;
  int *ids = smem + kWarps * E + warp * kPlanIdsPerWarp;
  for (int i = t; i < kWarps * E; i += kThreads) wh_all[i] = 0;
  __syncthreads();

  // Tile and warp ranges (the coordinator has none).
  const int64_t b0 = coord ? 0 : (int64_t)tile * p.ppb;
  const int64_t b1 = coord ? 0 : min(b0 + p.ppb, p.NKt);
  const int64_t n = b1 > b0 ? b1 - b0 : 0;
  const int64_t w0 = b0 + (n * warp) / kWarps;
  const int64_t w1 = b0 + (n * (warp + 1)) / kWarps;
  const bool keep = (w1 - w0) <= kPlanIdsPerWarp;  // ids stay in shared memory
  // 32-bit indices inside the warp's range (NK < 2^31 by the shape rules).
  const int nw = (int)(w1 - w0);
  const int32_t *idx_w = p.idx + w0;

  // ---- phase 1: warp-private histograms ------------------------------------
  bool bad = false;
  for (int c = 0; c < nw; c += 32 * kBatch) {
    int ev[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = c + u * 32 + lane;
      ev[u] = i < nw ? __ldg(idx_w + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = c + u * 32 + lane;
      if (i < nw) {
        const int e = ev[u];
        if ((unsigned)e < (unsigned)E) atomicAdd(wh + e, 1); else bad = true;
        if (keep) ids[i] = e;
      }
    }
  }
  __syncthreads();
  if (t < E) {  // per-warp exclusive offsets inside the tile; tile total
    int run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int v = wh_all[w * E + t];
      wh_all[w * E + t] = run;
      run += v;
    }
    if (!coord) __stcg(p.tile + (int64_t)t * p.nt + tile, run);
  }
  bad = __syncthreads_or(bad);

  if (!plan_sync(p, 1)) return;
  if (bad && t == 0) set_status(p.status, MEP_ERR_DEVICE_DATA);

  // ---- phase 2: per-expert scan over tiles ----------------------------------
  int tpe = 32;  // direct form: threads per expert, a power of two (groups inside a warp)
  while (tpe > 1 && tpe * E > kThreads) tpe >>= 1;
  const bool direct = p.nb > 1 && p.nt <= kDirectLoads * tpe;
  int *s_T = s_tab[5], *s_pre = s_tab[6];  // direct form: T_e, this tile's offsets
  if (direct) {
    const int e = t / tpe, sub = t % tpe;
    const int32_t *row = p.tile + (int64_t)min(e, E - 1) * p.nt;
    int v[kDirectLoads];
#pragma unroll
    for (int j = 0; j < kDirectLoads; ++j) {  // all loads in flight together
      const int b = sub + j * tpe;
      v[j] = (e < E && b < p.nt) ? __ldcg(row + b) : 0;
    }
    int tot = 0, pre = 0;
#pragma unroll
    for (int j = 0; j < kDirectLoads; ++j) {
      tot += v[j];
      if (sub + j * tpe < tile) pre += v[j];
    }
    for (int o = tpe >> 1; o > 0; o >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
      pre += __shfl_xor_sync(0xffffffffu, pre, o);
    }
    if (e < E && sub == 0) {
      s_T[e] = tot;
      s_pre[e] = pre;
    }
    __syncthreads();
  } else {
    const int per = (p.nt + 31) / 32;  // tiles per lane, <= 32
    for (int e = blockIdx.x * kWarps + warp; e < E; e += p.nb * kWarps) {
      int32_t *row = p.tile + (int64_t)e * p.nt;
      const int lo = min(lane * per, p.nt), hi = min(lo + per, p.nt);
      int v[8];
      int s = 0;
      if (per <= 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = lo + j < hi ? __ldcg(row + lo + j) : 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) s += v[j];
      } else {
        for (int b = lo; b < hi; ++b) s += __ldcg(row + b);
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (p.full) {
        int run = incl - s;
        if (per <= 8) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (lo + j < hi) {
              __stcg(row + lo + j, run);
              run += v[j];
            }
          }
        } else {
          for (int b = lo; b < hi; ++b) {
            const int x = __ldcg(row + b);
            __stcg(row + b, run);
            run += x;
          }
        }
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) __stcg(p.totals + e, total);
    }
  }

  if (!direct && !plan_sync(p, 2)) return;

  // ---- phase 3: offsets, scalars, segments, scatter -------------------------
  // Both loads issued together: one L2 round trip before the scans.
  const int Tt = t < E ? (direct ? s_T[t] : __ldcg(p.totals + t)) : 0;
  int tile_off =
      (p.full && !coord && t < E)
          ? (direct ? s_pre[t] : __ldcg(p.tile + (int64_t)t * p.nt + tile))
          : 0;
  int T = Tt;
  if (p.rank_counts != nullptr) {
    // One rank's share: T_e is the sum of the ranks' histograms, and the
    // rank's pairs of e follow those of the ranks before it (g = r*S + s is
    // rank-major).  The rank's own row must match what its tiles counted.
    int sum = 0, before = 0;
    bool mismatch = false;
    if (t < E) {
      for (int r = 0; r < p.R; ++r) {
        const int v = __ldg(p.rank_counts + (int64_t)r * E + t);
        if (r < p.rank) before += v;
        if (r == p.rank && v != Tt) mismatch = true;
        sum += v;
      }
    }
    T = sum;
    tile_off += before;
    if (mismatch) set_status(p.status, MEP_ERR_DEVICE_DATA);
  }
  if ((direct || p.rank_counts != nullptr) && blockIdx.x == 0 && t < E) p.counts[t] = T;
  int total;
  const int off = block_excl_scan(T, &total, s_w);
  if (t < E) s_off[t] = off;
  if (t == 0) s_off[E] = total;
  __syncthreads();

  if (blockIdx.x == 0) {
    const int mx = block_max(T, s_w);
    if (t == 0) {
      if (p.max_count != nullptr) *p.max_count = mx;
      if (p.maxvio != nullptr) *p.maxvio = (double)((long long)mx * E) / (double)p.NK - 1.0;
    }
  }

  const int C = (int)p.SK;  // slots per rank
  const int Bx = E / p.R;   // home experts per rank
  // Home-first tables, built by every block (they are small): per expert the
  // pairs kept home h_e and their start pre_e on the home rank, the overflow
  // prefix O_e and the count of overflowing / home-keeping experts before e;
  // per rank its home fill F_r and the prefix D_r of the spare room.
  int *s_h = s_tab[1], *s_O = s_tab[2], *s_F = s_tab[3], *s_D = s_tab[4];
  int *s_hp = s_tab[5], *s_op = s_tab[6];
  int h = 0, pre = 0, over = 0;
  if (p.full && p.kind == kPlanHomeFirst) {
    if (t < E) {
      const int before = off - s_off[(t / Bx) * Bx];  // home experts' pairs before e
      h = max(0, min(T, C - before));
      pre = min(before, C);
      over = T - h;
    }
    int otot, hptot = 0, optot = 0;
    const int O = block_excl_scan(over, &otot, s_w);
    // The piece counts before each expert are only needed for the
    // coordinator's tables.
    int hp = 0, op = 0;
    if (blockIdx.x == 0) {  // both counts (<= E < 2^16) in one scan
      int both_tot;
      const int both = block_excl_scan((h > 0 ? 1 : 0) | ((over > 0 ? 1 : 0) << 16), &both_tot, s_w);
      hp = both & 0xffff;
      op = both >> 16;
      hptot = both_tot & 0xffff;
      optot = both_tot >> 16;
    }
    int F = 0, room = 0;
    if (t < p.R) {
      const int load = s_off[(t + 1) * Bx] - s_off[t * Bx];
      F = min(load, C);
      room = C - F;
    }
    int dtot;
    const int D = block_excl_scan(room, &dtot, s_w);
    if (t < E) {
      s_h[t] = h;
      s_O[t] = O;
      s_hp[t] = hp;
      s_op[t] = op;
    }
    if (t < p.R) {
      s_F[t] = F;
      s_D[t] = D;
    }
    if (t == 0) {
      s_O[E] = otot;
      s_hp[E] = hptot;
      s_op[E] = optot;
      s_D[p.R] = dtot;
    }
    __syncthreads();
    if (t < E) s_rf[t] = over > 0 ? upper_bound_idx(s_D + 1, p.R, O) : 0;
    __syncthreads();
  }

  if (p.full && blockIdx.x == 0) {  // the coordinator (or the only block)
    if (p.kind == kPlanContiguous) {
      // Slot positions are < N*K < 2^31: 32-bit arithmetic throughout.
      const int SK = (int)p.SK;
      int *s_sbase = s_tab[1];
      int nseg_e = 0, r0 = 0, r1 = -1;
      if (t < E && T > 0) {
        r0 = (int)((unsigned)off / (unsigned)SK);
        r1 = (int)((unsigned)(off + T - 1) / (unsigned)SK);
        nseg_e = r1 - r0 + 1;
      }
      const int home = t / Bx;
      const int nrep_e = nseg_e - ((nseg_e > 0 && home >= r0 && home <= r1) ? 1 : 0);
      // segment and replica counts (totals <= E + R - 1 < 2^16) in one scan
      int both_tot;
      const int both = block_excl_scan(nseg_e | (nrep_e << 16), &both_tot, s_w);
      const int sbase = both & 0xffff, nseg = both_tot & 0xffff, nrep = both_tot >> 16;
      int rbase = both >> 16;
      if (t < E) {
        s_sbase[t] = sbase;
        p.expert_offset[t] = off;
        p.expert_seg_ptr[t] = sbase;
        for (int j = 0; j < nseg_e; ++j) {
          const int r = r0 + j;
          const int lo = max(off, r * SK);
          const int hi = min(off + T, (r + 1) * SK);
          p.seg[sbase + j] = make_int4(t, r, lo - r * SK, hi - lo);
          p.rank_seg_idx[sbase + j] = sbase + j;  // slot order is table order
          if (r != home) p.replica_seg[rbase++] = sbase + j;
        }
      }
      if (t == 0) {
        s_sbase[E] = nseg;
        p.expert_offset[E] = total;
        p.expert_seg_ptr[E] = nseg;
        *p.num_seg = nseg;
        *p.num_replicas = nrep;
      }
      __syncthreads();
      for (int r = t; r <= p.R; r += kThreads) {
        int ptr = nseg;
        if (r < p.R && r * SK < total) {
          const int e = upper_bound_idx(s_off, E + 1, r * SK) - 1;  // expert holding slot r*SK
          ptr = s_sbase[e] + (r - (int)((unsigned)s_off[e] / (unsigned)SK));
        }
        p.rank_seg_ptr[r] = ptr;
      }
    } else if (p.kind == kPlanHomeFirst) {
      int *s_rsp = s_tab[7];
      const int R = p.R;
      // Per rank: home pieces (home experts keeping pairs) + replica pieces
      // (overflowing experts whose overflow meets the rank's spare room).
      int nh = 0, nr = 0, ef = 0;
      if (t < R) {
        nh = s_hp[(t + 1) * Bx] - s_hp[t * Bx];
        const int d0 = s_D[t], d1 = s_D[t + 1];
        if (d1 > d0) {
          ef = upper_bound_idx(s_O, E + 1, d0) - 1;                 // expert holding d0
          const int el = upper_bound_idx(s_O, E + 1, d1 - 1) - 1;   // expert holding d1 - 1
          nr = s_op[el + 1] - s_op[ef];
        }
      }
      int ntot;
      const int rsp = block_excl_scan(nh + nr, &ntot, s_w);
      if (t < R) {
        s_rsp[t] = rsp;
        // rank t's replica piece of an overflowing expert e sits at
        // s_rank[t] + s_op[e] in its list (after its nh home pieces)
        s_rank[t] = rsp + nh - s_op[ef];
        p.rank_seg_ptr[t] = rsp;
      }
      if (t == 0) {
        s_rsp[R] = ntot;
        p.rank_seg_ptr[R] = ntot;
      }
      __syncthreads();
      // Per expert: its pieces in rank order (the home piece sits among the
      // replica pieces by rank).
      int rf = 0, rl = -1;
      if (t < E && over > 0) {
        const int O = s_O[t];
        rf = s_rf[t];                                        // first rank with D[r+1] > O
        rl = upper_bound_idx(s_D + 1, R, O + over - 1);      // rank holding the last pair
      }
      int nrep_e = 0;
      for (int r = rf; r <= rl; ++r)
        if (s_D[r + 1] > s_D[r]) ++nrep_e;
      const int nseg_e = nrep_e + (h > 0 ? 1 : 0);
      // segment and replica counts (totals <= E + R - 1 < 2^16) in one scan
      int both_tot;
      const int both = block_excl_scan(nseg_e | (nrep_e << 16), &both_tot, s_w);
      const int nseg = both_tot & 0xffff, nrep = both_tot >> 16;
      int sidx = both & 0xffff;
      int ridx = both >> 16;
      if (t < E) {
        const int home = t / Bx;
        p.expert_offset[t] = off;
        p.expert_seg_ptr[t] = sidx;
        const int O = s_O[t];
        bool home_done = h == 0;
        for (int r = rf; r <= rl + 1; ++r) {
          if (!home_done && (r > rl || r > home)) {  // home piece, in rank order
            p.seg[sidx] = make_int4(t, home, pre, h);
            p.rank_seg_idx[s_rsp[home] + (s_hp[t] - s_hp[home * Bx])] = sidx;
            ++sidx;
            home_done = true;
          }
          if (r > rl || s_D[r + 1] <= s_D[r]) continue;
          const int lo = max(O, s_D[r]), hi = min(O + over, s_D[r + 1]);
          p.seg[sidx] = make_int4(t, r, s_F[r] + (lo - s_D[r]), hi - lo);
          p.rank_seg_idx[s_rank[r] + s_op[t]] = sidx;
          p.replica_seg[ridx++] = sidx;
          ++sidx;
        }
      }
      if (t == 0) {
        p.expert_offset[E] = total;
        p.expert_seg_ptr[E] = nseg;
        *p.num_seg = nseg;
        *p.num_replicas = nrep;
      }
    } else {  // kPlanCapped: the coordinator (never a tile block) builds the tables
      if (t < E) p.expert_offset[t] = off;
      if (t == 0) p.expert_offset[E] = total;
      capped_tables(p, T, s_off, smem, s_w);
    }
  }

  // The capped plan's slots come in two passes around one more grid barrier:
  // before it, while the coordinator builds its tables, the tile blocks give
  // each pair its position in the expert-sorted order (kept in slot); after
  // it they turn that position into the slot through the published tables
  // (per expert h_e, its home slot base and first piece; per piece its first
  // overflow index and slot base) while the coordinator writes the segments.
  const bool cap = p.full && p.kind == kPlanCapped;
  const unsigned nk = (unsigned)p.NK;
  int32_t *slot_w = p.slot + p.pair0 + w0;
  const int q0 = (int)(p.pair0 + w0);  // global pair index of the warp's first pair
  if (p.full && !coord) {
    // Per expert: where this tile's pairs start in the expert-sorted order
    // (expert offset + tile offset); wh keeps the warp offsets in the tile.
    int *s_base = s_tab[7];
    __syncthreads();  // a single block has finished the coordinator's tables
    if (t < E) s_base[t] = off + tile_off;
    __syncthreads();

    const bool hf = p.kind == kPlanHomeFirst;
    const unsigned lt = lanemask_lt(), gt = lanemask_gt();
    for (int c = 0; c < nw; c += 32) {
      const int i = c + lane;
      const bool act = i < nw;
      int e = -1;
      if (act) e = keep ? ids[i] : __ldg(idx_w + i);
      const bool valid = (unsigned)e < (unsigned)E;
      const unsigned peers = peers_of(valid ? e : sentinel, nbits);
      const int wo = valid ? wh[e] : 0;
      __syncwarp();
      if (valid) {
        // rank among the tile's pairs of e -- one population count per step:
        // bit counts and leading-one searches go to the narrow XU pipe, which
        // the profile showed as this loop's busiest unit
        const int r = wo + __popc(peers & lt);
        int s = s_base[e] + r;  // position in the expert-sorted order
        if (hf) s = home_first_slot(e, s - s_off[e], Bx, C, p.R, s_h, s_off, s_O, s_F, s_D, s_rf);
        slot_w[i] = s;
        if (!cap && (unsigned)s < nk) p.src_pair[s] = q0 + i;
        if ((peers & gt) == 0) wh[e] = r + 1;  // the last of the peers moves the cursor
      } else if (act) {
        slot_w[i] = -1;
      }
      __syncwarp();
    }
  }
  if (cap) {
    if (!plan_sync(p, direct ? 2 : 3)) return;
    if (coord) {
      capped_segments(p, smem, s_w);
    } else {
      int *s_ch = s_tab[1], *s_chb = s_tab[2], *s_cpb = s_tab[3];
      int *s_cpq = &s_tab[4][0], *s_cpbase = &s_tab[4][0] + 2 * kTab;
      const int *tab_h = p.tab, *tab_hb = tab_h + E, *tab_pb = tab_hb + E;
      const int *tab_pq = tab_pb + E + 1, *tab_pbase = tab_pq + (E + p.R);
      const int npieces = min(__ldcg(tab_pb + E), 2 * kTab);
      for (int i = t; i < E; i += kThreads) {
        s_ch[i] = __ldcg(tab_h + i);
        s_chb[i] = __ldcg(tab_hb + i);
        s_cpb[i] = __ldcg(tab_pb + i);
      }
      if (t == 0) s_cpb[E] = npieces;
      for (int i = t; i < npieces; i += kThreads) {
        s_cpq[i] = __ldcg(tab_pq + i);
        s_cpbase[i] = __ldcg(tab_pbase + i);
      }
      __syncthreads();
      for (int c = 0; c < nw; c += 32 * kBatch) {
        int sv[kBatch], ev[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {  // all loads in flight together
          const int i = c + u * 32 + lane;
          sv[u] = -1;
          ev[u] = 0;
          if (i < nw) {
            sv[u] = slot_w[i];
            ev[u] = keep ? ids[i] : __ldg(idx_w + i);
          }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          if (sv[u] < 0) continue;  // an id out of range (slot -1)
          const int i = c + u * 32 + lane;
          const int e = ev[u];
          const int s = capped_slot(e, sv[u] - s_off[e], s_ch, s_chb, s_cpb, s_cpq, s_cpbase);
          slot_w[i] = s;
          if ((unsigned)s < nk) p.src_pair[s] = q0 + i;
        }
      }
    }
  }
  if (p.nb > 1) grid_barrier_exit(p.bar, p.nb);
}

// Per-device launch constants, shared by host threads.  The shared-memory
// attribute only grows (a launch may ask for less than it allows), and
// max_blocks is the co-resident block count at the largest size asked for,
// a lower bound for every smaller one.  Updates hold the mutex; a launch whose
// size is already allowed only reads the two atomics.
struct PlanDev {
  std::mutex mu;
  std::atomic<int> smem_attr{-1};  // largest dynamic shared memory allowed so far
  std::atomic<int> max_blocks{0};  // co-resident plan blocks (cooperative grid limit)
};

PlanDev g_plan_dev[64];

cudaError_t plan_dev_allow(PlanDev &d, int dev, int smem) {
  std::lock_guard<std::mutex> lock(d.mu);
  if (d.smem_attr.load(std::memory_order_acquire) >= smem) return cudaSuccess;
  cudaError_t err = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  int sms = 0, per_sm = 0;
  if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return err;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, plan_kernel, kThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  d.max_blocks.store(per_sm * sms, std::memory_order_relaxed);
  d.smem_attr.store(smem, std::memory_order_release);
  return cudaSuccess;
}

}  // namespace

size_t plan_workspace_bytes(const mep_shape_t &s) {
  return kPlanWsHeader + (size_t)s.E * kPlanMaxBlocks * sizeof(int32_t);
}

cudaError_t launch_plan(const mep_shape_t &s, const int32_t *idx, const mep_plan_t &pl,
                        int full, int kind, void *ws, uint64_t wait_ns, cudaStream_t stream,
                        const PlanExtra *extra) {
  const PlanExtra none{};
  const PlanExtra &x = extra != nullptr ? *extra : none;
  const bool ranked = x.rank_counts != nullptr;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  PlanDev &d = g_plan_dev[dev];
  const size_t smem = ((size_t)kWarps * s.E + (size_t)kWarps * kPlanIdsPerWarp) * sizeof(int);
  if (d.smem_attr.load(std::memory_order_acquire) < (int)smem &&
      (err = plan_dev_allow(d, dev, (int)smem)) != cudaSuccess)
    return err;
  const int max_blocks = d.max_blocks.load(std::memory_order_relaxed);
  const int64_t NK = (int64_t)s.R * s.S * s.K;
  const int64_t NKt = ranked ? (int64_t)s.S * s.K : NK;  // pairs the tiles cover
  int64_t want = (NKt + kPlanMinPairsPerBlock - 1) / kPlanMinPairsPerBlock;
  // One block for a single tile; otherwise a coordinator plus nt tiles.  The
  // capped plan always has a coordinator (it builds the tables in its free
  // shared memory), and keeps the last kPlanCappedTabRows tile-matrix rows'
  // worth of workspace for the tables it publishes.
  const bool capped = full && kind == kPlanCapped;
  int64_t cap = std::min(max_blocks, kPlanMaxBlocks) - 1;
  if (ranked) cap = std::min<int64_t>(cap, kPlanTotalsRow);
  if (capped) {
    cap = std::min<int64_t>(cap, kPlanMaxBlocks - kPlanCappedTabRows);
    if (cap < 1) return cudaErrorInvalidConfiguration;
    if (capped_tab_words(s.E, s.R) > (int64_t)s.E * kPlanCappedTabRows ||
        capped_smem_ints(s.E, s.R) > (int64_t)kWarps * (s.E + kPlanIdsPerWarp))
      return cudaErrorInvalidValue;
  }
  const int nt = (int)std::max<int64_t>(1, std::min<int64_t>(want, cap));
  const int nb = (nt > 1 || capped) ? nt + 1 : 1;
  const int64_t ppb = (NKt + nt - 1) / nt;
  PlanParams p{};
  p.idx = idx;
  p.R = s.R; p.S = s.S; p.E = s.E; p.K = s.K;
  p.NK = NK;
  p.SK = (int64_t)s.S * s.K;
  p.nb = nb;
  p.nt = nt;
  p.ppb = ppb;
  p.NKt = NKt;
  p.pair0 = ranked ? (int64_t)x.rank * s.S * s.K : 0;
  p.rank_counts = x.rank_counts;
  p.rank = x.rank;
  p.full = full;
  p.kind = kind;
  p.rank_seg_idx = pl.rank_seg_idx;
  p.counts = pl.counts; p.expert_offset = pl.expert_offset; p.slot = pl.slot;
  p.src_pair = pl.src_pair; p.seg = reinterpret_cast<int4 *>(pl.seg);
  p.rank_seg_ptr = pl.rank_seg_ptr; p.expert_seg_ptr = pl.expert_seg_ptr;
  p.replica_seg = pl.replica_seg; p.num_seg = pl.num_seg; p.num_replicas = pl.num_replicas;
  p.max_count = pl.max_count; p.status = pl.status; p.maxvio = pl.maxvio;
  p.bar = reinterpret_cast<uint32_t *>(ws);
  p.tile = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + kPlanWsHeader);
  p.wait_ns = wait_ns;
  p.B = x.B;
  p.max_rank_replicas = x.max_rank_replicas;
  p.tab = p.tile + (int64_t)s.E * (kPlanMaxBlocks - kPlanCappedTabRows);
  p.totals = ranked ? p.tile + (int64_t)s.E * kPlanTotalsRow : pl.counts;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nb);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, plan_kernel, p);
}

}  // namespace mep
