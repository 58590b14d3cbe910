/*
 * CPU oracle for MoonEP's balanced expert-parallel token plan and its data
 * movement.  TEST INFRASTRUCTURE ONLY: the product path never links, loads or
 * calls this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header, table or helper with
 * the CUDA library, and includes nothing from it.
 *
 * Plain, single-threaded C99 (built with -O2 -ffp-contract=off, no SIMD
 * intrinsics, no threads).  Floating-point results are accumulated in binary64
 * and rounded once at the end; integer results are the plain definitions.
 *
 * Sources, by page title and section:
 *   [P1-why]  "Moonshot AI Open-Sources MoonEP, the Library Used to Train the
 *             MoE Model Kimi K3", section "Why expert parallelism is needed":
 *             a router assigns each token to K experts; the imbalance metric
 *             maxvio = max_e(T_e / T-bar) - 1 is 0 for an even load.
 *   [P2-prob] "Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 *             Parallelism Library for MoE Training", section "The problem
 *             MoonEP targets": T_e is the number of tokens routed to expert e,
 *             T-bar the count expected under perfect balance.
 *   [P1-how]  first title, section "How MoonEP works": a rank's share is
 *             pinned at S x K token slots; a few duplicate experts are placed
 *             per step from that step's routing; in the backward pass their
 *             gradients are summed into the home copy.
 *   [P1-eng]  first title, section "Why this matters to engineers": fixed
 *             buffer shapes, no staging copy, each row lands directly in its
 *             expert-ordered slot; section "Key facts": B = E/R for
 *             training.
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): T-bar = R*S*K/E; the schedule is the stable sort of all (token, k)
 * pairs by (expert, global token g = r*S + s, k) cut into R contiguous chunks
 * of S*K slots; home(e) = e / (E/R); a (rank, expert) segment whose rank is
 * not home(e) is a replica; combine is the K-term weighted sum back to token
 * order; the replica reduction sums an expert's segment rows in ascending
 * segment order; the replica weight prefetch copies the home expert's weight
 * row to each replica, in replica-list order.  The backward of dispatch and combine (the training step's
 * return path, [P1-how]: a backward pass exists) is the adjoint of the
 * forward maps: combine's gradient flows to each slot weighted by its router
 * weight, and to each router weight as a dot product with the slot's expert
 * output; dispatch's gradient is the sum of the K slot gradients of a token.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define ORA_OK 0
#define ORA_ERR_ARG 1
#define ORA_ERR_DATA 2

/* ---- bf16 <-> binary32 / binary64, from the IEEE 754 layouts ----------- */

/* A bf16 value is the upper half of the binary32 with the same sign,
 * exponent and leading seven fraction bits. */
float ora_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary64 value to the nearest bf16, ties to even significand.
 * bf16: 1 sign bit, 8 exponent bits (bias 127), 7 stored fraction bits.
 * Normal binade [2^q, 2^(q+1)) has spacing 2^(q-7); below 2^-126 the spacing
 * stays 2^-133 (subnormals).  Overflow past the largest finite value plus
 * half a spacing gives infinity. */
uint16_t ora_f64_to_bf16(double d)
{
    uint16_t sign = signbit(d) ? 0x8000u : 0u;
    if (isnan(d))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(d);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int ex;
    (void)frexp(a, &ex);              /* a in [2^(ex-1), 2^ex) */
    int q = ex - 1;                   /* binade exponent */
    if (q < -126)
        q = -126;                     /* subnormal spacing */
    double spacing = ldexp(1.0, q - 7);
    double t = a / spacing;           /* exact: division by a power of two */
    double n = floor(t);
    double rem = t - n;               /* exact */
    if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0))
        n += 1.0;
    double v = n * spacing;           /* exact, representable in bf16 */
    /* largest finite bf16 = (2^8 - 1) * 2^120 */
    if (v > ldexp(255.0, 120))
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)v;               /* exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/* ---- shape rules -------------------------------------------------------- */

static int ora_check_shape(int R, int S, int E, int K)
{
    if (R < 1 || S < 1 || E < 1 || K < 1 || K > E)
        return ORA_ERR_ARG;
    if (E % R != 0)                   /* home(e) = e / (E/R) needs E/R whole */
        return ORA_ERR_ARG;
    if ((int64_t)R * S * K > INT32_MAX)
        return ORA_ERR_ARG;
    return ORA_OK;
}

/* ---- T_e and maxvio  [P1-why], [P2-prob] -------------------------------- */

/* counts[e] = T_e = number of (token, k) pairs routed to expert e. */
int ora_counts(int R, int S, int E, int K, const int32_t *idx, int32_t *counts)
{
    int st = ora_check_shape(R, S, E, K);
    if (st)
        return st;
    int64_t NK = (int64_t)R * S * K;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t p = 0; p < NK; ++p) {
        int32_t e = idx[p];
        if (e < 0 || e >= E)
            return ORA_ERR_DATA;
        counts[e] += 1;
    }
    return ORA_OK;
}

/* maxvio = max_e T_e / T-bar - 1 with T-bar = R*S*K/E, written as one
 * binary64 quotient of two exact integers: (max T_e * E) / (R*S*K) - 1. */
double ora_maxvio_from_counts(int R, int S, int E, int K, const int32_t *counts,
                              int32_t *max_count)
{
    int32_t m = 0;
    for (int e = 0; e < E; ++e)
        if (counts[e] > m)
            m = counts[e];
    if (max_count)
        *max_count = m;
    int64_t NK = (int64_t)R * S * K;
    return (double)((int64_t)m * E) / (double)NK - 1.0;
}

/* ---- the plan  [P1-how], [P1-eng] --------------------------------------- *
 * Output arrays (caller-allocated):
 *   counts[E], expert_offset[E+1], slot[N*K], src_pair[N*K],
 *   seg[4*(E+R-1)] as {expert, rank, start, count},
 *   rank_seg_ptr[R+1], expert_seg_ptr[E+1], replica_seg[E+R-1],
 *   num_seg, num_replicas, max_count (scalars), maxvio.
 */
int ora_plan(int R, int S, int E, int K, const int32_t *idx,
             int32_t *counts, int32_t *expert_offset, int32_t *slot,
             int32_t *src_pair, int32_t *seg, int32_t *num_seg,
             int32_t *num_replicas, int32_t *rank_seg_ptr,
             int32_t *expert_seg_ptr, int32_t *replica_seg,
             int32_t *max_count, double *maxvio)
{
    int st = ora_counts(R, S, E, K, idx, counts);
    if (st)
        return st;
    int64_t N = (int64_t)R * S;
    int64_t SK = (int64_t)S * K;
    int64_t NK = N * K;
    int B = E / R;                            /* home experts per rank */

    *maxvio = ora_maxvio_from_counts(R, S, E, K, counts, max_count);

    /* Expert e's slots start after all pairs of experts e' < e. */
    expert_offset[0] = 0;
    for (int e = 0; e < E; ++e)
        expert_offset[e + 1] = expert_offset[e] + counts[e];

    /* Stable counting sort: visit pairs in (g, k) order; each takes the next
     * free slot of its expert.  This is the sort by (expert, g, k). */
    for (int e = 0; e < E; ++e)
        counts[e] = 0;                        /* reused as per-expert cursor */
    for (int64_t g = 0; g < N; ++g) {
        for (int k = 0; k < K; ++k) {
            int64_t pair = g * K + k;
            int32_t e = idx[pair];
            int32_t p = expert_offset[e] + counts[e];
            counts[e] += 1;
            slot[pair] = p;
            src_pair[p] = (int32_t)pair;
        }
    }
    /* counts[] is the histogram again after the walk. */

    /* Cut the slot range into R chunks of S*K; a segment is a maximal run of
     * slots with the same (rank, expert). */
    int32_t ns = 0;
    int32_t prev_r = -1, prev_e = -1;
    for (int64_t p = 0; p < NK; ++p) {
        int32_t e = idx[src_pair[p]];
        int32_t r = (int32_t)(p / SK);
        if (r != prev_r || e != prev_e) {
            seg[4 * ns + 0] = e;
            seg[4 * ns + 1] = r;
            seg[4 * ns + 2] = (int32_t)(p - (int64_t)r * SK);
            seg[4 * ns + 3] = 0;
            ns += 1;
            prev_r = r;
            prev_e = e;
        }
        seg[4 * (ns - 1) + 3] += 1;
    }
    *num_seg = ns;

    /* A segment hosted away from its expert's home rank is a replica. */
    int32_t nr = 0;
    for (int32_t s = 0; s < ns; ++s) {
        int32_t e = seg[4 * s + 0], r = seg[4 * s + 1];
        if (r != e / B)
            replica_seg[nr++] = s;
    }
    *num_replicas = nr;

    /* CSR pointers: first segment on rank >= r, first segment of expert >= e. */
    int32_t s = 0;
    for (int r = 0; r <= R; ++r) {
        while (s < ns && seg[4 * s + 1] < r)
            ++s;
        rank_seg_ptr[r] = s;
    }
    s = 0;
    for (int e = 0; e <= E; ++e) {
        while (s < ns && seg[4 * s + 0] < e)
            ++s;
        expert_seg_ptr[e] = s;
    }
    return ORA_OK;
}

/* ---- zero-copy dispatch  [P1-eng] --------------------------------------- *
 * buf[p, :] = x[src_pair[p] / K, :] for the nslots slots listed. */
void ora_dispatch(int64_t nslots, int K, int64_t H, const int32_t *src_pair,
                  const uint16_t *x, uint16_t *buf)
{
    for (int64_t p = 0; p < nslots; ++p) {
        int64_t g = src_pair[p] / K;
        memcpy(buf + p * H, x + g * H, (size_t)H * sizeof(uint16_t));
    }
}

/* ---- weighted combine back to token order -------------------------------- *
 * out[g, h] = sum_k w[g,k] * y[slot[g,k], h], summed in binary64 and rounded
 * once to bf16.  exact[] (may be NULL) receives the binary64 sum and absum[]
 * (may be NULL) the sum of |w * y| terms, for error bounds. */
void ora_combine(int64_t ntok, int K, int64_t H, const int32_t *slot,
                 const float *w, const uint16_t *y, uint16_t *out,
                 double *exact, double *absum)
{
    for (int64_t g = 0; g < ntok; ++g) {
        for (int64_t h = 0; h < H; ++h) {
            double acc = 0.0, mag = 0.0;
            for (int k = 0; k < K; ++k) {
                int64_t p = slot[g * K + k];
                double term = (double)w[g * K + k] * (double)ora_bf16_to_f32(y[p * H + h]);
                acc += term;
                mag += fabs(term);
            }
            out[g * H + h] = ora_f64_to_bf16(acc);
            if (exact)
                exact[g * H + h] = acc;
            if (absum)
                absum[g * H + h] = mag;
        }
    }
}

/* ---- replica weight-gradient reduction  [P1-how] ------------------------ *
 * home[e, i] = sum over expert e's segments s (ascending) of G[s, i], zero
 * for an expert with no segment.  G has one row of P floats per segment. */
void ora_reduce(int E, const int32_t *expert_seg_ptr, int64_t P,
                const float *G, double *home, double *absum)
{
    for (int e = 0; e < E; ++e) {
        for (int64_t i = 0; i < P; ++i) {
            double acc = 0.0, mag = 0.0;
            for (int32_t s = expert_seg_ptr[e]; s < expert_seg_ptr[e + 1]; ++s) {
                double v = (double)G[(int64_t)s * P + i];
                acc += v;
                mag += fabs(v);
            }
            home[(int64_t)e * P + i] = acc;
            if (absum)
                absum[(int64_t)e * P + i] = mag;
        }
    }
}

/* ---- backward of combine (adjoint of ora_combine) ----------------------- *
 * For out[g] = sum_k w[g,k] * y[slot[g,k]]:
 *   grad_y[slot[g,k], h] = bf16( w[g,k] * grad_out[g, h] )     (one rounding)
 *   grad_w[g, k]         = sum_h grad_out[g, h] * y[slot[g,k], h]  (binary64)
 * grad_y has one row per slot; every slot belongs to exactly one (g, k).
 * gy_exact / gw_absum (may be NULL) receive the unrounded product and the
 * sum of |terms| of each dot product, for error bounds. */
void ora_combine_backward(int64_t ntok, int K, int64_t H, const int32_t *slot,
                          const float *w, const uint16_t *grad_out,
                          const uint16_t *y, uint16_t *grad_y, double *gy_exact,
                          double *grad_w, double *gw_absum)
{
    for (int64_t g = 0; g < ntok; ++g) {
        for (int k = 0; k < K; ++k) {
            int64_t p = slot[g * K + k];
            double wk = (double)w[g * K + k];
            double dot = 0.0, mag = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                double go = (double)ora_bf16_to_f32(grad_out[g * H + h]);
                double prod = wk * go;                 /* exact in binary64 */
                grad_y[p * H + h] = ora_f64_to_bf16(prod);
                if (gy_exact)
                    gy_exact[p * H + h] = prod;
                double term = go * (double)ora_bf16_to_f32(y[p * H + h]);  /* exact */
                dot += term;
                mag += fabs(term);
            }
            grad_w[g * K + k] = dot;
            if (gw_absum)
                gw_absum[g * K + k] = mag;
        }
    }
}

/* ---- backward of dispatch (adjoint of ora_dispatch) --------------------- *
 * For buf[slot[g,k]] = x[g]:  grad_x[g, h] = bf16( sum_k grad_buf[slot[g,k], h] ),
 * summed in binary64 and rounded once.  exact / absum as in ora_combine. */
void ora_dispatch_backward(int64_t ntok, int K, int64_t H, const int32_t *slot,
                           const uint16_t *grad_buf, uint16_t *grad_x,
                           double *exact, double *absum)
{
    for (int64_t g = 0; g < ntok; ++g) {
        for (int64_t h = 0; h < H; ++h) {
            double acc = 0.0, mag = 0.0;
            for (int k = 0; k < K; ++k) {
                double v = (double)ora_bf16_to_f32(grad_buf[(int64_t)slot[g * K + k] * H + h]);
                acc += v;
                mag += fabs(v);
            }
            grad_x[g * H + h] = ora_f64_to_bf16(acc);
            if (exact)
                exact[g * H + h] = acc;
            if (absum)
                absum[g * H + h] = mag;
        }
    }
}

/* ---- replica weight prefetch  [P1-how] ---------------------------------- *
 * The duplicates are given their expert's weights before the expert compute:
 * w_rep[j, :] = w_home[expert of segment replica_seg[j], :] for every replica
 * j < num_replicas.  Rows are opaque byte strings of row_bytes (any weight
 * type).  seg is the plan's {expert, rank, start, count} table. */
void ora_prefetch_replicas(int32_t num_replicas, const int32_t *replica_seg,
                           const int32_t *seg, int64_t row_bytes,
                           const uint8_t *w_home, uint8_t *w_rep)
{
    for (int32_t j = 0; j < num_replicas; ++j) {
        int32_t e = seg[4 * replica_seg[j] + 0];
        memcpy(w_rep + (int64_t)j * row_bytes, w_home + (int64_t)e * row_bytes,
               (size_t)row_bytes);
    }
}

/* ---- home-first plan (a low-replica schedule; [P1-how] "a small number of
 * duplicate experts") ------------------------------------------------------ *
 * Every rank still receives exactly S*K slots.  Reading taken for the pages'
 * "small number of redundant experts":
 *   1. each rank fills its S*K slots with its home experts first, in
 *      ascending expert order: expert e keeps h_e = min(T_e, room left);
 *   2. the overflow T_e - h_e of every expert, in ascending expert order,
 *      is cut contiguously over the spare room of the ranks, in ascending
 *      rank order; each (expert, rank) piece of overflow is a replica;
 *   3. rank r's slots hold its home pieces (expert order) and then its
 *      replica pieces (expert order); inside a piece, pairs keep (g, k) order;
 *      an expert's first h_e pairs are the home ones.
 * Segments are listed by (expert, rank); rank_seg_idx lists each rank's
 * segments in slot order (rank r: entries rank_seg_ptr[r] .. rank_seg_ptr[r+1]).
 * At most E + R - 1 segments: in every full rank at most one expert keeps
 * only part of its pairs home, so with Z experts keeping none, X overflowing
 * experts and Y ranks with room there are at most E - Z home pieces and
 * X + Y - 1 <= (R - Y) + Z + Y - 1 replica pieces.  expert_offset is the exclusive prefix of counts
 * (the pair's index in the expert-sorted order), not a slot position. */
int ora_plan_home_first(int R, int S, int E, int K, const int32_t *idx,
                        int32_t *counts, int32_t *expert_offset, int32_t *slot,
                        int32_t *src_pair, int32_t *seg, int32_t *num_seg,
                        int32_t *num_replicas, int32_t *rank_seg_ptr,
                        int32_t *rank_seg_idx, int32_t *expert_seg_ptr,
                        int32_t *replica_seg, int32_t *max_count, double *maxvio,
                        int32_t *scratch /* 6*E + 3*R + 2 ints */)
{
    int st = ora_counts(R, S, E, K, idx, counts);
    if (st)
        return st;
    int64_t N = (int64_t)R * S;
    int64_t C = (int64_t)S * K;
    int64_t NK = N * K;
    int B = E / R;
    *maxvio = ora_maxvio_from_counts(R, S, E, K, counts, max_count);
    expert_offset[0] = 0;
    for (int e = 0; e < E; ++e)
        expert_offset[e + 1] = expert_offset[e] + counts[e];

    int32_t *h = scratch, *pre = h + E, *over = pre + E, *O = over + E;   /* O: E+1 */
    int32_t *used = O + E + 1;                  /* per-expert pairs placed so far: E */
    int32_t *F = used + E, *D = F + R;          /* D: R+1 */
    int32_t *deficit = D + R + 1;               /* R */

    /* 1. home fill, rank by rank, home experts in ascending order */
    for (int r = 0; r < R; ++r) {
        int64_t fill = 0;
        for (int e = r * B; e < (r + 1) * B; ++e) {
            int64_t take = counts[e] < C - fill ? counts[e] : C - fill;
            pre[e] = (int32_t)fill;
            h[e] = (int32_t)take;
            fill += take;
        }
        F[r] = (int32_t)fill;
        deficit[r] = (int32_t)(C - fill);
    }
    /* 2. overflow stream (experts ascending) against spare room (ranks ascending) */
    O[0] = 0;
    for (int e = 0; e < E; ++e) {
        over[e] = counts[e] - h[e];
        O[e + 1] = O[e] + over[e];
    }
    D[0] = 0;
    for (int r = 0; r < R; ++r)
        D[r + 1] = D[r] + deficit[r];

    /* 3. place every pair, walking pairs in (g, k) order */
    for (int e = 0; e < E; ++e)
        used[e] = 0;
    for (int64_t pair = 0; pair < NK; ++pair) {      /* pair = g*K + k: (g, k) order */
        int32_t e = idx[pair];
        int32_t i = used[e]++;
        int64_t p;
        if (i < h[e]) {
            p = (int64_t)(e / B) * C + pre[e] + i;
        } else {
            int64_t q = (int64_t)O[e] + (i - h[e]);
            int r = 0;
            while (!(D[r] <= q && q < D[r + 1]))
                ++r;
            p = (int64_t)r * C + F[r] + (q - D[r]);
        }
        slot[pair] = (int32_t)p;
        src_pair[p] = (int32_t)pair;
    }

    /* 4. segments: maximal runs of one expert inside one rank, in slot order,
     *    then listed by (expert, rank) */
    int32_t nrun = 0;
    int32_t prev_r = -1, prev_e = -1;
    for (int64_t p = 0; p < NK; ++p) {
        int32_t e = idx[src_pair[p]];
        int32_t r = (int32_t)(p / C);
        if (e != prev_e || r != prev_r) {
            /* temporarily store runs in slot order in seg */
            seg[4 * nrun + 0] = e;
            seg[4 * nrun + 1] = r;
            seg[4 * nrun + 2] = (int32_t)(p - (int64_t)r * C);
            seg[4 * nrun + 3] = 0;
            ++nrun;
            prev_r = r;
            prev_e = e;
        }
        seg[4 * (nrun - 1) + 3] += 1;
    }
    *num_seg = nrun;
    /* stable selection sort of the runs by (expert, rank); rank_seg_idx keeps
     * each run's new index in slot order */
    for (int32_t a = 0; a < nrun; ++a)
        rank_seg_idx[a] = a;                     /* run a (slot order) -> index */
    for (int32_t a = 0; a < nrun; ++a) {
        int32_t best = a;
        for (int32_t b = a + 1; b < nrun; ++b) {
            int32_t eb = seg[4 * b], rb = seg[4 * b + 1];
            int32_t ek = seg[4 * best], rk = seg[4 * best + 1];
            if (eb < ek || (eb == ek && rb < rk))
                best = b;
        }
        if (best != a) {
            for (int c = 0; c < 4; ++c) {
                int32_t tmp = seg[4 * a + c];
                seg[4 * a + c] = seg[4 * best + c];
                seg[4 * best + c] = tmp;
            }
            int32_t tmp = rank_seg_idx[a];
            rank_seg_idx[a] = rank_seg_idx[best];
            rank_seg_idx[best] = tmp;
        }
    }
    /* rank_seg_idx[a] now holds the slot-order run id of table entry a;
     * invert it so that slot-order run j maps to its table index */
    for (int32_t a = 0; a < nrun; ++a)
        replica_seg[rank_seg_idx[a]] = a;        /* replica_seg used as scratch */
    for (int32_t j = 0; j < nrun; ++j)
        rank_seg_idx[j] = replica_seg[j];
    int32_t s = 0;
    for (int r = 0; r <= R; ++r) {               /* runs are rank-major in slot order */
        while (s < nrun && seg[4 * rank_seg_idx[s] + 1] < r)
            ++s;
        rank_seg_ptr[r] = s;
    }
    s = 0;
    for (int e = 0; e <= E; ++e) {
        while (s < nrun && seg[4 * s] < e)
            ++s;
        expert_seg_ptr[e] = s;
    }
    int32_t nr = 0;
    for (int32_t a = 0; a < nrun; ++a)
        if (seg[4 * a + 1] != seg[4 * a] / B)
            replica_seg[nr++] = a;
    *num_replicas = nr;
    return ORA_OK;
}

/* ---- capped plan: at most B replica experts per rank ([P1-how] "a small
 * number of duplicate experts"; [P1-eng] "Key facts": B = E/R for training,
 * B = 3-4 recommended for inference) ----------------------------------------- *
 * Reading taken for B: the number of redundant (replica) experts a rank may
 * host in one step -- the slots of its prefetch buffer for duplicates' weights
 * -- in addition to its home experts.  (Read instead as the number of distinct
 * experts a rank may host, the training value E/R would forbid every
 * duplicate whenever every expert has tokens, and exact S*K balance would be
 * unreachable: R = 2, E = 2, S*K = 10, T = (15, 5) needs a rank to take pairs
 * of two experts.)  Every rank still receives exactly S*K slots.
 *   1. Home fill: each rank takes its home experts in order of increasing
 *      count (ties: lower id first); expert e keeps h_e = min(T_e, room left)
 *      pairs home.  F_r = pairs kept on rank r, D_r = S*K - F_r its spare
 *      room, O_e = T_e - h_e the overflow of e.
 *   2. Items: experts with O_e > 0 by (O_e descending, e ascending); rooms:
 *      ranks with D_r > 0 by (D_r descending, r ascending); Dmax = the first
 *      room's D.
 *   3. Fillers: the items with O_e < Dmax.  Filler f (f = 0, 1, ... in item
 *      order) is offered to room f mod Y (Y rooms) in round f / Y; it is
 *      placed whole, as one replica piece, if the round is below B - 2 and the
 *      room's space left by earlier rounds holds it.
 *   4. Stream: the items not placed as fillers, in item order, are cut
 *      contiguously over the rooms' remaining space, in room order; each
 *      (item, room) intersection is a replica piece.
 *   5. Layout: rank r holds its home pieces in ascending expert order (slots
 *      0 .. F_r - 1), then its replica pieces: fillers by round, then stream
 *      pieces in stream order.  Expert e's pairs, in (g, k) order: the first
 *      h_e go home, the others fill its replica pieces in the order the
 *      pieces were made (its one filler piece, or its stream pieces in room
 *      order).
 * When every filler is placed and B >= 3, no rank holds more than B replica
 * pieces: a room takes at most B - 2 fillers, and the stream items are all at
 * least Dmax, so a room's remaining space meets at most two of them.
 * Segments are listed by (expert, rank); rank_seg_idx lists each rank's
 * segments in slot order.  *max_rank_replicas receives the largest number of
 * replica segments on one rank, *unplaced the number of fillers not placed.
 * scratch: 12*E + 10*R + 1 ints. */
int ora_plan_capped(int R, int S, int E, int K, int B, const int32_t *idx,
                    int32_t *counts, int32_t *expert_offset, int32_t *slot,
                    int32_t *src_pair, int32_t *seg, int32_t *num_seg,
                    int32_t *num_replicas, int32_t *rank_seg_ptr,
                    int32_t *rank_seg_idx, int32_t *expert_seg_ptr,
                    int32_t *replica_seg, int32_t *max_count, double *maxvio,
                    int32_t *max_rank_replicas, int32_t *unplaced,
                    int32_t *scratch)
{
    if (B < 1)
        return ORA_ERR_ARG;
    int st = ora_counts(R, S, E, K, idx, counts);
    if (st)
        return st;
    int64_t N = (int64_t)R * S;
    int64_t C = (int64_t)S * K;
    int64_t NK = N * K;
    int Bh = E / R;                               /* home experts per rank */
    *maxvio = ora_maxvio_from_counts(R, S, E, K, counts, max_count);
    expert_offset[0] = 0;
    for (int e = 0; e < E; ++e)
        expert_offset[e + 1] = expert_offset[e] + counts[e];

    int32_t *h = scratch;                         /* E: pairs kept home */
    int32_t *O = h + E;                           /* E: overflow */
    int32_t *item = O + E;                        /* E: items in item order */
    int32_t *placed_room = item + E;              /* E: room index of a placed filler, else -1 */
    int32_t *npiece = placed_room + E;            /* E: replica pieces of expert e */
    int32_t *used = npiece + E;                   /* E: pairs of e placed so far */
    int32_t *pstart = used + E;                   /* E+1: first piece of e (by expert) */
    int32_t *F = pstart + E + 1;                  /* R */
    int32_t *D = F + R;                           /* R */
    int32_t *room = D + R;                        /* R: rooms in room order */
    int32_t *left = room + R;                     /* R: space left in room j */
    int32_t *nrep = left + R;                     /* R: replica pieces on rank r so far */
    int32_t *rfill = nrep + R;                    /* R: replica slots used on rank r so far */
    int32_t *hpre = rfill + R;                    /* E: home start of e on its rank */
    /* pieces, at most E + R of them: expert, rank, size, first slot */
    int32_t *pe = hpre + E, *pr = pe + E + R, *pn = pr + E + R, *pslot = pn + E + R;
    (void)pslot;

    /* 1. home fill, smallest home experts first: ord[t] is the home expert of
     * rank t / Bh's block with (count, id) rank t % Bh */
    int32_t *ord = O;                             /* borrowed until step 1 ends */
    for (int r = 0; r < R; ++r) {
        for (int e = r * Bh; e < (r + 1) * Bh; ++e) {
            int rank_e = 0;
            for (int e2 = r * Bh; e2 < (r + 1) * Bh; ++e2)
                if (counts[e2] < counts[e] || (counts[e2] == counts[e] && e2 < e))
                    ++rank_e;
            ord[r * Bh + rank_e] = e;
        }
        int64_t fill = 0;
        for (int t = 0; t < Bh; ++t) {
            int e = ord[r * Bh + t];
            int64_t take = counts[e] < C - fill ? counts[e] : C - fill;
            h[e] = (int32_t)take;
            fill += take;
        }
        F[r] = (int32_t)fill;
        D[r] = (int32_t)(C - fill);
    }
    for (int r = 0; r < R; ++r) {                 /* home pieces in ascending expert order */
        int64_t at = 0;
        for (int e = r * Bh; e < (r + 1) * Bh; ++e) {
            hpre[e] = (int32_t)at;
            at += h[e];
        }
    }
    for (int e = 0; e < E; ++e)
        O[e] = counts[e] - h[e];

    /* 2. items and rooms, each by an insertion sort on its key */
    int X = 0, Y = 0;
    for (int e = 0; e < E; ++e) {
        if (O[e] <= 0)
            continue;
        int at = X++;
        while (at > 0 && (O[item[at - 1]] < O[e] ||
                          (O[item[at - 1]] == O[e] && item[at - 1] > e))) {
            item[at] = item[at - 1];
            --at;
        }
        item[at] = e;
    }
    for (int r = 0; r < R; ++r) {
        if (D[r] <= 0)
            continue;
        int at = Y++;
        while (at > 0 && (D[room[at - 1]] < D[r] ||
                          (D[room[at - 1]] == D[r] && room[at - 1] > r))) {
            room[at] = room[at - 1];
            --at;
        }
        room[at] = r;
    }
    for (int j = 0; j < Y; ++j)
        left[j] = D[room[j]];
    for (int e = 0; e < E; ++e) {
        placed_room[e] = -1;
        npiece[e] = 0;
    }
    for (int r = 0; r < R; ++r) {
        nrep[r] = 0;
        rfill[r] = F[r];
    }
    int np = 0;                                   /* pieces made so far */
    *unplaced = 0;

    /* 3. fillers, round by round */
    if (Y > 0) {
        int32_t dmax = D[room[0]];
        int f = 0;
        for (int i = 0; i < X; ++i) {
            int e = item[i];
            if (O[e] >= dmax)
                continue;
            int j = f % Y, round = f / Y;
            if (round < B - 2 && left[j] >= O[e]) {
                placed_room[e] = j;
                left[j] -= O[e];
                pstart[e] = np;
                npiece[e] = 1;
                pe[np] = e;
                pr[np] = room[j];
                pn[np] = O[e];
                ++np;
            } else {
                *unplaced += 1;
            }
            ++f;
        }
    }
    /* lay the fillers out: room by room, by round (= the order they were
     * offered to that room, which is item order) */
    for (int j = 0; j < Y; ++j) {
        for (int q = 0; q < np; ++q) {
            if (pr[q] != room[j])
                continue;
            pslot[q] = (int32_t)((int64_t)room[j] * C + rfill[room[j]]);
            rfill[room[j]] += pn[q];
            nrep[room[j]] += 1;
        }
    }
    /* 4. the stream: unplaced items against the rooms' remaining space */
    {
        int j = 0;
        int32_t jleft = Y > 0 ? left[0] : 0;
        for (int i = 0; i < X; ++i) {
            int e = item[i];
            if (placed_room[e] >= 0)
                continue;
            int32_t need = O[e];
            while (need > 0) {
                while (jleft == 0 && j + 1 < Y) { /* next room with space */
                    ++j;
                    jleft = left[j];
                }
                if (jleft == 0)
                    return ORA_ERR_DATA;          /* cannot happen: overflow = room */
                int32_t n = need < jleft ? need : jleft;
                int r = room[j];
                if (npiece[e] == 0)
                    pstart[e] = np;
                npiece[e] += 1;
                pe[np] = e;
                pr[np] = r;
                pn[np] = n;
                pslot[np] = (int32_t)((int64_t)r * C + rfill[r]);
                rfill[r] += n;
                nrep[r] += 1;
                ++np;
                need -= n;
                jleft -= n;
            }
        }
    }
    int32_t mx = 0;
    for (int r = 0; r < R; ++r)
        if (nrep[r] > mx)
            mx = nrep[r];
    *max_rank_replicas = mx;

    /* 5. place every pair, walking pairs in (g, k) order; expert e's replica
     * pieces are used in the order they were made (piece list order) */
    for (int e = 0; e < E; ++e)
        used[e] = 0;
    for (int64_t pair = 0; pair < NK; ++pair) {
        int32_t e = idx[pair];
        int32_t i = used[e]++;
        int64_t p;
        if (i < h[e]) {
            p = (int64_t)(e / Bh) * C + hpre[e] + i;
        } else {
            int32_t q = i - h[e];
            int t = pstart[e];                    /* e's pieces are consecutive */
            while (q >= pn[t]) {
                q -= pn[t];
                ++t;
            }
            p = (int64_t)pslot[t] + q;
        }
        slot[pair] = (int32_t)p;
        src_pair[p] = (int32_t)pair;
    }

    /* 6. segments by (expert, rank): expert e's home piece and replica
     * pieces, ordered by rank (insertion on the rank) */
    int32_t ns = 0;
    for (int e = 0; e < E; ++e) {
        expert_seg_ptr[e] = ns;
        int32_t first = ns;
        for (int t = -1; t < npiece[e]; ++t) {
            int32_t r, start, n;
            if (t < 0) {                          /* the home piece */
                if (h[e] == 0)
                    continue;
                r = e / Bh;
                start = hpre[e];
                n = h[e];
            } else {
                int q2 = pstart[e] + t;
                r = pr[q2];
                start = (int32_t)(pslot[q2] - (int64_t)r * C);
                n = pn[q2];
            }
            int32_t q = ns++;
            while (q > first && seg[4 * (q - 1) + 1] > r) {
                for (int c = 0; c < 4; ++c)
                    seg[4 * q + c] = seg[4 * (q - 1) + c];
                --q;
            }
            seg[4 * q + 0] = e;
            seg[4 * q + 1] = r;
            seg[4 * q + 2] = start;
            seg[4 * q + 3] = n;
        }
    }
    expert_seg_ptr[E] = ns;
    *num_seg = ns;
    /* each rank's segments in slot order: its segments, by insertion on
     * their start */
    int32_t at = 0;
    for (int r = 0; r < R; ++r) {
        rank_seg_ptr[r] = at;
        int32_t first = at;
        for (int32_t s2 = 0; s2 < ns; ++s2) {
            if (seg[4 * s2 + 1] != r)
                continue;
            int32_t q = at++;
            while (q > first && seg[4 * rank_seg_idx[q - 1] + 2] > seg[4 * s2 + 2]) {
                rank_seg_idx[q] = rank_seg_idx[q - 1];
                --q;
            }
            rank_seg_idx[q] = s2;
        }
    }
    rank_seg_ptr[R] = at;
    int32_t nr = 0;
    for (int32_t a = 0; a < ns; ++a)
        if (seg[4 * a + 1] != seg[4 * a] / Bh)
            replica_seg[nr++] = a;
    *num_replicas = nr;
    return ORA_OK;
}
