/*
 * ep_oracle.c -- plain, single-threaded CPU oracle for expert-parallel
 * dispatch / combine and replica routing expansion.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It shares no
 * code, header, table or helper with the CUDA path: every function below is
 * the plain definition of one step, written as loops in the order the
 * definition states, with no blocking, fusion or reordering.  Build with
 * plain gcc (no -ffast-math, -ffp-contract=off) so the float64 arithmetic is
 * IEEE round-to-nearest in program order.
 *
 * Sources (web pages; cited by title and section):
 *  [P1] NeMo AutoModel API docs, "nemo_automodel.components.moe.uccl_ep.buffer":
 *       Buffer.get_dispatch_layout, Buffer.dispatch, Buffer.low_latency_dispatch,
 *       Buffer.low_latency_combine, Buffer.get_next_low_latency_combine_buffer.
 *  [P3] GitDiagram, "dots-infra/ultraep architecture": GPU operations
 *       (load computation, placement planning, routing expansion).
 *  [P4] ai-dynamo/nixl PR "nixl_ep: Optimize low-latency NVLink path":
 *       active rank mask in combine; 32-bit topk index width.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - a pair (r,t,j) is live iff 0 <= e < E, active[r] and active[e / E_local];
 *    e == -1 means "no selection" ([P1] get_dispatch_layout), any other
 *    out-of-range id is counted as an error (status bit 1) and dropped;
 *  - rows inside an expert's receive slab are compact: the row of a live pair
 *    is its position in that expert's list of live pairs enumerated in
 *    (src_rank, token, slot) order, so valid rows are [0, recv_count[e]);
 *  - the slab holds num_ranks * num_tokens rows per expert ([P1]
 *    low_latency_dispatch shape); a pair whose row is past that capacity is
 *    counted as an overflow (status bit 2) and neither sent nor reduced;
 *  - combine is the weighted reduce of [P1] low_latency_combine, re-checking
 *    the active mask given at combine time ([P4]); rows of an inactive source
 *    rank come out as zeros; weights are not renormalised;
 *  - replica planning starts every logical expert at one replica and adds the
 *    extra replicas one at a time to the expert with the largest
 *    load/replicas (exact integer comparison, ties to the lowest id); replica
 *    i of logical expert e is physical expert phys_base[e] + i; a pair goes to
 *    replica (r*T + t) mod n_rep[e].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BAD_EXPERT 1
#define ORACLE_OVERFLOW   2


/* bfloat16 bit pattern -> double.  A bf16 value is the upper half of the
 * float32 with the same sign, exponent and leading 7 mantissa bits. */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int pair_is_live(int e, int r, int E, int E_local, const uint8_t *active) {
    if (e < 0 || e >= E) return 0;
    if (!active[r]) return 0;
    if (!active[e / E_local]) return 0;
    return 1;
}

/*
 * Layout ([P1] Buffer.get_dispatch_layout) plus the handle that dispatch and
 * combine share ([P1] Buffer.dispatch "handle", Buffer.low_latency_combine
 * "handle").  Enumerates (r, t, j) in lexicographic order and appends every
 * live pair to its expert's list.
 *
 * outputs:
 *   num_tokens_per_expert [R,E]  live pairs of source rank r routed to e
 *   num_tokens_per_rank   [R,R]  tokens of r with >= 1 live pair on rank d
 *   is_token_in_rank      [R,T,R]
 *   recv_count            [E]    length of list[e]
 *   expert_rank_offset    [E,R]  first index in list[e] whose source rank >= r
 *   pair_row              [R,T,k] position in list[e], -1 if not live
 *   src_list              [sum(recv_count), 2] (r, t) of list entries,
 *                                 expert-major; may be NULL
 *   list_base             [E+1]  start of list[e] in src_list
 * returns the status bits (1: bad expert id, 2: row past capacity).
 */
int oracle_layout(int R, int T, int k, int E, const int32_t *topk_idx, const uint8_t *active,
                  int32_t *num_tokens_per_expert, int32_t *num_tokens_per_rank,
                  uint8_t *is_token_in_rank, int32_t *recv_count, int32_t *expert_rank_offset,
                  int32_t *pair_row, int32_t *src_list, int64_t *list_base) {
    int status = 0;
    const int E_local = E / R;
    const int64_t capacity = (int64_t)R * T;

    memset(num_tokens_per_expert, 0, sizeof(int32_t) * (size_t)R * E);
    memset(num_tokens_per_rank, 0, sizeof(int32_t) * (size_t)R * R);
    memset(is_token_in_rank, 0, (size_t)R * T * R);
    memset(recv_count, 0, sizeof(int32_t) * (size_t)E);

    /* append every live pair to list[e]: its row is the list length so far */
    for (int r = 0; r < R; r++) {
        for (int t = 0; t < T; t++) {
            for (int j = 0; j < k; j++) {
                int64_t p = ((int64_t)r * T + t) * k + j;
                int e = topk_idx[p];
                if (e < -1 || e >= E) status |= ORACLE_BAD_EXPERT;
                if (!pair_is_live(e, r, E, E_local, active)) {
                    pair_row[p] = -1;
                    continue;
                }
                pair_row[p] = recv_count[e];
                recv_count[e] += 1;
                num_tokens_per_expert[(int64_t)r * E + e] += 1;
                is_token_in_rank[((int64_t)r * T + t) * R + e / E_local] = 1;
            }
        }
    }
    for (int e = 0; e < E; e++)
        if (recv_count[e] > capacity) status |= ORACLE_OVERFLOW;

    /* a token counts once per destination rank */
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int d = 0; d < R; d++)
                num_tokens_per_rank[(int64_t)r * R + d] += is_token_in_rank[((int64_t)r * T + t) * R + d];

    /* materialise the lists: entry pair_row of list[e] is (r, t) */
    list_base[0] = 0;
    for (int e = 0; e < E; e++) list_base[e + 1] = list_base[e] + recv_count[e];
    int32_t *list = src_list;
    int32_t *own = NULL;
    if (list == NULL) {
        own = (int32_t *)malloc(sizeof(int32_t) * 2 * (size_t)(list_base[E] > 0 ? list_base[E] : 1));
        list = own;
    }
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < k; j++) {
                int64_t p = ((int64_t)r * T + t) * k + j;
                if (pair_row[p] < 0) continue;
                int e = topk_idx[p];
                int64_t at = list_base[e] + pair_row[p];
                list[2 * at + 0] = r;
                list[2 * at + 1] = t;
            }

    /* offset of source rank r inside list[e]: first entry with src rank >= r */
    for (int e = 0; e < E; e++) {
        for (int r = 0; r < R; r++) {
            int32_t pos = recv_count[e];
            for (int32_t i = 0; i < recv_count[e]; i++) {
                if (list[2 * (list_base[e] + i)] >= r) { pos = i; break; }
            }
            expert_rank_offset[(int64_t)e * R + r] = pos;
        }
    }
    free(own);
    return status;
}

/*
 * Dispatch ([P1] Buffer.low_latency_dispatch with use_fp8=False): every live
 * pair's token row is copied, bit for bit, into its expert's list position.
 * Only list entries are materialised (packed, expert-major at list_base[e]),
 * never the empty tail of the receive slab.  Rows past the slab capacity are
 * not sent.
 *   x       [R,T,H] bf16 bits
 *   packed  [list_base[E], H] bf16 bits (rows past capacity left untouched)
 */
int oracle_dispatch(int R, int T, int k, int E, int H, const uint16_t *x, const int32_t *topk_idx,
                    const int32_t *pair_row, const int64_t *list_base, uint16_t *packed) {
    int status = 0;
    const int64_t capacity = (int64_t)R * T;
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < k; j++) {
                int64_t p = ((int64_t)r * T + t) * k + j;
                int32_t row = pair_row[p];
                if (row < 0) continue;
                if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }
                int e = topk_idx[p];
                if (e < 0 || e >= E) continue;
                const uint16_t *src = x + ((int64_t)r * T + t) * H;
                uint16_t *dst = packed + (list_base[e] + row) * H;
                for (int h = 0; h < H; h++) dst[h] = src[h];
            }
    return status;
}

/*
 * Combine ([P1] Buffer.low_latency_combine, "reduce with weights"; active
 * mask per [P4]) for a list of tokens.  For token (r, t):
 *   out[h] = sum over slots j whose pair is live under active_now and whose
 *            row is inside the capacity of  w[r,t,j] * y[e][row][h]
 * accumulated in float64.  Rows of an inactive source rank are 0.
 *   y        bf16 bits; row (e, row) lives at y + (y_row_base[e] + row) * H
 *   tokens   [n_tokens, 2] (r, t) pairs, or NULL for every (r, t) in order
 *   out      float64 [n_tokens, H]
 */
int oracle_combine(int R, int T, int k, int E, int H, const uint16_t *y, const int64_t *y_row_base,
                   const int32_t *topk_idx, const float *topk_weights, const int32_t *pair_row,
                   const uint8_t *active_now, const int32_t *tokens, int64_t n_tokens, double *out) {
    int status = 0;
    const int E_local = E / R;
    const int64_t capacity = (int64_t)R * T;
    if (tokens == NULL) n_tokens = (int64_t)R * T;
    for (int64_t i = 0; i < n_tokens; i++) {
        int r = tokens ? tokens[2 * i] : (int)(i / T);
        int t = tokens ? tokens[2 * i + 1] : (int)(i % T);
        double *o = out + i * H;
        for (int h = 0; h < H; h++) o[h] = 0.0;
        if (!active_now[r]) continue;
        for (int j = 0; j < k; j++) {
            int64_t p = ((int64_t)r * T + t) * k + j;
            int32_t row = pair_row[p];
            int e = topk_idx[p];
            if (row < 0) continue;
            if (e < 0 || e >= E) continue;
            if (!active_now[e / E_local]) continue;
            if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }
            double w = (double)topk_weights[p];
            const uint16_t *yr = y + (y_row_base[e] + row) * H;
            for (int h = 0; h < H; h++) o[h] += w * bf16_to_double(yr[h]);
        }
    }
    return status;
}

/*
 * Load computation, placement planning and routing expansion ([P3] GPU
 * operations: load_compute, placement, reroute).
 *   load        [E_log]   (token, slot) pairs routed to each logical expert
 *   n_rep       [E_log]   replicas per logical expert (sum = E_log + n_extra)
 *   phys_base   [E_log+1] exclusive prefix sum of n_rep
 *   topk_phys   [R,T,k]   physical id, -1 where the logical id is -1 or bad
 */
int oracle_reroute(int R, int T, int k, int E_log, int n_extra, const int32_t *topk_logical,
                   int32_t *load, int32_t *n_rep, int32_t *phys_base, int32_t *topk_phys) {
    int status = 0;
    const int64_t n_pairs = (int64_t)R * T * k;

    for (int e = 0; e < E_log; e++) load[e] = 0;
    for (int64_t p = 0; p < n_pairs; p++) {
        int e = topk_logical[p];
        if (e >= 0 && e < E_log) load[e] += 1;
        else if (e != -1) status |= ORACLE_BAD_EXPERT;
    }

    for (int e = 0; e < E_log; e++) n_rep[e] = 1;
    for (int step = 0; step < n_extra; step++) {
        int best = 0;
        for (int e = 1; e < E_log; e++) {
            /* load[e]/n_rep[e] > load[best]/n_rep[best], compared exactly */
            int64_t lhs = (int64_t)load[e] * n_rep[best];
            int64_t rhs = (int64_t)load[best] * n_rep[e];
            if (lhs > rhs) best = e;
        }
        n_rep[best] += 1;
    }

    phys_base[0] = 0;
    for (int e = 0; e < E_log; e++) phys_base[e + 1] = phys_base[e] + n_rep[e];

    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < k; j++) {
                int64_t p = ((int64_t)r * T + t) * k + j;
                int e = topk_logical[p];
                if (e < 0 || e >= E_log) { topk_phys[p] = -1; continue; }
                int64_t global_token = (int64_t)r * T + t;
                topk_phys[p] = phys_base[e] + (int32_t)(global_token % n_rep[e]);
            }
    return status;
}

/*
 * FP8 dispatch ([P1] Buffer.low_latency_dispatch, use_fp8=True): each token row
 * is cast to float8 e4m3 with one scale per 128 channels; round_scale makes the
 * scales powers of two; use_ue8m0 stores them as UE8M0 (biased exponent bytes),
 * four per int32.  The pages name the format but not the arithmetic; the
 * reading used here (also in the design notes):
 *   amax  = max |x| over the group (bf16 values, exact in float32)
 *   scale = 1 if amax == 0, else amax / 448 in float32 (448 = largest e4m3)
 *   with round_scale: scale = 2^e, e = ceil(log2(amax / 448)) clamped to
 *                     [-127, 127] (1 when amax == 0); UE8M0 byte = e + 127
 *   code  = e4m3(x / scale), the division in float32, round to nearest even,
 *           saturating at +-448.
 */

/* float32 -> float8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, 0x7F/0xFF = NaN): round to nearest, ties to even;
 * magnitudes at or beyond 448 (and infinities) saturate to 448; NaN -> NaN. */
uint8_t oracle_e4m3_from_float(float v) {
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    const uint8_t sign = (uint8_t)((bits >> 24) & 0x80u);
    if (v != v) return (uint8_t)(sign | 0x7Fu);
    const double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    if (a == 0.0) return sign;
    /* binade exponent of a (a = m * 2^e, 1 <= m < 2); values below 2^-6 are
     * subnormal and share the quantum 2^-9 of the smallest binade */
    int e;
    frexp(a, &e);
    e -= 1;
    if (e < -6) e = -6;
    const double quantum = ldexp(1.0, e - 3);
    const double val = rint(a / quantum) * quantum; /* rint: nearest, ties to even */
    if (val == 0.0) return sign;
    if (val < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(val / ldexp(1.0, -9)));
    int ve;
    const double m = frexp(val, &ve); /* val = m * 2^ve, 0.5 <= m < 1 */
    const int mant = (int)((m * 2.0 - 1.0) * 8.0);
    return (uint8_t)(sign | (uint8_t)((ve - 1 + 7) << 3) | (uint8_t)mant);
}

/* Scale of one 128-channel group (see above); *ue8m0 gets the byte when
 * pow2 is set. */
static float group_scale(const uint16_t *x, int n, int pow2, uint8_t *ue8m0) {
    float amax = 0.0f;
    for (int i = 0; i < n; i++) {
        uint32_t u = ((uint32_t)x[i]) << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        if (f < 0) f = -f;
        if (f > amax) amax = f;
    }
    if (!pow2) {
        if (ue8m0) *ue8m0 = 127;
        return amax == 0.0f ? 1.0f : amax / 448.0f;
    }
    int e = 0;
    if (amax != 0.0f) {
        const float s = amax / 448.0f;
        /* smallest e with 2^e >= s: s = m * 2^f with 0.5 <= m < 1, so e = f unless m == 0.5 */
        int f;
        const double m = frexp((double)s, &f);
        e = m == 0.5 ? f - 1 : f;
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }
    if (ue8m0) *ue8m0 = (uint8_t)(e + 127);
    return (float)ldexp(1.0, e);
}

/* Quantise one row of H channels: codes[H], scales[H/128] (float32), and the
 * UE8M0 bytes ue8m0[H/128] when pow2 is set (may be NULL). */
void oracle_fp8_quantize_row(const uint16_t *x, int H, int pow2, uint8_t *codes, float *scales,
                             uint8_t *ue8m0) {
    for (int g = 0; g < H / 128; g++) {
        const uint16_t *xg = x + g * 128;
        const float scale = group_scale(xg, 128, pow2, ue8m0 ? ue8m0 + g : NULL);
        scales[g] = scale;
        for (int i = 0; i < 128; i++) {
            uint32_t u = ((uint32_t)xg[i]) << 16;
            float f;
            memcpy(&f, &u, sizeof f);
            const float q = f / scale;
            codes[g * 128 + i] = oracle_e4m3_from_float(q);
        }
    }
}

/* FP8 dispatch of every live pair, packed in list order like oracle_dispatch:
 *   codes  [list_base[E], H]      e4m3 codes
 *   scales [list_base[E], H/128]  float32 scales (row-major here)
 *   ue8m0  [list_base[E], H/128]  UE8M0 bytes (pow2 only; may be NULL) */
int oracle_dispatch_fp8(int R, int T, int k, int E, int H, int pow2, const uint16_t *x,
                        const int32_t *topk_idx, const int32_t *pair_row, const int64_t *list_base,
                        uint8_t *codes, float *scales, uint8_t *ue8m0) {
    int status = 0;
    const int64_t capacity = (int64_t)R * T;
    const int G = H / 128;
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int j = 0; j < k; j++) {
                int64_t p = ((int64_t)r * T + t) * k + j;
                int32_t row = pair_row[p];
                if (row < 0) continue;
                if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }
                int e = topk_idx[p];
                if (e < 0 || e >= E) continue;
                const int64_t at = list_base[e] + row;
                oracle_fp8_quantize_row(x + ((int64_t)r * T + t) * H, H, pow2, codes + at * H, scales + at * G,
                                        ue8m0 ? ue8m0 + at * G : NULL);
            }
    return status;
}

/* e4m3 encoding of an array (element by element). */
void oracle_e4m3_array(const float *v, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_from_float(v[i]);
}

/*
 * Normal (high-throughput) mode ([P1] Buffer.dispatch and Buffer.combine):
 * a token goes ONCE to every rank that one of its live pairs reaches
 * (is_token_in_rank), and combine adds the returned rows WITHOUT weights.
 * Readings (also in the design notes): rank d's received tokens are ordered
 * by (source rank, token); a receive buffer holds `capacity` rows
 * (num_worst_tokens), rows past it are counted as overflow and neither
 * written nor read; recv_topk_idx holds the local expert id (e - d*E_local)
 * of slots whose live expert is on rank d and -1 elsewhere, recv_topk_weights
 * the slot's weight there and 0 elsewhere; the per-expert receive counts are
 * the live pairs of each expert rounded up to a multiple of expert_alignment.
 *   token_recv_row [R,T,R]  row of (r,t) in rank d's buffer, -1 if not sent
 *   recv_tokens    [R]
 *   num_recv_tokens_per_expert [E]
 */
int oracle_normal_layout(int R, int T, int k, int E, const int32_t *topk_idx, const uint8_t *active,
                         int alignment, int capacity, int32_t *token_recv_row, int32_t *recv_tokens,
                         int32_t *num_recv_tokens_per_expert) {
    int status = 0;
    const int E_local = E / R;
    for (int d = 0; d < R; d++) recv_tokens[d] = 0;
    for (int e = 0; e < E; e++) num_recv_tokens_per_expert[e] = 0;
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++) {
            for (int d = 0; d < R; d++) {
                int sent = 0;
                for (int j = 0; j < k; j++) {
                    int e = topk_idx[((int64_t)r * T + t) * k + j];
                    if (pair_is_live(e, r, E, E_local, active) && e / E_local == d) sent = 1;
                }
                int64_t at = ((int64_t)r * T + t) * R + d;
                if (sent) {
                    token_recv_row[at] = recv_tokens[d];
                    recv_tokens[d] += 1;
                    if (token_recv_row[at] >= capacity) status |= ORACLE_OVERFLOW;
                } else {
                    token_recv_row[at] = -1;
                }
            }
            for (int j = 0; j < k; j++) {
                int e = topk_idx[((int64_t)r * T + t) * k + j];
                if (e < -1 || e >= E) status |= ORACLE_BAD_EXPERT;
                if (pair_is_live(e, r, E, E_local, active)) num_recv_tokens_per_expert[e] += 1;
            }
        }
    for (int e = 0; e < E; e++) {
        int n = num_recv_tokens_per_expert[e];
        num_recv_tokens_per_expert[e] = ((n + alignment - 1) / alignment) * alignment;
    }
    return status;
}

/*   recv_x [R,capacity,H] bf16 bits, recv_topk_idx / recv_topk_weights [R,capacity,k],
 *   src_info [R,capacity,2]; rows past recv_tokens[d] are left untouched. */
int oracle_normal_dispatch(int R, int T, int k, int E, int H, int capacity, const uint16_t *x,
                           const int32_t *topk_idx, const float *topk_weights, const uint8_t *active,
                           const int32_t *token_recv_row, uint16_t *recv_x, int32_t *recv_topk_idx,
                           float *recv_topk_weights, int32_t *src_info) {
    int status = 0;
    const int E_local = E / R;
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++)
            for (int d = 0; d < R; d++) {
                int32_t row = token_recv_row[((int64_t)r * T + t) * R + d];
                if (row < 0) continue;
                if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }
                int64_t dst = (int64_t)d * capacity + row;
                for (int h = 0; h < H; h++) recv_x[dst * H + h] = x[((int64_t)r * T + t) * H + h];
                for (int j = 0; j < k; j++) {
                    int64_t p = ((int64_t)r * T + t) * k + j;
                    int e = topk_idx[p];
                    int here = pair_is_live(e, r, E, E_local, active) && e / E_local == d;
                    recv_topk_idx[dst * k + j] = here ? e - d * E_local : -1;
                    recv_topk_weights[dst * k + j] = here ? topk_weights[p] : 0.0f;
                }
                src_info[2 * dst] = r;
                src_info[2 * dst + 1] = t;
            }
    return status;
}

/* out [R,T,H] float64: for (r,t), the sum over ranks d in order of y[d][row]
 * for every row the token was sent to, skipping ranks masked in active_now;
 * zero rows for a masked source rank. */
int oracle_normal_combine(int R, int T, int H, int capacity, const uint16_t *y, const int32_t *token_recv_row,
                          const uint8_t *active_now, double *out) {
    int status = 0;
    for (int r = 0; r < R; r++)
        for (int t = 0; t < T; t++) {
            double *o = out + ((int64_t)r * T + t) * H;
            for (int h = 0; h < H; h++) o[h] = 0.0;
            if (!active_now[r]) continue;
            for (int d = 0; d < R; d++) {
                int32_t row = token_recv_row[((int64_t)r * T + t) * R + d];
                if (row < 0 || !active_now[d]) continue;
                if (row >= capacity) { status |= ORACLE_OVERFLOW; continue; }
                const uint16_t *yr = y + ((int64_t)d * capacity + row) * H;
                for (int h = 0; h < H; h++) o[h] += bf16_to_double(yr[h]);
            }
        }
    return status;
}

/*
 * Replica weight sync and replica gradient reduction ([P3] GPU operations:
 * "Replica weight sync" copies master expert weights to the replicas before
 * expert compute; "Replica gradient reduction" sums the replicas' gradients
 * into the master gradients in backward).  Replica i of logical expert e is
 * physical expert phys_base[e] + i (the routing expansion's numbering).
 */

/* replicas[phys_base[e] + i] = master[e], bytes copied as they are. */
void oracle_replica_weight_sync(int E_log, const int32_t *phys_base, int64_t param_bytes, const uint8_t *master,
                                uint8_t *replicas) {
    for (int e = 0; e < E_log; e++)
        for (int32_t p = phys_base[e]; p < phys_base[e + 1]; p++)
            for (int64_t b = 0; b < param_bytes; b++) replicas[(int64_t)p * param_bytes + b] = master[(int64_t)e * param_bytes + b];
}

/* master[e][i] = sum over replicas, in replica order, of replica_grads[p][i] (float64). */
void oracle_replica_grad_reduce(int E_log, const int32_t *phys_base, int64_t num_params, const float *replica_grads,
                                double *master) {
    for (int e = 0; e < E_log; e++)
        for (int64_t i = 0; i < num_params; i++) {
            double acc = 0.0;
            for (int32_t p = phys_base[e]; p < phys_base[e + 1]; p++) acc += (double)replica_grads[(int64_t)p * num_params + i];
            master[(int64_t)e * num_params + i] = acc;
        }
}
