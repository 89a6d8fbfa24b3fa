/*
 * moonep_oracle.c -- CPU oracle for the balanced expert-parallel hot path
 * (planner, dispatch, combine, weight prefetch, grad-slot reduction).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * helper with the CUDA path.  It is deliberately plain and slow: one thread,
 * no blocking, no fusion, every step in the order the rule states it.
 * Floating point is accumulated in fp64 and rounded once at the end.
 *
 * Sources (web pages about MoonEP; "README" is the project's GitHub README,
 * "MTP" the MarkTechPost article "Moonshot AI Open-Sources MoonEP: A Perfectly
 * Balanced Expert Parallelism Library for MoE Training"):
 *   - maxvio = max_e(T_e / T_bar) - 1, T_bar the per-expert count under perfect
 *     balance: README section "Performance"; MTP, "The problem MoonEP targets".
 *   - every rank receives exactly S x K token slots: README, intro item 1
 *     ("Perfect balance"); MTP, "Core idea: dynamic redundant experts".
 *   - training copies come from at most one remote home group per rank, so
 *     B = E/R; inference may use B < E/R and then reads overflow experts from
 *     their home rows: README, "How to set B"; MTP, "Memory contract".
 *   - rows [0,E) are the home experts, rows [E,E+B) the prefetch slots,
 *     cu_seqlens[E+B] the padded end offset of each row: README, "Weight
 *     buffer" and "dispatch fwd"; MTP, "Memory contract".
 *   - dispatch writes each token straight into its expert-grouped slot and
 *     returns the route weight per slot; combine gathers the K rows back and
 *     weights them: README, "dispatch fwd", "combine fwd", "dispatch bwd".
 *   - reduce_grad adds every rank's slot gradients of a home expert into its
 *     parameter gradient and zeroes the consumed slots: README, "Grad buffer";
 *     MTP, "Memory contract".
 *
 * The pages name the invariants but print no planning rule.  The rule below is
 * this library's fixed reading; every choice the pages leave open is marked
 * [reading].
 *
 * Plan rule.  G = E/R experts per home group, C = S*K slots per rank,
 * home(e) = e / G.
 *  1. cnt[r][e] = picks of expert e on source rank r; T_e = sum_r cnt[r][e];
 *     L_h = sum of T_e over group h; maxvio = max_e T_e / (R*S*K/E) - 1.
 *  2. The group sequence of home rank h lists every pick (r,t,k) whose expert
 *     lies in group h, ordered by expert, then source rank, then token.
 *     [reading]
 *  3. Walker/Vose alias chain over the loads L_h: the lowest-numbered
 *     under-loaded rank takes C - cur from the lowest-numbered over-loaded
 *     rank; a donor that drops below C is served next.  Each rank receives
 *     from at most one donor; there are at most R-1 donations.  [reading]
 *  4. A donor keeps the prefix of its group sequence; its donations take
 *     consecutive ranges after it, in the order they were made.  [reading]
 *  5. On rank s: row e (e in group s) holds the kept picks of e; the distinct
 *     experts s received, in ascending id, take slots b = 0,1,.. (row E+b);
 *     past B they go to row e itself (inference overflow).  [reading]
 *     mode 2 (inference, slots by token count): the B received experts with
 *     the most picks on s take the slots (ties: the lower id), in ascending
 *     id; the rest overflow.  [reading; the README leaves the choice open]
 *     mode 3 (training, fewest copies): step 2 orders the experts of a home
 *     group by their pick count T_e ascending (ties: the lower id) instead
 *     of by id, so a donor keeps its smallest experts and the ranges it gives
 *     away start at its largest ones: a recipient's deficit is covered by as
 *     few distinct experts (copies) as the donation allows, the fewest
 *     possible when one donor serves one recipient.  [reading; the README
 *     calls the planner "near-optimal" without defining the objective]
 *  6. Within a row, picks keep group-sequence order.  Rows are padded to a
 *     multiple of tp (empty rows stay empty); cu_seqlens is the inclusive
 *     running sum of the padded lengths over the E+B rows.  [reading]
 *  7. NvS = roundup(C + 2*G*(tp-1), tp): at most G home rows plus G received
 *     rows are non-empty.  [reading]
 *  8. dst[r,t,k] = dest_rank*NvS + row start + position inside the row.
 *
 * oracle_plan_rank gives one rank's share: steps 1-6 from the gathered counts
 * alone, and step 8 for the rank's own picks in closed form (a pick's place
 * in its group sequence follows from the counts of the ranks before it).
 * The tests check it against oracle_plan's walk on every rank.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* status bits (kept numerically equal to the public header's by the tests) */
#define ORC_BAD_EXPERT 1
#define ORC_DUP_EXPERT 2
#define ORC_COUNT_MISMATCH 4
#define ORC_BAD_ARGS 256

static int64_t pad_up(int64_t n, int64_t tp) { return (n + tp - 1) / tp * tp; }

int64_t oracle_nvs(int S, int K, int E, int R, int tp)
{
    int64_t C = (int64_t)S * K, G = E / R;
    return pad_up(C + 2 * G * (tp - 1), tp);
}

/* ---- bf16 <-> double ------------------------------------------------------ */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round x to the nearest bf16 value, ties to even, directly from fp64 (no
 * intermediate fp32 rounding).  bf16 keeps 8 significant bits and the fp32
 * exponent range; below 2^-126 its spacing is fixed at 2^-133. */
uint16_t oracle_double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double ax = fabs(x);
    if (ax == 0.0) return sign;
    int ex;
    frexp(ax, &ex); /* ax = m * 2^ex, m in [0.5, 1) */
    int lsb = ex - 8;
    if (lsb < -133) lsb = -133;
    double q = ldexp(1.0, lsb);
    double v = nearbyint(ax / q) * q; /* default rounding: to nearest, ties to even */
    float f = (float)v;               /* exact, or +inf past the bf16 range */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* ---- plan --------------------------------------------------------------- */

/* What step 8 needs from the layout (see plan_layout). */
struct layout {
    int64_t *T, *L, *keep, *estart, *don_amt, *don_start;
    int *don_from, *don_to;
    int *order; /* [E]: order[h*G + j] = the j-th expert of group h's sequence */
    int ndon;
};

static void layout_free(struct layout *y)
{
    free(y->T); free(y->L); free(y->keep); free(y->estart); free(y->don_amt);
    free(y->don_start); free(y->don_from); free(y->don_to); free(y->order);
}

/*
 * Steps 1 (loads, maxvio) to 6 from the per-rank counts [R,E] alone: the
 * alias chain, the kept prefixes and donated ranges, the rows of every rank
 * and their padded end offsets.  Writes maxvio, assign, row_counts,
 * slot_expert and cu_seqlens; returns in *y what step 8 needs (free with
 * layout_free).  The counts must hold S*K picks per rank.
 */
static void plan_layout(int R, int S, int K, int E, int B, int tp, int mode, const int32_t *counts,
                        float *maxvio, int32_t *assign, int32_t *row_counts, int32_t *slot_expert,
                        int32_t *cu_seqlens, struct layout *y)
{
    const int G = E / R;
    const int64_t C = (int64_t)S * K;
    const int NR = E + B; /* rows per rank */
    int64_t *T = calloc(E, sizeof(int64_t));
    int64_t *L = calloc(R, sizeof(int64_t));
    for (int e = 0; e < E; e++) {
        for (int r = 0; r < R; r++) T[e] += counts[(int64_t)r * E + e];
        L[e / G] += T[e];
    }
    int64_t maxT = 0;
    for (int e = 0; e < E; e++)
        if (T[e] > maxT) maxT = T[e];
    double Tbar = (double)((int64_t)R * S * K) / (double)E;
    *maxvio = (float)((double)maxT / Tbar - 1.0);

    /* step 3: alias chain.  small is a deque (push to the front when a donor
     * falls below C), large a queue, both seeded in ascending rank order. */
    int64_t *cur = malloc(sizeof(int64_t) * R);
    int *smallq = malloc(sizeof(int) * 2 * R), sh = R, st = R; /* [sh, st) */
    int *largeq = malloc(sizeof(int) * R), lh = 0, lt = 0;
    int *don_from = malloc(sizeof(int) * R), *don_to = malloc(sizeof(int) * R);
    int64_t *don_amt = malloc(sizeof(int64_t) * R);
    int ndon = 0;
    for (int h = 0; h < R; h++) {
        cur[h] = L[h];
        if (L[h] < C) smallq[st++] = h;
        if (L[h] > C) largeq[lt++] = h;
    }
    while (sh < st) {
        int s = smallq[sh++];
        int l = largeq[lh]; /* exists: sum(cur) == R*C */
        int64_t d = C - cur[s];
        don_from[ndon] = l; don_to[ndon] = s; don_amt[ndon] = d; ndon++;
        cur[s] = C;
        cur[l] -= d;
        if (cur[l] < C) { lh++; smallq[--sh] = l; }
        else if (cur[l] == C) lh++;
    }

    /* step 4: kept prefix and donated ranges of each donor's group sequence */
    int64_t *keep = malloc(sizeof(int64_t) * R);
    int64_t *don_start = malloc(sizeof(int64_t) * R);
    for (int h = 0; h < R; h++) {
        keep[h] = L[h];
        for (int j = 0; j < ndon; j++)
            if (don_from[j] == h) keep[h] -= don_amt[j];
    }
    for (int h = 0; h < R; h++) {
        int64_t next = keep[h];
        for (int j = 0; j < ndon; j++)
            if (don_from[j] == h) { don_start[j] = next; next += don_amt[j]; }
    }
    for (int s = 0; s < R; s++) {
        assign[s * 4 + 0] = (int32_t)keep[s];
        assign[s * 4 + 1] = -1;
        assign[s * 4 + 2] = 0;
        assign[s * 4 + 3] = 0;
    }
    for (int j = 0; j < ndon; j++) {
        int s = don_to[j];
        assign[s * 4 + 1] = don_from[j];
        assign[s * 4 + 2] = (int32_t)don_start[j];
        assign[s * 4 + 3] = (int32_t)don_amt[j];
    }

    /* step 2's order of each group's experts: by id, or in mode 3 by pick
     * count ascending with ties by id (a plain insertion sort) */
    int *order = malloc(sizeof(int) * (size_t)E);
    for (int h = 0; h < R; h++) {
        int *o = order + (int64_t)h * G;
        for (int j = 0; j < G; j++) o[j] = h * G + j;
        if (mode == 3)
            for (int j = 1; j < G; j++) {
                int e = o[j], i = j - 1;
                while (i >= 0 && (T[o[i]] > T[e] || (T[o[i]] == T[e] && o[i] > e))) {
                    o[i + 1] = o[i];
                    i--;
                }
                o[i + 1] = e;
            }
    }

    /* start of each expert's run inside its group sequence */
    int64_t *estart = calloc(E, sizeof(int64_t));
    for (int h = 0; h < R; h++) {
        int64_t run = 0;
        for (int j = 0; j < G; j++) {
            int e = order[(int64_t)h * G + j];
            estart[e] = run;
            run += T[e];
        }
    }

    /* step 5: rows of every rank */
    int *rx_e = malloc(sizeof(int) * (size_t)G);
    int64_t *rx_n = malloc(sizeof(int64_t) * (size_t)G);
    memset(row_counts, 0, sizeof(int32_t) * (size_t)R * NR);
    for (int64_t i = 0; i < (int64_t)R * B; i++) slot_expert[i] = -1;
    for (int s = 0; s < R; s++) {
        int32_t *n = row_counts + (int64_t)s * NR;
        for (int e = s * G; e < (s + 1) * G; e++) {
            int64_t lo = estart[e], hi = estart[e] + T[e];
            if (hi > keep[s]) hi = keep[s];
            if (hi > lo) n[e] = (int32_t)(hi - lo);
        }
        int h = assign[s * 4 + 1];
        if (h >= 0) {
            int64_t a = assign[s * 4 + 2], b = a + assign[s * 4 + 3];
            /* the received experts of s in ascending id, with their picks */
            int nrx = 0;
            for (int e = h * G; e < (h + 1) * G; e++) {
                int64_t lo = estart[e] > a ? estart[e] : a;
                int64_t hi = estart[e] + T[e] < b ? estart[e] + T[e] : b;
                if (hi <= lo) continue;
                rx_e[nrx] = e;
                rx_n[nrx] = hi - lo;
                nrx++;
            }
            int q = 0;
            for (int j = 0; j < nrx; j++) {
                int take;
                if (mode == 2) { /* rank by picks, more first, ties by lower id */
                    int better = 0;
                    for (int m = 0; m < nrx; m++)
                        if (rx_n[m] > rx_n[j] || (rx_n[m] == rx_n[j] && m < j)) better++;
                    take = better < B;
                } else {
                    take = j < B;
                }
                if (take) {
                    slot_expert[(int64_t)s * B + q] = rx_e[j];
                    n[E + q] += (int32_t)rx_n[j];
                    q++;
                } else {
                    n[rx_e[j]] += (int32_t)rx_n[j]; /* overflow: the expert's home row */
                }
            }
        }
    }

    /* step 6: padded inclusive end offsets */
    for (int s = 0; s < R; s++) {
        int64_t run = 0;
        for (int i = 0; i < NR; i++) {
            int64_t n = row_counts[(int64_t)s * NR + i];
            run += n ? pad_up(n, tp) : 0;
            cu_seqlens[(int64_t)s * NR + i] = (int32_t)run;
        }
    }

    free(rx_n); free(rx_e); free(largeq); free(smallq); free(cur);
    y->T = T; y->L = L; y->keep = keep; y->estart = estart; y->don_amt = don_amt;
    y->don_start = don_start; y->don_from = don_from; y->don_to = don_to; y->ndon = ndon;
    y->order = order;
}

/*
 * Inputs: topk [R,S,K] int32 (expert ids), tpe [R,E] int32 or NULL (the
 * router's local counts, checked against the picks).  mode 0 = training
 * (B >= E/R), 1 = inference, 2 = inference with slots by token count,
 * 3 = training with the fewest-copies group order (B >= E/R).
 * Outputs (caller-allocated): dst [R,S,K], cu_seqlens [R,E+B],
 * row_counts [R,E+B], slot_expert [R,B] (-1 = unused), counts [R,E],
 * maxvio [1], assign [R,4] = {kept, donor group or -1, received start in the
 * donor's group sequence, received length}.
 * Returns 0 or a bitmask of ORC_* errors; on error the outputs other than
 * counts are not written.
 */
int oracle_plan(int R, int S, int K, int E, int B, int tp, int mode,
                const int32_t *topk, const int32_t *tpe,
                int32_t *dst, int32_t *cu_seqlens, int32_t *row_counts,
                int32_t *slot_expert, int32_t *counts, float *maxvio,
                int32_t *assign)
{
    if (R < 1 || S < 1 || K < 1 || E < 1 || E % R || K > E || B < 0 || tp < 1)
        return ORC_BAD_ARGS;
    const int G = E / R;
    if (mode < 0 || mode > 3 || ((mode == 0 || mode == 3) && B < G)) return ORC_BAD_ARGS;
    const int64_t C = (int64_t)S * K;
    const int NR = E + B; /* rows per rank */
    const int64_t NvS = oracle_nvs(S, K, E, R, tp);
    int status = 0;

    /* validation: ids in [0,E), no expert twice within one token */
    for (int r = 0; r < R; r++)
        for (int t = 0; t < S; t++) {
            const int32_t *tok = topk + ((int64_t)r * S + t) * K;
            for (int k = 0; k < K; k++) {
                int e = tok[k];
                if (e < 0 || e >= E) { status |= ORC_BAD_EXPERT; continue; }
                for (int k2 = 0; k2 < k; k2++)
                    if (tok[k2] == e) status |= ORC_DUP_EXPERT;
            }
        }

    /* step 1: counts over the valid picks */
    memset(counts, 0, sizeof(int32_t) * (size_t)R * E);
    for (int r = 0; r < R; r++)
        for (int64_t i = 0; i < C; i++) {
            int e = topk[(int64_t)r * C + i];
            if (e >= 0 && e < E) counts[(int64_t)r * E + e]++;
        }
    if (tpe)
        for (int64_t i = 0; i < (int64_t)R * E; i++)
            if (tpe[i] != counts[i]) status |= ORC_COUNT_MISMATCH;
    if (status) return status;

    struct layout y;
    plan_layout(R, S, K, E, B, tp, mode, counts, maxvio, assign, row_counts, slot_expert, cu_seqlens, &y);
    int64_t *keep = y.keep, *don_start = y.don_start, *don_amt = y.don_amt;
    int *don_from = y.don_from, *don_to = y.don_to;
    const int ndon = y.ndon;

    /* step 8: walk each group sequence in order and place every pick */
    int32_t *fill = calloc((size_t)R * NR, sizeof(int32_t));
    for (int h = 0; h < R; h++) {
        int64_t g = 0;
        for (int jj = 0; jj < G; jj++) {
            const int e = y.order[(int64_t)h * G + jj];
            for (int r = 0; r < R; r++)
                for (int t = 0; t < S; t++)
                    for (int k = 0; k < K; k++) {
                        int64_t idx = ((int64_t)r * S + t) * K + k;
                        if (topk[idx] != e) continue;
                        int dest = h, row = e;
                        if (g >= keep[h]) {
                            for (int j = 0; j < ndon; j++)
                                if (don_from[j] == h && g >= don_start[j] &&
                                    g < don_start[j] + don_amt[j])
                                    dest = don_to[j];
                            for (int b = 0; b < B; b++)
                                if (slot_expert[(int64_t)dest * B + b] == e) row = E + b;
                        }
                        int64_t ri = (int64_t)dest * NR + row;
                        int64_t n = row_counts[ri];
                        int64_t row_start = cu_seqlens[ri] - pad_up(n, tp);
                        dst[idx] = (int32_t)(dest * NvS + row_start + fill[ri]);
                        fill[ri]++;
                        g++;
                    }
        }
    }

    free(fill);
    layout_free(&y);
    return 0;
}

/*
 * One rank's share of the plan, from what a rank of a real EP group holds:
 * its own picks topk [S,K] and every rank's counts [R,E] (gathered; README
 * "dispatch fwd" gives each rank its local tokens_per_expert).  The layout
 * (steps 1-6) needs only the counts.  In step 2's order, a pick of expert e
 * at token t of this rank sits at
 *   g = estart[e] + sum_{q < rank} counts[q][e] + (its rank among this
 *       rank's picks of e, in token order)
 * of its group sequence; step 8 puts it at row position g - (the first g of
 * that row's run of e), a closed form of the walk oracle_plan performs.
 * Outputs: dst [S,K] for this rank's picks; cu_seqlens, row_counts,
 * slot_expert, maxvio and assign of the whole group, as oracle_plan writes
 * them.  Returns 0 or ORC_* bits: BAD_EXPERT / DUP_EXPERT in the rank's
 * picks; COUNT_MISMATCH when row `rank` of the counts differs from the
 * picks, or a row holds a negative count or does not sum to S*K.
 */
int oracle_plan_rank(int R, int S, int K, int E, int B, int tp, int mode, int rank,
                     const int32_t *topk, const int32_t *counts,
                     int32_t *dst, int32_t *cu_seqlens, int32_t *row_counts,
                     int32_t *slot_expert, float *maxvio, int32_t *assign)
{
    if (R < 1 || S < 1 || K < 1 || E < 1 || E % R || K > E || B < 0 || tp < 1 || rank < 0 || rank >= R)
        return ORC_BAD_ARGS;
    const int G = E / R;
    if (mode < 0 || mode > 3 || ((mode == 0 || mode == 3) && B < G)) return ORC_BAD_ARGS;
    const int64_t C = (int64_t)S * K;
    const int NR = E + B;
    const int64_t NvS = oracle_nvs(S, K, E, R, tp);
    int status = 0;

    int64_t *mine = calloc(E, sizeof(int64_t));
    for (int t = 0; t < S; t++) {
        const int32_t *tok = topk + (int64_t)t * K;
        for (int k = 0; k < K; k++) {
            int e = tok[k];
            if (e < 0 || e >= E) { status |= ORC_BAD_EXPERT; continue; }
            for (int k2 = 0; k2 < k; k2++)
                if (tok[k2] == e) status |= ORC_DUP_EXPERT;
            mine[e]++;
        }
    }
    for (int e = 0; e < E; e++)
        if (mine[e] != counts[(int64_t)rank * E + e]) status |= ORC_COUNT_MISMATCH;
    for (int q = 0; q < R; q++) {
        int64_t sum = 0;
        for (int e = 0; e < E; e++) {
            int32_t v = counts[(int64_t)q * E + e];
            if (v < 0) status |= ORC_COUNT_MISMATCH;
            sum += v;
        }
        if (sum != C) status |= ORC_COUNT_MISMATCH;
    }
    free(mine);
    if (status) return status;

    struct layout y;
    plan_layout(R, S, K, E, B, tp, mode, counts, maxvio, assign, row_counts, slot_expert, cu_seqlens, &y);
    int64_t *seen = calloc(E, sizeof(int64_t));
    for (int t = 0; t < S; t++)
        for (int k = 0; k < K; k++) {
            const int e = topk[(int64_t)t * K + k], h = e / G;
            int64_t pre = 0;
            for (int q = 0; q < rank; q++) pre += counts[(int64_t)q * E + e];
            const int64_t g = y.estart[e] + pre + seen[e]++;
            int dest = h, row = e;
            int64_t first = y.estart[e];
            if (g >= y.keep[h]) {
                for (int j = 0; j < y.ndon; j++)
                    if (y.don_from[j] == h && g >= y.don_start[j] && g < y.don_start[j] + y.don_amt[j]) {
                        dest = y.don_to[j];
                        first = y.estart[e] > y.don_start[j] ? y.estart[e] : y.don_start[j];
                    }
                for (int b = 0; b < B; b++)
                    if (slot_expert[(int64_t)dest * B + b] == e) row = E + b;
            }
            const int64_t ri = (int64_t)dest * NR + row;
            const int64_t row_start = cu_seqlens[ri] - pad_up(row_counts[ri], tp);
            dst[(int64_t)t * K + k] = (int32_t)(dest * NvS + row_start + (g - first));
        }
    free(seen);
    layout_free(&y);
    return 0;
}

/* ---- dispatch / combine --------------------------------------------------- */

/* buf[dst[r,t,k], :] = hidden[r,t,:]; w_nvs[dst] = w[r,t,k] (both optional). */
void oracle_dispatch(int R, int S, int K, int H, const int32_t *dst,
                     const uint16_t *hidden, const float *w, uint16_t *buf, float *w_nvs)
{
    for (int r = 0; r < R; r++)
        for (int t = 0; t < S; t++)
            for (int k = 0; k < K; k++) {
                int64_t idx = ((int64_t)r * S + t) * K + k;
                int64_t d = dst[idx];
                for (int c = 0; c < H; c++)
                    buf[d * H + c] = hidden[((int64_t)r * S + t) * H + c];
                if (w && w_nvs) w_nvs[d] = w[idx];
            }
}

/* out[r,t,:] = bf16( sum_k w_nvs[d_k] * y[d_k,:] ), the sum in fp64 and
 * rounded once; w_nvs NULL = unweighted.  gathered_w[r,t,k] = w_nvs[d_k]. */
void oracle_combine(int R, int S, int K, int H, const int32_t *dst, const uint16_t *y,
                    const float *w_nvs, uint16_t *out, float *gathered_w)
{
    for (int r = 0; r < R; r++)
        for (int t = 0; t < S; t++) {
            const int32_t *d = dst + ((int64_t)r * S + t) * K;
            for (int c = 0; c < H; c++) {
                double acc = 0.0;
                for (int k = 0; k < K; k++) {
                    double wk = w_nvs ? (double)w_nvs[d[k]] : 1.0;
                    acc += wk * bf16_to_double(y[(int64_t)d[k] * H + c]);
                }
                out[((int64_t)r * S + t) * H + c] = oracle_double_to_bf16(acc);
            }
            if (w_nvs && gathered_w)
                for (int k = 0; k < K; k++)
                    gathered_w[((int64_t)r * S + t) * K + k] = w_nvs[d[k]];
        }
}

/* ---- weight prefetch / grad-slot reduction (one projection per call) ------ */

/* pool[s,:] = W[slot_expert[s],:] for every used slot s of the R*B slots. */
void oracle_prefetch(int R, int B, int64_t HHp, const int32_t *slot_expert,
                     const uint16_t *W, uint16_t *pool)
{
    for (int64_t s = 0; s < (int64_t)R * B; s++) {
        int e = slot_expert[s];
        if (e < 0) continue;
        memcpy(pool + s * HHp, W + (int64_t)e * HHp, sizeof(uint16_t) * (size_t)HHp);
    }
}

/* For each expert e: G[e] += sum of RB[s] over the slots s holding e, in
 * ascending slot order (s = r*B + b), the sum in fp64 rounded once to fp32;
 * then every consumed slot is set to +0.0.  Unused slots are untouched. */
void oracle_reduce_grad(int R, int B, int E, int64_t HHp, const int32_t *slot_expert,
                        float *Gr, float *RB)
{
    int64_t nslot = (int64_t)R * B;
    int64_t *holders = malloc(sizeof(int64_t) * (size_t)(nslot > 0 ? nslot : 1));
    for (int e = 0; e < E; e++) {
        int64_t nh = 0;
        for (int64_t s = 0; s < nslot; s++)
            if (slot_expert[s] == e) holders[nh++] = s; /* ascending slot order */
        if (nh == 0) continue;
        for (int64_t i = 0; i < HHp; i++) {
            double acc = (double)Gr[(int64_t)e * HHp + i];
            for (int64_t j = 0; j < nh; j++) acc += (double)RB[holders[j] * HHp + i];
            Gr[(int64_t)e * HHp + i] = (float)acc;
        }
        for (int64_t j = 0; j < nh; j++)
            for (int64_t i = 0; i < HHp; i++) RB[holders[j] * HHp + i] = 0.0f;
    }
    free(holders);
}
