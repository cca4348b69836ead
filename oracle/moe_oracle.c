/*
 * moe_oracle.c -- the ORACLE for the MoE dispatch / combine path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded CPU
 * statement of what every step of the path computes, written so that a
 * reader can check it against the source pages by eye.  It exists to check
 * the CUDA library, never to stand in for it: only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg may load it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Sources (page title -- section):
 *   [EC]  "Expert Coupling in MoE Pretraining: Reducing All-to-All Overhead
 *          with Correlated Placement and Token Shuffling" (PicX summary)
 *   [DD]  "DODOCO: MoE AlltoAll Traffic Matrices on Real Text" (dataset card)
 *   [A2A] "AllToAllDispatchScenario" (mlsysim API page)
 *
 * Notation: T tokens, H hidden size, E experts, k = top-k, R = expert-parallel
 * ranks, T_r = T / R tokens per source rank, src(t) = t / T_r, p[e] = rank
 * holding expert e, S(t) = token t's selected experts in slot order.
 *
 * Floating point: gates are computed in double and rounded once to float.
 * The combine accumulates in float with explicit fmaf, because that
 * accumulation order and precision is part of the specified result.
 *
 * Every function returns 0 on success and a non-zero code on bad arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16 <-> float, round-to-nearest-even written out.                        */
/* ------------------------------------------------------------------------ */

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint16_t float_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)      /* NaN: keep it a quiet NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    /* add half an ulp of the kept part, plus one if the kept part is odd */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* Router: top-k selection and gate weights.                                 */
/* [EC] "Background": each token is routed to its top-k of E experts.        */
/* [EC] "Method 1": routing probabilities travel with the dispatched rows.   */
/* ------------------------------------------------------------------------ */

typedef struct {
    float logit;
    int32_t expert;
} cand_t;

/* Larger logit first (IEEE comparison, so -0.0 equals +0.0); equal logits:
 * lower expert index first. */
static int cmp_cand(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->logit > y->logit) return -1;
    if (x->logit < y->logit) return 1;
    return (x->expert > y->expert) - (x->expert < y->expert);
}

/*
 * idx[t*k + j] = the j-th expert of token t in (logit desc, expert asc) order.
 * gate_mode 0: w_j = softmax over the k selected logits.
 * gate_mode 1: w_j = softmax over all E logits, read at the selected experts.
 * Both use the largest logit (slot 0) as the shift; the result is rounded to
 * float once.
 */
int oracle_route_topk(const float *logits, int64_t T, int E, int k, int gate_mode,
                      int32_t *idx, float *w)
{
    if (T < 0 || E < 1 || k < 1 || k > E || (gate_mode != 0 && gate_mode != 1))
        return 1;
    cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)E);
    if (!c) return 2;
    for (int64_t t = 0; t < T; ++t) {
        const float *row = logits + t * E;
        for (int e = 0; e < E; ++e) {
            c[e].logit = row[e];
            c[e].expert = e;
        }
        qsort(c, (size_t)E, sizeof(cand_t), cmp_cand);
        for (int j = 0; j < k; ++j)
            idx[t * k + j] = c[j].expert;

        double m = (double)c[0].logit;
        double denom = 0.0;
        if (gate_mode == 0) {
            for (int j = 0; j < k; ++j) denom += exp((double)c[j].logit - m);
        } else {
            for (int e = 0; e < E; ++e) denom += exp((double)row[e] - m);
        }
        for (int j = 0; j < k; ++j)
            w[t * k + j] = (float)(exp((double)c[j].logit - m) / denom);
    }
    free(c);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dispatch layout.                                                          */
/* [DD] "Reading the counts": counts are token-expert assignments, a token   */
/*      sent to several experts on one rank is counted once per expert, and  */
/*      each row of the send matrix sums to (tokens per rank) x top-k.       */
/* [DD] "Setup": each rank routes a contiguous block of tokens; contiguous   */
/*      placement puts experts r*E/R .. (r+1)*E/R-1 on rank r.               */
/* [EC] "Method 1": the deduplicating dispatcher sends one row per distinct  */
/*      (token, destination rank) pair, carrying every selected expert there.*/
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t a, b, c;    /* sort key, compared in this order */
    int64_t t;
    int j;
} lkey_t;

static int cmp_lkey(const void *x_, const void *y_)
{
    const lkey_t *x = (const lkey_t *)x_, *y = (const lkey_t *)y_;
    if (x->a != y->a) return x->a < y->a ? -1 : 1;
    if (x->b != y->b) return x->b < y->b ? -1 : 1;
    if (x->c != y->c) return x->c < y->c ? -1 : 1;
    return 0;
}

/*
 * Conventional rows: one per (t, j), ordered by (p[e], e, t) with e = S(t)_j,
 * i.e. grouped by destination rank, then by expert, then by token.
 * Dedup rows: one per distinct (t, d) with d in {p[e] : e in S(t)}, ordered
 * by (d, t); bit j of the row's mask is set when p[S(t)_j] = d.
 *
 * Outputs (all sizes are the caller's):
 *   assign_row[T*k]      conventional row of (t, j), in both modes
 *   row_of_slot[T*k]     row of (t, j) in this mode's layout
 *   row_token[n_rows]    token of each row
 *   row_mask[n_rows]     slots of that token carried by the row
 *   send_counts[R*R]     [s*R + d] rows from source rank s to rank d
 *   expert_counts[E]     #{t : e in S(t)}
 *   expert_offsets[E+1]  first conventional row of expert e; [E] = T*k
 *   rank_offsets[R+1]    first row of rank d in this mode; [R] = n_rows
 *   n_rows               number of rows in this mode
 */
int oracle_dispatch_layout(const int32_t *idx, int64_t T, int E, int k, int R,
                           const int32_t *p, int mode,
                           int32_t *row_of_slot, int32_t *assign_row,
                           int32_t *row_token, uint32_t *row_mask,
                           int64_t *send_counts, int64_t *expert_counts,
                           int64_t *expert_offsets, int64_t *rank_offsets,
                           int64_t *n_rows)
{
    if (T < 0 || E < 1 || k < 1 || k > E || k > 32 || R < 1 || T % R != 0 ||
        (mode != 0 && mode != 1))
        return 1;
    for (int e = 0; e < E; ++e)
        if (p[e] < 0 || p[e] >= R) return 1;
    for (int64_t i = 0; i < T * k; ++i)
        if (idx[i] < 0 || idx[i] >= E) return 1;
    const int64_t Tr = T / R;
    if (Tr == 0) {             /* no tokens: everything is empty */
        for (int e = 0; e < E; ++e) { expert_counts[e] = 0; expert_offsets[e] = 0; }
        expert_offsets[E] = 0;
        for (int64_t i = 0; i < (int64_t)R * R; ++i) send_counts[i] = 0;
        for (int d = 0; d <= R; ++d) rank_offsets[d] = 0;
        *n_rows = 0;
        return 0;
    }

    /* conventional positions: sort all (t, j) by (p[e], e, t) */
    int64_t npairs = T * k;
    lkey_t *keys = (lkey_t *)malloc(sizeof(lkey_t) * (size_t)(npairs > 0 ? npairs : 1));
    if (!keys) return 2;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            lkey_t *q = &keys[t * k + j];
            q->a = p[e];
            q->b = e;
            q->c = t;
            q->t = t;
            q->j = j;
        }
    qsort(keys, (size_t)npairs, sizeof(lkey_t), cmp_lkey);
    for (int64_t i = 0; i < npairs; ++i)
        assign_row[keys[i].t * k + keys[i].j] = (int32_t)i;

    for (int e = 0; e < E; ++e) expert_counts[e] = 0;
    for (int64_t i = 0; i < npairs; ++i) expert_counts[idx[i]] += 1;

    /* first conventional row of expert e = number of pairs whose (p, e')
     * key sorts before (p[e], e) */
    for (int e = 0; e < E; ++e) {
        int64_t before = 0;
        for (int e2 = 0; e2 < E; ++e2)
            if (p[e2] < p[e] || (p[e2] == p[e] && e2 < e)) before += expert_counts[e2];
        expert_offsets[e] = before;
    }
    expert_offsets[E] = npairs;

    for (int64_t i = 0; i < (int64_t)R * R; ++i) send_counts[i] = 0;

    if (mode == 0) {
        for (int64_t i = 0; i < npairs; ++i) {
            int64_t t = keys[i].t;
            int j = keys[i].j;
            row_of_slot[t * k + j] = (int32_t)i;
            row_token[i] = (int32_t)t;
            row_mask[i] = 1u << j;
        }
        for (int64_t t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                send_counts[(t / Tr) * R + p[idx[t * k + j]]] += 1;
        for (int d = 0; d <= R; ++d) {
            int64_t before = 0;
            for (int e = 0; e < E; ++e)
                if (p[e] < d) before += expert_counts[e];
            rank_offsets[d] = before;
        }
        *n_rows = npairs;
        free(keys);
        return 0;
    }

    /* dedup: one entry per distinct (t, d), sorted by (d, t) */
    int64_t nd = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int d = p[idx[t * k + j]];
            int seen = 0;
            for (int j2 = 0; j2 < j; ++j2)
                if (p[idx[t * k + j2]] == d) seen = 1;
            if (!seen) {
                lkey_t *q = &keys[nd++];
                q->a = d;
                q->b = t;
                q->c = 0;
                q->t = t;
                q->j = d; /* remember the rank */
            }
        }
    qsort(keys, (size_t)nd, sizeof(lkey_t), cmp_lkey);
    for (int64_t i = 0; i < nd; ++i) {
        int64_t t = keys[i].t;
        int d = keys[i].j;
        uint32_t mask = 0;
        for (int j = 0; j < k; ++j)
            if (p[idx[t * k + j]] == d) {
                mask |= 1u << j;
                row_of_slot[t * k + j] = (int32_t)i;
            }
        row_token[i] = (int32_t)t;
        row_mask[i] = mask;
        send_counts[(t / Tr) * R + d] += 1;
    }
    for (int d = 0; d <= R; ++d) {
        int64_t before = 0;
        for (int64_t i = 0; i < nd; ++i)
            if (keys[i].j < d) before += 1;
        rank_offsets[d] = before;
    }
    *n_rows = nd;
    free(keys);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Dispatch permute.  The dispatch buffer holds, in row order, the hidden    */
/* state of each row's token ([DD] "Reading the counts": payload = count x   */
/* hidden x bytes per element).                                              */
/* ------------------------------------------------------------------------ */

int oracle_dispatch_permute(const uint16_t *x, int64_t T, int64_t H,
                            const int32_t *row_token, int64_t n_rows, uint16_t *out)
{
    if (T < 0 || H < 1 || n_rows < 0) return 1;
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t t = row_token[r];
        if (t < 0 || t >= T) return 1;
        memcpy(out + r * H, x + t * H, sizeof(uint16_t) * (size_t)H);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Receiver-side expand of deduplicated rows.                                */
/* [EC] Method 1, Deduplicating Dispatcher: a rank receives one row per      */
/* (token, rank) carrying all of the token's experts on that rank; each of   */
/* those experts needs its own copy of the row.  Slot j of token t goes to   */
/* its conventional (expert-grouped) position assign_row[t][j], copied from  */
/* the deduplicated row row_of_slot[t][j] that carried it.                   */
/* ------------------------------------------------------------------------ */

int oracle_dedup_expand(const uint16_t *wire, int64_t n_wire, int64_t H,
                        const int32_t *row_of_slot, const int32_t *assign_row, int64_t T, int k,
                        int64_t n_out, uint16_t *out)
{
    if (T < 0 || H < 1 || k < 1 || n_wire < 0 || n_out < 0) return 1;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t src = row_of_slot[t * k + j], dst = assign_row[t * k + j];
            if (src < 0 || src >= n_wire || dst < 0 || dst >= n_out) return 1;
            memcpy(out + dst * H, wire + src * H, sizeof(uint16_t) * (size_t)H);
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Combine.                                                                  */
/* [DD] "Send matrices": combine returns the same volumes in reverse.        */
/* [EC] "The Communication Bottleneck": dispatch and combine per MoE layer.  */
/* The result is the gate-weighted sum of the token's expert outputs,        */
/* accumulated in float in ascending expert order and rounded to bf16 once.  */
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t key1, key2;
    int j;
} slot_t;

static int cmp_slot(const void *x_, const void *y_)
{
    const slot_t *x = (const slot_t *)x_, *y = (const slot_t *)y_;
    if (x->key1 != y->key1) return x->key1 < y->key1 ? -1 : 1;
    if (x->key2 != y->key2) return x->key2 < y->key2 ? -1 : 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * y: expert outputs, one row per (t, j) at row assign_row[t*k+j], bf16 [*, H].
 * mode 0 (fused): out[t] = bf16( sum over slots by ascending expert of
 *                 fmaf(w, y, acc) ), acc starting at +0.0f.
 * mode 1 (wire):  for each destination rank d of t, ascending d:
 *                   z(t,d) = bf16( same sum over the slots with p[e] = d );
 *                   written to z at row row_of_slot of those slots;
 *                 out[t] = bf16( sum over ascending d of float(z(t,d)) ).
 */
int oracle_combine(const uint16_t *y, int64_t y_rows, const int32_t *assign_row,
                   const int32_t *idx, const float *w, int64_t T, int k, int64_t H,
                   int mode, const int32_t *p, int R, const int32_t *row_of_slot,
                   uint16_t *z, uint16_t *out)
{
    if (T < 0 || k < 1 || H < 1 || (mode != 0 && mode != 1)) return 1;
    slot_t *s = (slot_t *)malloc(sizeof(slot_t) * (size_t)k);
    if (!s) return 2;
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t r = assign_row[t * k + j];
            if (r < 0 || r >= y_rows) { free(s); return 1; }
            int e = idx[t * k + j];
            s[j].key1 = mode == 0 ? e : p[e];
            s[j].key2 = e;
            s[j].j = j;
        }
        qsort(s, (size_t)k, sizeof(slot_t), cmp_slot);
        for (int64_t h = 0; h < H; ++h) {
            if (mode == 0) {
                float acc = 0.0f;
                for (int i = 0; i < k; ++i) {
                    int j = s[i].j;
                    float v = bf16_to_float(y[(int64_t)assign_row[t * k + j] * H + h]);
                    acc = fmaf(w[t * k + j], v, acc);
                }
                out[t * H + h] = float_to_bf16(acc);
            } else {
                float total = 0.0f;
                int i = 0;
                while (i < k) {
                    int64_t d = s[i].key1;
                    int64_t zrow = row_of_slot[t * k + s[i].j];
                    float acc = 0.0f;
                    for (; i < k && s[i].key1 == d; ++i) {
                        int j = s[i].j;
                        float v = bf16_to_float(y[(int64_t)assign_row[t * k + j] * H + h]);
                        acc = fmaf(w[t * k + j], v, acc);
                    }
                    uint16_t zb = float_to_bf16(acc);
                    if (z) z[zrow * H + h] = zb;
                    total = total + bf16_to_float(zb);
                }
                out[t * H + h] = float_to_bf16(total);
            }
        }
    }
    (void)R;
    free(s);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Co-selection statistics.                                                  */
/* [EC] "Correlated Placement": W[e,e'] counts tokens selecting both e, e'.  */
/* [EC] "Cross-layer correlation": layer-l experts predict layer-l+1 ones.   */
/* ------------------------------------------------------------------------ */

/*
 * W[e*E+e'] += #{t < T_fit : e in S(t) and e' in S(t)}  (diagonal = load)
 * C[e*E+e'] += #{(t, i, j) : t < T_fit, S_l(t)_i = e, S_l+1(t)_j = e'}
 * W or C may be NULL; accumulate = 0 clears them first.
 */
int oracle_coselect(const int32_t *idx_l, const int32_t *idx_next, int64_t T_fit,
                    int E, int k, uint32_t *W, uint32_t *C, int accumulate)
{
    if (T_fit < 0 || E < 1 || k < 1) return 1;
    if (!accumulate) {
        if (W) memset(W, 0, sizeof(uint32_t) * (size_t)E * E);
        if (C) memset(C, 0, sizeof(uint32_t) * (size_t)E * E);
    }
    for (int64_t t = 0; t < T_fit; ++t)
        for (int i = 0; i < k; ++i)
            for (int j = 0; j < k; ++j) {
                int a = idx_l[t * k + i];
                if (a < 0 || a >= E) return 1;
                if (W) {
                    int b = idx_l[t * k + j];
                    W[(int64_t)a * E + b] += 1;
                }
                if (C && idx_next) {
                    int b = idx_next[t * k + j];
                    if (b < 0 || b >= E) return 1;
                    C[(int64_t)a * E + b] += 1;
                }
            }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Correlated placement.                                                     */
/* [EC] "Correlated Placement": a Kernighan-Lin-style local search starts    */
/* from contiguous placement and swaps experts between GPUs to maximise the  */
/* sum of W over pairs that share a GPU; every GPU keeps exactly E/EP        */
/* experts.  The page does not print the search itself, so the steps below  */
/* are the plainest reading: repeat the single best swap while it gains.     */
/* ------------------------------------------------------------------------ */

/* sum of W[e][e'] over unordered pairs e != e' on the same rank */
long long oracle_placement_objective(const uint32_t *W, int E, const int32_t *p)
{
    long long s = 0;
    for (int a = 0; a < E; ++a)
        for (int b = a + 1; b < E; ++b)
            if (p[a] == p[b]) s += (long long)W[(int64_t)a * E + b];
    return s;
}

typedef struct {
    uint32_t wv;
    int a, b;
} pair_t;

static int cmp_pair(const void *x_, const void *y_)
{
    const pair_t *x = (const pair_t *)x_, *y = (const pair_t *)y_;
    if (x->wv != y->wv) return x->wv > y->wv ? -1 : 1;
    if (x->a != y->a) return x->a < y->a ? -1 : 1;
    return (x->b > y->b) - (x->b < y->b);
}

/*
 * seed_mode 0: start from contiguous placement (the page's starting point).
 * seed_mode 1: greedy pair seed ("co-locate the top pairs first"): scan the
 *   pairs e < e' with W[e][e'] > 0 by (W desc, e asc, e' asc);
 *   both unplaced  -> both go to the rank with the most free slots (lowest
 *                     rank on ties) if it has at least two;
 *   one placed     -> the other joins it if its rank has a free slot;
 *   then experts still unplaced go, in ascending order, to the lowest rank
 *   with a free slot.
 * refine != 0: repeat the swap (a on P, b on Q, P != Q, a < b) of largest
 *   gain  A[a][Q] - A[a][P] + A[b][P] - A[b][Q] - 2 W[a][b]
 *   (A[e][d] = sum of W[e][e'] over e' != e on rank d), lowest (a, b) on
 *   ties, while that gain is > 0, at most E*E swaps.
 * W must be symmetric, as the co-selection count is.
 */
int oracle_place_correlated(const uint32_t *W, int E, int R, int seed_mode, int refine,
                            int32_t *p)
{
    if (E < 1 || R < 1 || E % R != 0 || (seed_mode != 0 && seed_mode != 1)) return 1;
    const int cap = E / R;

    if (seed_mode == 0) {
        for (int e = 0; e < E; ++e) p[e] = e / cap;
    } else {
        int *fill = (int *)calloc((size_t)R, sizeof(int));
        int64_t np = 0;
        pair_t *pairs = (pair_t *)malloc(sizeof(pair_t) * ((size_t)E * (E - 1) / 2 + 1));
        if (!fill || !pairs) { free(fill); free(pairs); return 2; }
        for (int e = 0; e < E; ++e) p[e] = -1;
        for (int a = 0; a < E; ++a)
            for (int b = a + 1; b < E; ++b)
                if (W[(int64_t)a * E + b] > 0) {
                    pairs[np].wv = W[(int64_t)a * E + b];
                    pairs[np].a = a;
                    pairs[np].b = b;
                    ++np;
                }
        qsort(pairs, (size_t)np, sizeof(pair_t), cmp_pair);
        for (int64_t i = 0; i < np; ++i) {
            int a = pairs[i].a, b = pairs[i].b;
            if (p[a] < 0 && p[b] < 0) {
                int best = 0;
                for (int d = 1; d < R; ++d)
                    if (cap - fill[d] > cap - fill[best]) best = d;
                if (cap - fill[best] >= 2) {
                    p[a] = best;
                    p[b] = best;
                    fill[best] += 2;
                }
            } else if (p[a] >= 0 && p[b] < 0) {
                if (fill[p[a]] < cap) { p[b] = p[a]; fill[p[a]] += 1; }
            } else if (p[a] < 0 && p[b] >= 0) {
                if (fill[p[b]] < cap) { p[a] = p[b]; fill[p[b]] += 1; }
            }
        }
        for (int e = 0; e < E; ++e)
            if (p[e] < 0)
                for (int d = 0; d < R; ++d)
                    if (fill[d] < cap) { p[e] = d; fill[d] += 1; break; }
        free(fill);
        free(pairs);
    }
    if (!refine) return 0;

    long long *A = (long long *)malloc(sizeof(long long) * (size_t)E * R);
    if (!A) return 2;
    for (long long iter = 0; iter < (long long)E * E; ++iter) {
        /* A[e][d] = sum of W[e][e'] over e' != e with p[e'] = d */
        for (int64_t i = 0; i < (int64_t)E * R; ++i) A[i] = 0;
        for (int e = 0; e < E; ++e)
            for (int e2 = 0; e2 < E; ++e2)
                if (e2 != e) A[(int64_t)e * R + p[e2]] += W[(int64_t)e * E + e2];
        long long best_gain = 0;
        int ba = -1, bb = -1;
        for (int a = 0; a < E; ++a)
            for (int b = a + 1; b < E; ++b) {
                int P = p[a], Q = p[b];
                if (P == Q) continue;
                long long g = A[(int64_t)a * R + Q] - A[(int64_t)a * R + P] +
                              A[(int64_t)b * R + P] - A[(int64_t)b * R + Q] -
                              2LL * (long long)W[(int64_t)a * E + b];
                if (g > best_gain) { best_gain = g; ba = a; bb = b; }
            }
        if (ba < 0) break;
        int P = p[ba];
        p[ba] = p[bb];
        p[bb] = P;
    }
    free(A);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Token shuffle.                                                            */
/* [EC] "Method 2: Token Shuffling", Mechanism: predict each token's owner   */
/* rank at the next layer; every rank owns exactly T/EP tokens, so tokens    */
/* are assigned in decreasing confidence to their most preferred rank with   */
/* capacity left.  The single-expert form of the prediction is used: the     */
/* token's top-1 expert e1 at layer l predicts the next-layer expert         */
/* argmax_e' C[e1][e'].                                                      */
/* ------------------------------------------------------------------------ */

typedef struct {
    uint64_t num, den;   /* confidence = num / den; den = 0 means zero */
    int64_t t;
} conf_t;

/* decreasing confidence, then increasing token; a zero-count row has
 * confidence 0 */
static int cmp_conf(const void *x_, const void *y_)
{
    const conf_t *x = (const conf_t *)x_, *y = (const conf_t *)y_;
    /* compare x.num/x.den with y.num/y.den exactly; 0/0 counts as 0 */
    uint64_t xn = x->den ? x->num : 0, xd = x->den ? x->den : 1;
    uint64_t yn = y->den ? y->num : 0, yd = y->den ? y->den : 1;
    unsigned __int128 l = (unsigned __int128)xn * yd, r = (unsigned __int128)yn * xd;
    if (l != r) return l > r ? -1 : 1;
    return (x->t > y->t) - (x->t < y->t);
}

/*
 * For each token t with top-1 expert e1 = idx_l[t*k]:
 *   e*   = argmax_e' C[e1][e'] (lowest e' on ties); first choice p_next[e*];
 *   then the other ranks by sigma(d) = sum_{e' : p_next[e'] = d} C[e1][e']
 *   descending, lowest d on ties;
 *   confidence = C[e1][e*] / sum_e' C[e1][e'].
 *   A row of C that is all zero gives confidence 0 and the preference order
 *   src(t), then the other ranks ascending.
 * Tokens are visited by (confidence desc, t asc); each takes its first
 * preferred rank that still has fewer than T/R tokens.
 * pred_rank[t] = the rank t was assigned; rank d's tokens take the new
 * positions d*T_r .. (d+1)*T_r - 1 in ascending t; perm[t] = new position,
 * inv[perm[t]] = t.
 */
int oracle_token_shuffle(const int32_t *idx_l, const uint32_t *C, const int32_t *p_next,
                         int64_t T, int E, int k, int R,
                         int32_t *pred_rank, int32_t *perm, int32_t *inv)
{
    if (T < 0 || E < 1 || k < 1 || R < 1 || T % R != 0) return 1;
    const int64_t Tr = T / R;
    int32_t *pref = (int32_t *)malloc(sizeof(int32_t) * (size_t)E * R);
    uint64_t *num = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)E);
    uint64_t *den = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)E);
    uint64_t *sigma = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)R);
    conf_t *order = (conf_t *)malloc(sizeof(conf_t) * (size_t)(T > 0 ? T : 1));
    int64_t *load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    int rc = 0;
    if (!pref || !num || !den || !sigma || !order || !load) { rc = 2; goto done; }

    for (int e1 = 0; e1 < E; ++e1) {
        const uint32_t *row = C + (int64_t)e1 * E;
        uint64_t total = 0;
        int best = 0;
        for (int e = 0; e < E; ++e) {
            total += row[e];
            if (row[e] > row[best]) best = e;
        }
        num[e1] = row[best];
        den[e1] = total;
        for (int d = 0; d < R; ++d) sigma[d] = 0;
        for (int e = 0; e < E; ++e) sigma[p_next[e]] += row[e];
        int32_t *pl = pref + (int64_t)e1 * R;
        pl[0] = p_next[best];
        int n = 1;
        /* remaining ranks, sigma descending, lowest rank on ties:
         * selection by repeated scan */
        while (n < R) {
            int pick = -1;
            for (int d = 0; d < R; ++d) {
                int used = 0;
                for (int i = 0; i < n; ++i)
                    if (pl[i] == d) used = 1;
                if (used) continue;
                if (pick < 0 || sigma[d] > sigma[pick]) pick = d;
            }
            pl[n++] = pick;
        }
    }

    for (int64_t t = 0; t < T; ++t) {
        int e1 = idx_l[t * k];
        if (e1 < 0 || e1 >= E) { rc = 1; goto done; }
        order[t].num = num[e1];
        order[t].den = den[e1];
        order[t].t = t;
    }
    qsort(order, (size_t)T, sizeof(conf_t), cmp_conf);

    for (int64_t i = 0; i < T; ++i) {
        int64_t t = order[i].t;
        int e1 = idx_l[t * k];
        int chosen = -1;
        if (den[e1] == 0) {
            int s = (int)(t / Tr);
            if (load[s] < Tr) chosen = s;
            for (int d = 0; chosen < 0 && d < R; ++d)
                if (load[d] < Tr) chosen = d;
        } else {
            const int32_t *pl = pref + (int64_t)e1 * R;
            for (int n = 0; chosen < 0 && n < R; ++n)
                if (load[pl[n]] < Tr) chosen = pl[n];
        }
        pred_rank[t] = chosen;
        load[chosen] += 1;
    }

    for (int d = 0; d < R; ++d) load[d] = 0;
    for (int64_t t = 0; t < T; ++t) {
        int d = pred_rank[t];
        int64_t pos = (int64_t)d * Tr + load[d];
        load[d] += 1;
        perm[t] = (int32_t)pos;
        inv[pos] = (int32_t)t;
    }
done:
    free(pref); free(num); free(den); free(sigma); free(order); free(load);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Pair-based shuffle prediction.                                            */
/* [EC] "Method 2: Token Shuffling", Mechanism, Prediction: the owner rank at */
/* layer l+1 is predicted from the experts the token selected at the two     */
/* preceding layers -- a pair-based lookup -- with a fall back to the        */
/* single-expert prediction where the pair has too few observations.        */
/* The pair counts extend C the way C extends W:                             */
/*   C2[a][b][e'] = #{t < T_fit : a in S_{l-1}(t), b in S_l(t),              */
/*                                e' in S_{l+1}(t)}   (all k^3 triples).     */
/* ------------------------------------------------------------------------ */

int oracle_coselect_pair(const int32_t *idx_prev, const int32_t *idx_l, const int32_t *idx_next,
                         int64_t T_fit, int E, int k, uint32_t *C2)
{
    if (T_fit < 0 || E < 1 || k < 1) return 1;
    memset(C2, 0, sizeof(uint32_t) * (size_t)E * E * E);
    for (int64_t t = 0; t < T_fit; ++t)
        for (int i = 0; i < k; ++i)
            for (int j = 0; j < k; ++j)
                for (int m = 0; m < k; ++m) {
                    int a = idx_prev[t * k + i], b = idx_l[t * k + j], c = idx_next[t * k + m];
                    if (a < 0 || a >= E || b < 0 || b >= E || c < 0 || c >= E) return 1;
                    C2[((int64_t)a * E + b) * E + c] += 1;
                }
    return 0;
}

/* preference list, confidence numerator and denominator of one count row,
 * by the same rules as the single-expert form above */
static void row_prediction(const uint32_t *row, int E, const int32_t *p_next, int R,
                           uint64_t *sigma, int32_t *pl, uint64_t *num, uint64_t *den)
{
    uint64_t total = 0;
    int best = 0;
    for (int e = 0; e < E; ++e) {
        total += row[e];
        if (row[e] > row[best]) best = e;
    }
    *num = row[best];
    *den = total;
    for (int d = 0; d < R; ++d) sigma[d] = 0;
    for (int e = 0; e < E; ++e) sigma[p_next[e]] += row[e];
    pl[0] = p_next[best];
    int n = 1;
    while (n < R) {
        int pick = -1;
        for (int d = 0; d < R; ++d) {
            int used = 0;
            for (int i = 0; i < n; ++i)
                if (pl[i] == d) used = 1;
            if (used) continue;
            if (pick < 0 || sigma[d] > sigma[pick]) pick = d;
        }
        pl[n++] = pick;
    }
}

/*
 * As oracle_token_shuffle, with the prediction row of token t chosen as:
 *   a = idx_prev[t*k] (top-1 at l-1), b = idx_l[t*k] (top-1 at l);
 *   the pair row C2[a][b] if its total is at least min_obs,
 *   else the single-expert row C[b].
 * Preference order, confidence, visit order and capacity rule are those of
 * the single-expert form, applied to the chosen row.  use_pair[t] = 1 when
 * the pair row was used.
 */
int oracle_token_shuffle_pair(const int32_t *idx_prev, const int32_t *idx_l, const uint32_t *C,
                              const uint32_t *C2, const int32_t *p_next, int64_t T, int E, int k,
                              int R, uint64_t min_obs, int32_t *pred_rank, int32_t *perm,
                              int32_t *inv, int32_t *use_pair)
{
    if (T < 0 || E < 1 || k < 1 || R < 1 || T % R != 0 || min_obs < 1) return 1;
    const int64_t Tr = T / R;
    int32_t *pref = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * R);
    uint64_t *sigma = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)R);
    conf_t *order = (conf_t *)malloc(sizeof(conf_t) * (size_t)(T > 0 ? T : 1));
    int64_t *load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    int rc = 0;
    if (!pref || !sigma || !order || !load) { rc = 2; goto done; }

    for (int64_t t = 0; t < T; ++t) {
        int a = idx_prev[t * k], b = idx_l[t * k];
        if (a < 0 || a >= E || b < 0 || b >= E) { rc = 1; goto done; }
        const uint32_t *prow = C2 + ((int64_t)a * E + b) * E;
        uint64_t psum = 0;
        for (int e = 0; e < E; ++e) psum += prow[e];
        use_pair[t] = psum >= min_obs;
        const uint32_t *row = use_pair[t] ? prow : C + (int64_t)b * E;
        row_prediction(row, E, p_next, R, sigma, pref + t * R, &order[t].num, &order[t].den);
        order[t].t = t;
    }
    /* the per-token denominators, kept by token before the sort reorders */
    uint64_t *den_t = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)(T > 0 ? T : 1));
    if (!den_t) { rc = 2; goto done; }
    for (int64_t t = 0; t < T; ++t) den_t[t] = order[t].den;
    qsort(order, (size_t)T, sizeof(conf_t), cmp_conf);

    for (int64_t i = 0; i < T; ++i) {
        int64_t t = order[i].t;
        int chosen = -1;
        if (den_t[t] == 0) {
            int s = (int)(t / Tr);
            if (load[s] < Tr) chosen = s;
            for (int d = 0; chosen < 0 && d < R; ++d)
                if (load[d] < Tr) chosen = d;
        } else {
            const int32_t *pl = pref + t * R;
            for (int n = 0; chosen < 0 && n < R; ++n)
                if (load[pl[n]] < Tr) chosen = pl[n];
        }
        pred_rank[t] = chosen;
        load[chosen] += 1;
    }
    free(den_t);

    for (int d = 0; d < R; ++d) load[d] = 0;
    for (int64_t t = 0; t < T; ++t) {
        int d = pred_rank[t];
        int64_t pos = (int64_t)d * Tr + load[d];
        load[d] += 1;
        perm[t] = (int32_t)pos;
        inv[pos] = (int32_t)t;
    }
done:
    free(pref); free(sigma); free(order); free(load);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Routing statistics.                                                       */
/* [EC] Offline Placement and Prediction Statistics, Table I: "Same GPU" =   */
/* share of tokens whose k experts all sit on one rank, "GPUs" = distinct    */
/* ranks per token, "Dedup" = rows removed by deduplication = 1 - GPUs / k.  */
/* hist[D] = number of tokens with exactly D distinct destination ranks.     */
/* ------------------------------------------------------------------------ */

int oracle_rank_stats(const int32_t *idx, int64_t T, int E, int k, int R, const int32_t *p,
                      int64_t *hist)
{
    if (T < 0 || E < 1 || k < 1 || R < 1) return 1;
    for (int d = 0; d <= k; ++d) hist[d] = 0;
    for (int64_t t = 0; t < T; ++t) {
        int distinct = 0;
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            if (e < 0 || e >= E || p[e] < 0 || p[e] >= R) return 1;
            int seen = 0;
            for (int i = 0; i < j; ++i)
                if (p[idx[t * k + i]] == p[e]) seen = 1;
            if (!seen) ++distinct;
        }
        hist[distinct] += 1;
    }
    return 0;
}

/* [EC] Cross-layer correlation: a layer-l expert "sends" a share of its      */
/* tokens to one layer-l+1 expert.  With C (all k x k cross-layer pairs) and */
/* W (diagonal = tokens selecting e) fitted on the same tokens, the share of */
/* e's tokens that select e' next is C[e][e'] / W[e][e]; num[e] is the       */
/* largest C[e][e'] and den[e] = W[e][e].                                    */
int oracle_successor_share(const uint32_t *C, const uint32_t *W, int E, uint32_t *num,
                           uint32_t *den)
{
    if (E < 1) return 1;
    for (int e = 0; e < E; ++e) {
        uint32_t m = 0;
        for (int e2 = 0; e2 < E; ++e2)
            if (C[(int64_t)e * E + e2] > m) m = C[(int64_t)e * E + e2];
        num[e] = m;
        den[e] = W[(int64_t)e * E + e];
    }
    return 0;
}

/* [EC] Correlation Formation and Stability: Pearson correlation between a    */
/* fitted and a held-out count table.  The five sums are exact integers      */
/* (128-bit); sums[0..4] = (sx, sy, sxx, syy, sxy), each as (low, high)      */
/* 64-bit words.                                                             */
int oracle_count_sums(const uint32_t *x, const uint32_t *y, int64_t n, uint64_t *sums)
{
    if (n < 0) return 1;
    unsigned __int128 s[5] = {0, 0, 0, 0, 0};
    for (int64_t i = 0; i < n; ++i) {
        unsigned __int128 a = x[i], b = y[i];
        s[0] += a;
        s[1] += b;
        s[2] += a * a;
        s[3] += b * b;
        s[4] += a * b;
    }
    for (int i = 0; i < 5; ++i) {
        sums[2 * i] = (uint64_t)s[i];
        sums[2 * i + 1] = (uint64_t)(s[i] >> 64);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Kernighan-Lin passes and two-level placement.                             */
/* [EC] Correlated Placement: a Kernighan-Lin-style local search (Algorithm  */
/* 1, not printed) swaps experts between GPUs; for multi-node groups the     */
/* partition is made across nodes first, then across the GPUs of each node.  */
/* A KL pass, as in Kernighan and Lin's graph bisection: repeatedly take the */
/* best swap among experts not yet moved in this pass (gain may be           */
/* negative; ties to the lowest (a, b)), move and lock both, until no        */
/* unlocked pair on different ranks is left or E/2 swaps were made; then     */
/* keep the shortest prefix of moves with the largest total gain and undo    */
/* the rest.  Passes repeat while that total is positive (at most E passes). */
/* ------------------------------------------------------------------------ */

static void compute_A(const uint32_t *W, int E, int R, const int32_t *p, long long *A)
{
    for (int64_t i = 0; i < (int64_t)E * R; ++i) A[i] = 0;
    for (int e = 0; e < E; ++e)
        for (int e2 = 0; e2 < E; ++e2)
            if (e2 != e) A[(int64_t)e * R + p[e2]] += W[(int64_t)e * E + e2];
}

static long long kl_pass(const uint32_t *W, int E, int R, int32_t *p, long long *A, char *locked,
                         int *sa, int *sb, long long *sg)
{
    memset(locked, 0, (size_t)E);
    int n = 0;
    for (int step = 0; step < E / 2; ++step) {
        compute_A(W, E, R, p, A);
        int ba = -1, bb = -1;
        long long best = 0;
        for (int a = 0; a < E; ++a) {
            if (locked[a]) continue;
            for (int b = a + 1; b < E; ++b) {
                if (locked[b] || p[a] == p[b]) continue;
                int P = p[a], Q = p[b];
                long long g = A[(int64_t)a * R + Q] - A[(int64_t)a * R + P] +
                              A[(int64_t)b * R + P] - A[(int64_t)b * R + Q] -
                              2LL * (long long)W[(int64_t)a * E + b];
                if (ba < 0 || g > best) { best = g; ba = a; bb = b; }
            }
        }
        if (ba < 0) break;
        int P = p[ba];
        p[ba] = p[bb];
        p[bb] = P;
        locked[ba] = locked[bb] = 1;
        sa[n] = ba;
        sb[n] = bb;
        sg[n] = best;
        ++n;
    }
    long long run = 0, keep = 0;
    int m = 0;
    for (int i = 0; i < n; ++i) {
        run += sg[i];
        if (run > keep) { keep = run; m = i + 1; }
    }
    for (int i = n - 1; i >= m; --i) {
        int P = p[sa[i]];
        p[sa[i]] = p[sb[i]];
        p[sb[i]] = P;
    }
    return keep;
}

/* refine_mode: 0 none, 1 best single swaps (as oracle_place_correlated),
 * 2 KL passes.  Single level. */
static int place_one_level(const uint32_t *W, int E, int R, int seed_mode, int refine_mode,
                           int32_t *p)
{
    int rc = oracle_place_correlated(W, E, R, seed_mode, refine_mode == 1, p);
    if (rc || refine_mode != 2) return rc;
    long long *A = (long long *)malloc(sizeof(long long) * (size_t)E * R);
    char *locked = (char *)malloc((size_t)E);
    int *sa = (int *)malloc(sizeof(int) * (size_t)(E / 2 + 1));
    int *sb = (int *)malloc(sizeof(int) * (size_t)(E / 2 + 1));
    long long *sg = (long long *)malloc(sizeof(long long) * (size_t)(E / 2 + 1));
    if (!A || !locked || !sa || !sb || !sg) rc = 2;
    for (int pass = 0; !rc && pass < E; ++pass)
        if (kl_pass(W, E, R, p, A, locked, sa, sb, sg) <= 0) break;
    free(A); free(locked); free(sa); free(sb); free(sg);
    return rc;
}

/*
 * Two-level placement over `nodes` nodes of R/nodes ranks each (nodes = 1:
 * one level).  Level 1 places the experts on nodes (E/nodes each) with the
 * seed and refinement given; level 2 places each node's experts, taken in
 * ascending id, on its R/nodes ranks with W restricted to them.  p[e] =
 * node * (R/nodes) + rank within the node.
 */
int oracle_place_two_level(const uint32_t *W, int E, int R, int nodes, int seed_mode,
                           int refine_mode, int32_t *p)
{
    if (E < 1 || R < 1 || nodes < 1 || R % nodes != 0 || E % R != 0) return 1;
    if (refine_mode < 0 || refine_mode > 2) return 1;
    if (nodes == 1) return place_one_level(W, E, R, seed_mode, refine_mode, p);
    const int G = R / nodes, En = E / nodes;
    int32_t *pn = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int *mem = (int *)malloc(sizeof(int) * (size_t)En);
    uint32_t *sub = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)En * En);
    int32_t *pg = (int32_t *)malloc(sizeof(int32_t) * (size_t)En);
    int rc = (!pn || !mem || !sub || !pg) ? 2 : 0;
    if (!rc) rc = place_one_level(W, E, nodes, seed_mode, refine_mode, pn);
    for (int n = 0; !rc && n < nodes; ++n) {
        int c = 0;
        for (int e = 0; e < E; ++e)
            if (pn[e] == n) mem[c++] = e;
        for (int i = 0; i < En; ++i)
            for (int j = 0; j < En; ++j) sub[(int64_t)i * En + j] = W[(int64_t)mem[i] * E + mem[j]];
        rc = place_one_level(sub, En, G, seed_mode, refine_mode, pg);
        for (int i = 0; !rc && i < En; ++i) p[mem[i]] = n * G + pg[i];
    }
    free(pn); free(mem); free(sub); free(pg);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Rounds-based capacity assignment (a parallel alternative to the          */
/* sequential visit of [EC] Method 2, Capacity Constraint).  Priorities and */
/* preference lists are those of oracle_token_shuffle.  In each round every  */
/* unassigned token proposes to the first rank of its list that was not     */
/* full when the round began; each rank accepts its highest-priority         */
/* proposers up to its remaining capacity and the others stay unassigned.   */
/* Rounds repeat until every token is assigned: a round either accepts all  */
/* its proposers or fills at least one rank, so there are at most R + 1.    */
/* rounds_out = the number of rounds that accepted at least one token.      */
/* ------------------------------------------------------------------------ */

int oracle_token_shuffle_rounds(const int32_t *idx_l, const uint32_t *C, const int32_t *p_next,
                                int64_t T, int E, int k, int R, int32_t *pred_rank,
                                int32_t *perm, int32_t *inv, int32_t *rounds_out)
{
    if (T < 0 || E < 1 || k < 1 || R < 1 || T % R != 0) return 1;
    const int64_t Tr = T / R;
    int32_t *pref = (int32_t *)malloc(sizeof(int32_t) * (size_t)E * R);
    uint64_t *num = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)E);
    uint64_t *den = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)E);
    uint64_t *sigma = (uint64_t *)malloc(sizeof(uint64_t) * (size_t)R);
    conf_t *order = (conf_t *)malloc(sizeof(conf_t) * (size_t)(T > 0 ? T : 1));
    int64_t *load = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    int64_t *taken = (int64_t *)calloc((size_t)R, sizeof(int64_t));
    char *full = (char *)calloc((size_t)R, 1);
    int rc = 0, rounds = 0;
    if (!pref || !num || !den || !sigma || !order || !load || !taken || !full) { rc = 2; goto done; }

    for (int e1 = 0; e1 < E; ++e1)
        row_prediction(C + (int64_t)e1 * E, E, p_next, R, sigma, pref + (int64_t)e1 * R, &num[e1],
                       &den[e1]);
    for (int64_t t = 0; t < T; ++t) {
        int e1 = idx_l[t * k];
        if (e1 < 0 || e1 >= E) { rc = 1; goto done; }
        order[t].num = num[e1];
        order[t].den = den[e1];
        order[t].t = t;
        pred_rank[t] = -1;
    }
    qsort(order, (size_t)T, sizeof(conf_t), cmp_conf);

    for (int round = 0; round <= R; ++round) {
        int64_t accepted = 0, left = 0;
        for (int d = 0; d < R; ++d) {
            taken[d] = 0;
            full[d] = load[d] >= Tr;
        }
        /* visiting proposers in priority order, rank d accepts while it has
         * room left from the start of the round */
        for (int64_t i = 0; i < T; ++i) {
            int64_t t = order[i].t;
            if (pred_rank[t] >= 0) continue;
            int e1 = idx_l[t * k], d = -1;
            if (den[e1] == 0) {
                int s = (int)(t / Tr);
                if (!full[s]) d = s;
                for (int q = 0; d < 0 && q < R; ++q)
                    if (!full[q]) d = q;
            } else {
                const int32_t *pl = pref + (int64_t)e1 * R;
                for (int n = 0; d < 0 && n < R; ++n)
                    if (!full[pl[n]]) d = pl[n];
            }
            if (d < 0) { rc = 1; goto done; }
            if (load[d] + taken[d] < Tr) {
                pred_rank[t] = d;
                taken[d] += 1;
                ++accepted;
            } else {
                ++left;
            }
        }
        for (int d = 0; d < R; ++d) load[d] += taken[d];
        if (accepted) ++rounds;
        if (!left) break;
    }
    *rounds_out = rounds;

    for (int d = 0; d < R; ++d) load[d] = 0;
    for (int64_t t = 0; t < T; ++t) {
        int d = pred_rank[t];
        if (d < 0) { rc = 1; goto done; }
        int64_t pos = (int64_t)d * Tr + load[d];
        load[d] += 1;
        perm[t] = (int32_t)pos;
        inv[pos] = (int32_t)t;
    }
done:
    free(pref); free(num); free(den); free(sigma); free(order); free(load); free(taken); free(full);
    return rc;
}
