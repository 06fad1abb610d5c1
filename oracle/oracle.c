/*
 * CPU oracle for the MoE router-and-dispatch path.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the slow, plain, fp64 restatement of what the path computes.
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
 * arm may load it.  It shares no code, header, table or constant with the CUDA
 * library in token_dispatch_moe_b200/csrc, and the library never calls it.
 *
 * Every quantity is computed in double precision from inputs widened exactly
 * (bf16 -> double and fp32 -> double are exact).  Nothing is blocked, fused or
 * reordered beyond the plain definition of each step; loops run in the obvious
 * index order so that a reader can check them against the pages by eye.
 *
 * Sources (page title, then the section on it):
 *   [DS]  "DeepSeek-V3.2-Exp - Select experts": the "Explanation" prose and
 *         the gate-forward code excerpt (linear in fp32, softmax or sigmoid,
 *         selection-only bias, group score = amax or sum of the top two biased
 *         scores, keep topk_groups groups, top-k, gather the unbiased scores,
 *         renormalise for sigmoid, multiply by route_scale).
 *   [FX]  "Crate ferrox_moe" (docs.rs), section "Functions": route_top_k_softmax
 *         (softmax over every expert, then top-k, norm_topk_prob flag),
 *         route_top_k_softmax_weight (gpt-oss: top-k on raw logits, then softmax
 *         over those k), route_top_k_sigmoid(_with_bias),
 *         route_top_k_sqrtsoftplus(_with_bias) (score sqrt(softplus(logit)),
 *         bias on selection only, renormalise, scaling factor), route_hash
 *         (token-id -> expert-id table lookup), combine_expert_outputs
 *         (routed + shared).
 *   [DK]  "Feature Request: dynamic number of experts (hyperparam per request)":
 *         k is a per-request value picked from the full ranking, no other change.
 *
 * Readings where the pages are silent:
 *   - equal keys: the lower expert id ranks first; equal group scores: the
 *     lower group id ranks first;
 *   - NaN keys rank below every number (including -inf); the status reports it;
 *   - softplus is the exact form max(l,0) + log1p(exp(-|l|)), no threshold;
 *   - renormalisation is an explicit flag; route_scale always multiplies;
 *   - hash-routed weights: if logits are given, the layer's score of the looked
 *     up expert, then the renormalise flag and route_scale; otherwise
 *     route_scale / k per slot;
 *   - combine adds the shared expert at unit weight after the routed sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_INDEX 4
#define ORACLE_ERR_NAN 6

#define ORACLE_SOFTMAX 0
#define ORACLE_SIGMOID 1
#define ORACLE_SQRT_SOFTPLUS 2
#define ORACLE_TOPK_SOFTMAX 3

/* bf16 is the top half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ---------------------------------------------------------------- gate ---- */
/* [DS] gate linear: logits[t][e] = sum_i x[t][i] * W[e][i], summed in
 * ascending i, for the listed rows only (so large inputs can be sampled). */
void oracle_gate_rows(const uint16_t *x, const uint16_t *w, int32_t d, int32_t E,
                      const int64_t *rows, int64_t nrows, double *out) {
    for (int64_t r = 0; r < nrows; ++r) {
        const uint16_t *xr = x + rows[r] * (int64_t)d;
        for (int32_t e = 0; e < E; ++e) {
            const uint16_t *we = w + (int64_t)e * d;
            double acc = 0.0;
            for (int32_t i = 0; i < d; ++i)
                acc += oracle_bf16_to_double(xr[i]) * oracle_bf16_to_double(we[i]);
            out[r * E + e] = acc;
        }
    }
}

/* --------------------------------------------------------------- score ---- */
static double softplus(double l) { return fmax(l, 0.0) + log1p(exp(-fabs(l))); }

/* Unbiased per-expert scores of one row ([DS] softmax / sigmoid, [FX]
 * sqrt-softplus; for the gpt-oss rule the selection score is the raw logit). */
static void row_scores(const float *l, int32_t E, int32_t score, double *s) {
    if (score == ORACLE_SOFTMAX) {
        double m = -INFINITY;
        for (int32_t e = 0; e < E; ++e)
            if ((double)l[e] > m) m = (double)l[e];
        double z = 0.0;
        for (int32_t e = 0; e < E; ++e) z += exp((double)l[e] - m);
        for (int32_t e = 0; e < E; ++e) s[e] = exp((double)l[e] - m) / z;
    } else if (score == ORACLE_SIGMOID) {
        for (int32_t e = 0; e < E; ++e) s[e] = 1.0 / (1.0 + exp(-(double)l[e]));
    } else if (score == ORACLE_SQRT_SOFTPLUS) {
        for (int32_t e = 0; e < E; ++e) s[e] = sqrt(softplus((double)l[e]));
    } else {
        for (int32_t e = 0; e < E; ++e) s[e] = (double)l[e];
    }
}

void oracle_scores(const float *logits, int64_t T, int32_t E, int32_t score, double *out) {
    for (int64_t t = 0; t < T; ++t) row_scores(logits + t * E, E, score, out + t * E);
}

/* ------------------------------------------------------------- ranking ---- */
typedef struct {
    double key;
    int32_t id;
} ranked;

/* Descending key, then ascending id; NaN below every number. */
static int by_key_desc(const void *pa, const void *pb) {
    const ranked *a = (const ranked *)pa, *b = (const ranked *)pb;
    int an = isnan(a->key), bn = isnan(b->key);
    if (an != bn) return an ? 1 : -1;
    if (!an) {
        if (a->key > b->key) return -1;
        if (a->key < b->key) return 1;
    }
    return (a->id > b->id) - (a->id < b->id);
}

/* Weights for a given selection ([DS] gather the unbiased scores, divide by
 * their sum, multiply by route_scale; [FX] gpt-oss: softmax over the selected
 * logits).  ids[j] < 0 marks an empty slot; its weight is 0 and it takes no
 * part in the sums. */
static void row_weights(const float *l, const double *s, const int32_t *ids, int32_t k_max,
                        int32_t score, int32_t renormalize, double route_scale, double *w) {
    for (int32_t j = 0; j < k_max; ++j) w[j] = 0.0;
    if (score == ORACLE_TOPK_SOFTMAX) {
        double m = -INFINITY;
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0 && (double)l[ids[j]] > m) m = (double)l[ids[j]];
        double z = 0.0;
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0) z += exp((double)l[ids[j]] - m);
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0) w[j] = exp((double)l[ids[j]] - m) / z;
    } else {
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0) w[j] = s[ids[j]];
    }
    if (renormalize) {
        double sum = 0.0;
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0) sum += w[j];
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[j] >= 0) w[j] /= sum;
    }
    for (int32_t j = 0; j < k_max; ++j)
        if (ids[j] >= 0) w[j] *= route_scale;
}

/* --------------------------------------------------------------- route ---- */
/* One pass per token row, in the order of [DS]:
 *   1. scores from the logits (row_scores);
 *   2. selection key = score + bias (bias optional; weights keep the score);
 *   3. if n_groups > 1: group score = sum of the group_topn largest keys of
 *      each contiguous group of E/n_groups experts (group_topn = 1 is amax);
 *      keep the topk_groups best groups, drop the others from selection;
 *   4. the k_t largest remaining keys, in descending key order ([DK]: k_t is
 *      the token's own k, or k_max when no per-token k is given);
 *   5. weights from the unbiased scores (row_weights).
 * Outputs: ids [T][k_max] (-1 padded), w [T][k_max] (0 padded); optionally the
 * per-expert selection keys [T][E] (-inf for experts of dropped groups) and the
 * relative gap between the last kept and the first dropped group score [T]
 * (+inf when no group is dropped).  Returns ORACLE_ERR_NAN if a NaN key was
 * seen (rows are still routed), ORACLE_ERR_ARG on a bad argument. */
int oracle_route(const float *logits, const float *bias, const int32_t *k_per_token, int64_t T,
                 int32_t E, int32_t k_max, int32_t score, int32_t n_groups, int32_t topk_groups,
                 int32_t group_topn, int32_t renormalize, double route_scale, int32_t *ids,
                 double *w, double *keys_out, double *group_gap) {
    if (E <= 0 || k_max < 0 || k_max > E || n_groups < 1 || E % n_groups != 0) return ORACLE_ERR_ARG;
    if (n_groups > 1 && (topk_groups < 1 || topk_groups > n_groups || group_topn < 1 ||
                         group_topn > E / n_groups || k_max > topk_groups * (E / n_groups)))
        return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    double *s = (double *)malloc(sizeof(double) * E);
    double *key = (double *)malloc(sizeof(double) * E);
    ranked *cand = (ranked *)malloc(sizeof(ranked) * E);
    ranked *grp = (ranked *)malloc(sizeof(ranked) * (n_groups > 0 ? n_groups : 1));
    char *kept = (char *)malloc((size_t)n_groups);
    const int32_t gsz = E / n_groups;

    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        int32_t kt = k_per_token ? k_per_token[t] : k_max;
        if (kt < 0 || kt > k_max) {
            free(s), free(key), free(cand), free(grp), free(kept);
            return ORACLE_ERR_ARG;
        }
        row_scores(l, E, score, s);
        for (int32_t e = 0; e < E; ++e) {
            key[e] = s[e] + (bias ? (double)bias[e] : 0.0);
            if (isnan(key[e])) status = ORACLE_ERR_NAN;
        }

        for (int32_t g = 0; g < n_groups; ++g) kept[g] = 1;
        if (group_gap) group_gap[t] = INFINITY;
        if (n_groups > 1) {
            for (int32_t g = 0; g < n_groups; ++g) {
                for (int32_t i = 0; i < gsz; ++i) {
                    cand[i].key = key[g * gsz + i];
                    cand[i].id = g * gsz + i;
                }
                qsort(cand, (size_t)gsz, sizeof(ranked), by_key_desc);
                double gs = 0.0;
                for (int32_t i = 0; i < group_topn; ++i) gs += cand[i].key;
                grp[g].key = gs;
                grp[g].id = g;
            }
            qsort(grp, (size_t)n_groups, sizeof(ranked), by_key_desc);
            for (int32_t g = 0; g < n_groups; ++g) kept[g] = 0;
            for (int32_t i = 0; i < topk_groups; ++i) kept[grp[i].id] = 1;
            if (group_gap && topk_groups < n_groups) {
                double a = grp[topk_groups - 1].key, b = grp[topk_groups].key;
                double den = fabs(a) > 1e-300 ? fabs(a) : 1e-300;
                group_gap[t] = (isnan(a) || isnan(b)) ? 0.0 : (a - b) / den;
            }
        }

        int32_t nc = 0;
        for (int32_t e = 0; e < E; ++e) {
            if (!kept[e / gsz]) continue;
            cand[nc].key = key[e];
            cand[nc].id = e;
            ++nc;
        }
        qsort(cand, (size_t)nc, sizeof(ranked), by_key_desc);

        int32_t *row_ids = ids + t * k_max;
        for (int32_t j = 0; j < k_max; ++j) row_ids[j] = (j < kt && j < nc) ? cand[j].id : -1;
        row_weights(l, s, row_ids, k_max, score, renormalize, route_scale, w + t * k_max);

        if (keys_out)
            for (int32_t e = 0; e < E; ++e) keys_out[t * E + e] = kept[e / gsz] ? key[e] : -INFINITY;
    }
    free(s), free(key), free(cand), free(grp), free(kept);
    return status;
}

/* Weights for a selection made elsewhere (used to check the weights of rows
 * where a near-tie let the device pick a different but equally valid set). */
int oracle_weights_for_ids(const float *logits, const int32_t *ids, int64_t T, int32_t E,
                           int32_t k_max, int32_t score, int32_t renormalize, double route_scale,
                           double *w) {
    double *s = (double *)malloc(sizeof(double) * E);
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < k_max; ++j)
            if (ids[t * k_max + j] >= E) {
                free(s);
                return ORACLE_ERR_INDEX;
            }
        row_scores(logits + t * E, E, score, s);
        row_weights(logits + t * E, s, ids + t * k_max, k_max, score, renormalize, route_scale,
                    w + t * k_max);
    }
    free(s);
    return ORACLE_OK;
}

/* ------------------------------------------------------- grouped route ---- */
/* [FX] route_top_k_grouped: cut the E experts into n_groups contiguous groups,
 * keep the k_per_group best of each group (by the same score as the flat
 * router), then keep the total_k best of those candidates across groups.
 * Readings: no bias (the page gives none for this rule); candidates and the
 * final choice both rank by (score desc, id asc), the output in that order;
 * total_k = k_max, the output width, and k_max <= n_groups * k_per_group;
 * weights as the flat router (row_weights).  keys_out (optional) receives the
 * candidates' scores and -inf for experts their group did not keep. */
int oracle_route_grouped(const float *logits, int64_t T, int32_t E, int32_t k_max,
                         int32_t score, int32_t n_groups, int32_t k_per_group,
                         int32_t renormalize, double route_scale, int32_t *ids, double *w,
                         double *keys_out) {
    if (E <= 0 || n_groups < 1 || E % n_groups != 0 || k_per_group < 1 ||
        k_per_group > E / n_groups || k_max < 0 || k_max > n_groups * k_per_group)
        return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    const int32_t gsz = E / n_groups;
    double *s = (double *)malloc(sizeof(double) * E);
    ranked *grp = (ranked *)malloc(sizeof(ranked) * gsz);
    ranked *cand = (ranked *)malloc(sizeof(ranked) * E);
    for (int64_t t = 0; t < T; ++t) {
        const float *l = logits + t * E;
        row_scores(l, E, score, s);
        int32_t nc = 0;
        if (keys_out)
            for (int32_t e = 0; e < E; ++e) keys_out[t * E + e] = -INFINITY;
        for (int32_t g = 0; g < n_groups; ++g) {
            for (int32_t i = 0; i < gsz; ++i) {
                grp[i].key = s[g * gsz + i];
                grp[i].id = g * gsz + i;
                if (isnan(grp[i].key)) status = ORACLE_ERR_NAN;
            }
            qsort(grp, (size_t)gsz, sizeof(ranked), by_key_desc);
            for (int32_t i = 0; i < k_per_group; ++i) {
                cand[nc++] = grp[i];
                if (keys_out) keys_out[t * E + grp[i].id] = grp[i].key;
            }
        }
        qsort(cand, (size_t)nc, sizeof(ranked), by_key_desc);
        int32_t *sel = ids + t * k_max;
        for (int32_t j = 0; j < k_max; ++j) sel[j] = cand[j].id;
        row_weights(l, s, sel, k_max, score, renormalize, route_scale, w + t * k_max);
    }
    free(s), free(grp), free(cand);
    return status;
}

/* ---------------------------------------------------------- hash route ---- */
/* [FX] route_hash: the expert ids of token t are row tok[t] of the table
 * (row-major [vocab][k], one row of k ids per token id; a repeated id in a row
 * keeps both slots).  Weights: the reading stated in the header.  A token id
 * outside [0, vocab) empties its whole row; a table entry outside [0, E)
 * empties its slot; both return ORACLE_ERR_INDEX. */
int oracle_hash_route(const int32_t *tok, const int32_t *table, int32_t vocab, int32_t k,
                      const float *logits, int64_t T, int32_t E, int32_t score,
                      int32_t renormalize, double route_scale, int32_t *ids, double *w) {
    int status = ORACLE_OK;
    double *s = (double *)malloc(sizeof(double) * E);
    for (int64_t t = 0; t < T; ++t) {
        int32_t *ri = ids + t * k;
        double *rw = w + t * k;
        int32_t v = tok[t];
        for (int32_t j = 0; j < k; ++j) {
            ri[j] = -1;
            rw[j] = 0.0;
        }
        if (v < 0 || v >= vocab) {
            status = ORACLE_ERR_INDEX;
            continue;
        }
        for (int32_t j = 0; j < k; ++j) {
            int32_t e = table[(int64_t)v * k + j];
            if (e < 0 || e >= E) {
                status = ORACLE_ERR_INDEX;
                continue;
            }
            ri[j] = e;
        }
        if (logits) {
            row_scores(logits + t * E, E, score, s);
            row_weights(logits + t * E, s, ri, k, score, renormalize, route_scale, rw);
        } else {
            for (int32_t j = 0; j < k; ++j)
                if (ri[j] >= 0) rw[j] = route_scale / (double)k;
        }
    }
    free(s);
    return status;
}

/* ------------------------------------------------------------ dispatch ---- */
/* Expert-contiguous layout of the assignments:
 *   counts[e]  = number of slots (t, j) whose id is e;
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e] (offsets[E] = N);
 *   walking the slots in flat order a = t*k_max + j (empty slots, id -1,
 *   skipped), the slot gets pos = offsets[e] + (number of earlier slots with
 *   the same e); sorted_token[pos] = t and dest_pos[a] = pos (-1 if empty).
 * An id outside [-1, E) is treated as empty and returns ORACLE_ERR_INDEX. */
int oracle_dispatch(const int32_t *ids, int64_t T, int32_t k_max, int32_t E, int32_t *counts,
                    int32_t *offsets, int32_t *sorted_token, int32_t *dest_pos) {
    int status = ORACLE_OK;
    int64_t n = T * (int64_t)k_max;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < n; ++a) {
        int32_t e = ids[a];
        if (e >= 0 && e < E)
            counts[e] += 1;
        else if (e != -1)
            status = ORACLE_ERR_INDEX;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *seen = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int64_t a = 0; a < n; ++a) {
        int32_t e = ids[a];
        if (e >= 0 && e < E) {
            int32_t pos = offsets[e] + seen[e];
            seen[e] += 1;
            sorted_token[pos] = (int32_t)(a / k_max);
            dest_pos[a] = pos;
        } else {
            dest_pos[a] = -1;
        }
    }
    free(seen);
    return status;
}

/* ------------------------------------------- dispatch with a capacity ---- */
/* Top-1 with a per-expert capacity in the Switch style (the open-MoE router
 * survey, its paragraph on the five router levers) and expert blocks padded
 * for a tiled expert GEMM.  Reading: expert e keeps the first `capacity` of its
 * slots in flat order a = t*k_max + j and drops the rest (dest_pos = -1);
 * capacity <= 0 keeps all.  Expert e's block holds kept[e] rows rounded up to
 * a multiple of `pad`; offsets is the exclusive scan of the block sizes; the
 * padding rows of sorted_token hold -1.  counts[e] is the demand before the
 * capacity cut, *dropped the number of slots cut. */
int oracle_dispatch_limited(const int32_t *ids, int64_t T, int32_t k_max, int32_t E,
                            int32_t capacity, int32_t pad, int32_t *counts, int32_t *offsets,
                            int32_t *sorted_token, int32_t *dest_pos, int64_t *dropped) {
    int status = ORACLE_OK;
    int64_t n = T * (int64_t)k_max;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < n; ++a) {
        int32_t e = ids[a];
        if (e >= 0 && e < E)
            counts[e] += 1;
        else if (e != -1)
            status = ORACLE_ERR_INDEX;
    }
    *dropped = 0;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t kept = counts[e];
        if (capacity > 0 && kept > capacity) {
            *dropped += kept - capacity;
            kept = capacity;
        }
        int32_t block = (kept + pad - 1) / pad * pad;
        offsets[e + 1] = offsets[e] + block;
        for (int32_t r = kept; r < block; ++r) sorted_token[offsets[e] + r] = -1;
    }
    int32_t *seen = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    for (int64_t a = 0; a < n; ++a) {
        int32_t e = ids[a];
        dest_pos[a] = -1;
        if (e < 0 || e >= E) continue;
        int32_t rank = seen[e];
        seen[e] += 1;
        if (capacity > 0 && rank >= capacity) continue;
        int32_t pos = offsets[e] + rank;
        sorted_token[pos] = (int32_t)(a / k_max);
        dest_pos[a] = pos;
    }
    free(seen);
    return status;
}

/* --------------------------------------------- expert-parallel exchange ---- */
/* Expert-parallel placement (the open-MoE router survey: in multi-GPU expert
 * parallelism every router choice becomes all-to-all traffic).  G ranks hold T
 * tokens each; expert e lives on rank e / (E/G).  Reading of the receive
 * layout: rank d's buffer holds its experts in ascending order; inside an
 * expert, the rows of source rank 0, then rank 1, ...; inside a source, that
 * rank's slots in flat order a = t*k_max + j.  ids_all is [G][T][k_max];
 * dest_rank / dest_row [G][T][k_max] receive the owner rank and row of every
 * slot (-1 / -1 for empty slots); recv_rows[d] the row count of rank d. */
int oracle_ep_layout(const int32_t *ids_all, int32_t G, int64_t T, int32_t k_max, int32_t E,
                     int32_t *dest_rank, int32_t *dest_row, int64_t *recv_rows) {
    if (G < 1 || E % G != 0) return ORACLE_ERR_ARG;
    int status = ORACLE_OK;
    const int32_t el = E / G;
    const int64_t n = T * (int64_t)k_max;
    for (int64_t i = 0; i < (int64_t)G * n; ++i) {
        dest_rank[i] = -1;
        dest_row[i] = -1;
        if (ids_all[i] < -1 || ids_all[i] >= E) status = ORACLE_ERR_INDEX;
    }
    for (int32_t d = 0; d < G; ++d) recv_rows[d] = 0;
    /* Experts in ascending order visit the owners in order and each owner's
     * experts in order; inside an expert, sources in rank order, then slots. */
    for (int32_t e = 0; e < E; ++e) {
        const int32_t d = e / el;
        for (int32_t r = 0; r < G; ++r)
            for (int64_t a = 0; a < n; ++a)
                if (ids_all[(int64_t)r * n + a] == e) {
                    dest_rank[(int64_t)r * n + a] = d;
                    dest_row[(int64_t)r * n + a] = (int32_t)recv_rows[d];
                    recv_rows[d] += 1;
                }
    }
    return status;
}

/* ------------------------------------------------------- expert FFN ---- */
/* [FX] run_expert / run_expert_oai / swiglu_oai: an expert's FFN is gate and
 * up projections of the hidden row, a gated activation, and a down
 * projection (gpt-oss: a bias on each product, the clamped SwiGLU with
 * alpha = 1.702 and limit 7.0).  The page gives the constants but not the
 * clamped formula; the reading is the published gpt-oss one:
 *   act = 0 (SwiGLU):  g * sigmoid(g) * u
 *   act = 1 (gpt-oss): g' = min(g, 7), u' = clamp(u, -7, 7),
 *                      g' * sigmoid(1.702 g') * (u' + 1)
 * Row r belongs to expert e with offsets[e] <= r < offsets[e+1].  Returns -1
 * for a row outside every block. */
#define ORACLE_OAI_ALPHA 1.702
#define ORACLE_OAI_LIMIT 7.0

static double oracle_act(int32_t act, double g, double u) {
    if (act == 1) {
        double gc = g < ORACLE_OAI_LIMIT ? g : ORACLE_OAI_LIMIT;
        double uc = u < -ORACLE_OAI_LIMIT ? -ORACLE_OAI_LIMIT : (u > ORACLE_OAI_LIMIT ? ORACLE_OAI_LIMIT : u);
        return gc * (1.0 / (1.0 + exp(-ORACLE_OAI_ALPHA * gc))) * (uc + 1.0);
    }
    return g * (1.0 / (1.0 + exp(-g))) * u;
}

static int32_t row_expert(const int32_t *offsets, int32_t E, int64_t r) {
    for (int32_t e = 0; e < E; ++e)
        if (offsets[e] <= r && r < offsets[e + 1]) return e;
    return -1;
}

/* h[i][f] (fp64, before any rounding) for the listed rows of xs; g_out and
 * u_out (optional) receive the two pre-activation products. */
int oracle_expert_gate_up(const uint16_t *xs, const int32_t *offsets, const uint16_t *w1,
                          const uint16_t *w3, const float *b1, const float *b3, int32_t E,
                          int32_t d, int32_t F, int32_t act, const int64_t *rows, int64_t nrows,
                          double *h, double *g_out, double *u_out) {
    for (int64_t i = 0; i < nrows; ++i) {
        const int32_t e = row_expert(offsets, E, rows[i]);
        if (e < 0) return ORACLE_ERR_INDEX;
        const uint16_t *x = xs + rows[i] * (int64_t)d;
        for (int32_t f = 0; f < F; ++f) {
            const uint16_t *r1 = w1 + ((int64_t)e * F + f) * d;
            const uint16_t *r3 = w3 + ((int64_t)e * F + f) * d;
            double g = 0.0, u = 0.0;
            for (int32_t k = 0; k < d; ++k) {
                g += oracle_bf16_to_double(x[k]) * oracle_bf16_to_double(r1[k]);
                u += oracle_bf16_to_double(x[k]) * oracle_bf16_to_double(r3[k]);
            }
            if (b1) g += (double)b1[(int64_t)e * F + f];
            if (b3) u += (double)b3[(int64_t)e * F + f];
            h[i * F + f] = oracle_act(act, g, u);
            if (g_out) g_out[i * F + f] = g;
            if (u_out) u_out[i * F + f] = u;
        }
    }
    return ORACLE_OK;
}

/* y[i][c] = sum_f h[row][f] * W2[e][c][f] + b2[e][c] (fp64) for the listed rows
 * of h (bf16 bits, e.g. the device's h). */
int oracle_expert_down(const uint16_t *h, const int32_t *offsets, const uint16_t *w2,
                       const float *b2, int32_t E, int32_t d, int32_t F, const int64_t *rows,
                       int64_t nrows, double *y) {
    for (int64_t i = 0; i < nrows; ++i) {
        const int32_t e = row_expert(offsets, E, rows[i]);
        if (e < 0) return ORACLE_ERR_INDEX;
        const uint16_t *hr = h + rows[i] * (int64_t)F;
        for (int32_t c = 0; c < d; ++c) {
            const uint16_t *wr = w2 + ((int64_t)e * d + c) * F;
            double acc = 0.0;
            for (int32_t f = 0; f < F; ++f)
                acc += oracle_bf16_to_double(hr[f]) * oracle_bf16_to_double(wr[f]);
            if (b2) acc += (double)b2[(int64_t)e * d + c];
            y[i * d + c] = acc;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------- permute ---- */
/* xs[dest_pos[t][j]] = x[t] for every filled slot: a bit-exact row copy. */
void oracle_permute(const uint16_t *x, const int32_t *dest_pos, int64_t T, int32_t k_max,
                    int32_t d, uint16_t *xs) {
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k_max; ++j) {
            int32_t pos = dest_pos[t * k_max + j];
            if (pos >= 0) memcpy(xs + (int64_t)pos * d, x + t * (int64_t)d, sizeof(uint16_t) * d);
        }
}

/* ------------------------------------------------------------- combine ---- */
/* [FX] combine_expert_outputs: out[t] = sum over filled slots j (in slot
 * order) of w[t][j] * y[dest_pos[t][j]], plus shared[t] at unit weight when a
 * shared expert is given.  Left in fp64 (the comparison is made before the
 * device's rounding to bf16).  mag (optional) receives, per element, the sum
 * of the magnitudes of the terms: the scale of the rounding error any
 * summation order can make. */
void oracle_combine(const uint16_t *y, const float *w, const int32_t *dest_pos,
                    const uint16_t *shared, int64_t T, int32_t k_max, int32_t d, double *out,
                    double *mag) {
    for (int64_t t = 0; t < T; ++t)
        for (int32_t c = 0; c < d; ++c) {
            double acc = 0.0, m = 0.0;
            for (int32_t j = 0; j < k_max; ++j) {
                int32_t pos = dest_pos[t * k_max + j];
                if (pos < 0) continue;
                double term = (double)w[t * k_max + j] * oracle_bf16_to_double(y[(int64_t)pos * d + c]);
                acc += term;
                m += fabs(term);
            }
            if (shared) {
                double sv = oracle_bf16_to_double(shared[t * (int64_t)d + c]);
                acc += sv;
                m += fabs(sv);
            }
            out[t * (int64_t)d + c] = acc;
            if (mag) mag[t * (int64_t)d + c] = m;
        }
}
