/*
 * oracle.c -- plain fp64 CPU oracle for the routed MoE FFN with an
 * expert-parallel band decomposition.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path in expert_decode_b200/.
 *
 * Every quantity is computed in double from the exact input values (a bf16 or
 * fp32 value converts to double without rounding), with straight sequential
 * loops and no blocking, reordering or fused multiply-add.  Sources:
 *
 *  [EP]   fak note "GLM-5.2 multi-GPU: expert-parallel sharding + the
 *         resident-fit benchmark", section "What landed (SHIPPED,
 *         host-proven): expert-parallel MoE FFN sharding" and its gate table.
 *  [XS]   TensorFold issue #214 "GLM-5.3-Flash on CUDA: attention on one GPU,
 *         routed experts on the Sparks (proposal)", Description, "Per MoE
 *         layer" (rows + top-k ids + weights in, partials summed in rank order).
 *  [TP3]  TensorFold issue #310 "GLM-5.3-Flash on CUDA over three ranks
 *         (--tp 3)", the share rule (whole units, the first units % world
 *         ranks take one more) and the maintainer's reply (largest remainder,
 *         equal remainders to the lower rank; one fixed sum order).
 *  [GATE] TensorFold issue #593 "GLM-5.3-Flash and full GLM-5.3 on the native
 *         CUDA engine (tracker)", "The gate" (an FP64 reference per
 *         projection class).
 *
 * Readings where the pages are silent (router nonlinearity, tie-break, fold
 * order, where the shared expert enters): softmax router with renormalised
 * top-k, ties to the lower expert id,
 * picks folded in ascending (expert id, slot), the shared expert added after
 * the routed sum, routed scaling factor 1.  The GLM router variant of the
 * tracker page (a sigmoid score, a bias in the selection, weights from the
 * unbiased scores) is read as in
 * oracle_route_sigmoid below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)   /* bad sizes, null pointers */
#define ORACLE_EPLAN (-2)    /* plan refused: ranks > units, ranks < 1, extent mismatch */
#define ORACLE_EBADID (-3)   /* an expert id outside [0, E) */

/* bf16 is the upper half of an IEEE binary32; widening to double is exact. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double activation_value(const void *x, int x_is_f32, int64_t index)
{
    if (x_is_f32)
        return (double)((const float *)x)[index];
    return bf16_value(((const uint16_t *)x)[index]);
}

/* ------------------------------------------------------------------------ */
/* Plan: contiguous bands in whole units.                                    */
/* ------------------------------------------------------------------------ */

/*
 * ExpertParallelPlan(numExperts, ranks) is a named plan over [0, NumExperts)
 * giving each rank one contiguous band [EP, "What landed"].  Band sizes follow
 * the shard rule of [TP3]: an extent splits in whole units of `unit`, as
 * evenly as it goes, the first (units % ranks) ranks taking one unit more.
 * For experts the unit is 1.  Refused (fail closed, [EP] gate table row
 * "fail-closed"): ranks < 1, ranks > units, extent not a whole number of units.
 *
 * start has ranks + 1 entries; band r is [start[r], start[r+1]).
 */
int oracle_expert_parallel_plan(int64_t extent, int64_t unit, int32_t ranks, int64_t *start)
{
    if (start == NULL || unit < 1 || extent < 1)
        return ORACLE_EINVAL;
    if (extent % unit != 0)
        return ORACLE_EPLAN;
    int64_t units = extent / unit;
    if (ranks < 1 || (int64_t)ranks > units)
        return ORACLE_EPLAN;
    int64_t base = units / ranks;
    int64_t extra = units % ranks;
    start[0] = 0;
    for (int32_t r = 0; r < ranks; ++r) {
        int64_t share = base + (r < extra ? 1 : 0);
        start[r + 1] = start[r] + share * unit;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Router: logits, softmax, top-k, renormalise.                              */
/* ------------------------------------------------------------------------ */

/* Order used for the top-k: larger logit first; equal logits, lower id first. */
static int ranks_before(double la, int32_t ea, double lb, int32_t eb)
{
    if (la != lb)
        return la > lb;
    return ea < eb;
}

/*
 * Every rank runs its own copy of the router on the same rows and so gets the
 * same picks [EP, "What landed"].  For token t:
 *   l_e = sum_h x[t,h] * W_r[e,h] + b_e                (sequential over h)
 *   p   = softmax(l), computed with the largest logit subtracted
 *   S   = the top_k experts by logit, ties to the lower id
 *   w_j = p_{S_j} / sum_{e in S} p_e
 * ids[t, j] and weights[t, j] are written in the order of S (descending logit,
 * equal logits by ascending id).  logits (optional) receives l, [T][E].
 */
int oracle_route(const void *x, int x_is_f32, int64_t T, int64_t H,
                 const uint16_t *w_router, const double *bias, int64_t E, int32_t top_k,
                 int32_t *ids, double *weights, double *logits, int nthreads)
{
    if (T < 0 || H < 1 || E < 1 || top_k < 1 || top_k > E)
        return ORACLE_EINVAL;
    if (T == 0)
        return ORACLE_OK;
    if (x == NULL || w_router == NULL || ids == NULL || weights == NULL)
        return ORACLE_EINVAL;
    int status = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t t = 0; t < T; ++t) {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
        if (l == NULL || p == NULL || order == NULL) {
            free(l); free(p); free(order);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = ORACLE_EINVAL;
            continue;
        }
        /* logits */
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h)
                acc += activation_value(x, x_is_f32, t * H + h) * bf16_value(w_router[e * H + h]);
            if (bias != NULL)
                acc += bias[e];
            l[e] = acc;
        }
        /* softmax with the maximum subtracted */
        double m = l[0];
        for (int64_t e = 1; e < E; ++e)
            if (l[e] > m)
                m = l[e];
        double z = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            p[e] = exp(l[e] - m);
            z += p[e];
        }
        for (int64_t e = 0; e < E; ++e)
            p[e] = p[e] / z;
        /* full order of the experts by (logit desc, id asc): insertion sort */
        for (int64_t e = 0; e < E; ++e) {
            int64_t pos = e;
            while (pos > 0 && ranks_before(l[e], (int32_t)e, l[order[pos - 1]], order[pos - 1])) {
                order[pos] = order[pos - 1];
                --pos;
            }
            order[pos] = (int32_t)e;
        }
        /* renormalise over the picked set */
        double s = 0.0;
        for (int32_t j = 0; j < top_k; ++j)
            s += p[order[j]];
        for (int32_t j = 0; j < top_k; ++j) {
            ids[t * top_k + j] = order[j];
            weights[t * top_k + j] = p[order[j]] / s;
        }
        if (logits != NULL)
            for (int64_t e = 0; e < E; ++e)
                logits[t * E + e] = l[e];
        free(l); free(p); free(order);
    }
    return status;
}

/*
 * The GLM router variant [GATE page, a contributor's comment "What exists
 * now": glm_route.cu, described only as a sigmoid score, a bias in the top-k
 * choice and weights from the unbiased scores].  The page names only these
 * three ingredients; they are read here as:
 *   l_e = sum_h x[t,h] * W_r[e,h]          (sequential over h, no bias)
 *   s_e = 1 / (1 + exp(-l_e))              the expert's score
 *   k_e = s_e + b_e                        the bias moves the selection only
 *   S   = the top_k experts by key, ties to the lower id
 *   w_j = scale * s_{S_j}                  the raw score (normalize = 0), or
 *   w_j = scale * s_{S_j} / sum_{e in S} s_e  (normalize = 1)
 * ids[t, j] and weights[t, j] are written in the order of S (descending key,
 * equal keys by ascending id).  keys and scores (optional) receive k and s,
 * [T][E].
 */
int oracle_route_sigmoid(const void *x, int x_is_f32, int64_t T, int64_t H,
                         const uint16_t *w_router, const double *bias, int64_t E,
                         int32_t top_k, int normalize, double scale, int32_t *ids,
                         double *weights, double *keys, double *scores, int nthreads)
{
    if (T < 0 || H < 1 || E < 1 || top_k < 1 || top_k > E)
        return ORACLE_EINVAL;
    if (T == 0)
        return ORACLE_OK;
    if (x == NULL || w_router == NULL || ids == NULL || weights == NULL)
        return ORACLE_EINVAL;
    int status = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t t = 0; t < T; ++t) {
        double *sc = (double *)malloc(sizeof(double) * (size_t)E);
        double *key = (double *)malloc(sizeof(double) * (size_t)E);
        int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
        if (sc == NULL || key == NULL || order == NULL) {
            free(sc); free(key); free(order);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = ORACLE_EINVAL;
            continue;
        }
        for (int64_t e = 0; e < E; ++e) {
            double l = 0.0;
            for (int64_t h = 0; h < H; ++h)
                l += activation_value(x, x_is_f32, t * H + h) * bf16_value(w_router[e * H + h]);
            sc[e] = 1.0 / (1.0 + exp(-l));
            key[e] = bias != NULL ? sc[e] + bias[e] : sc[e];
        }
        /* full order of the experts by (key desc, id asc): insertion sort */
        for (int64_t e = 0; e < E; ++e) {
            int64_t pos = e;
            while (pos > 0 && ranks_before(key[e], (int32_t)e, key[order[pos - 1]], order[pos - 1])) {
                order[pos] = order[pos - 1];
                --pos;
            }
            order[pos] = (int32_t)e;
        }
        double sum = 0.0;
        for (int32_t j = 0; j < top_k; ++j)
            sum += sc[order[j]];
        for (int32_t j = 0; j < top_k; ++j) {
            ids[t * top_k + j] = order[j];
            weights[t * top_k + j] = normalize ? scale * (sc[order[j]] / sum) : scale * sc[order[j]];
        }
        for (int64_t e = 0; e < E; ++e) {
            if (keys != NULL)
                keys[t * E + e] = key[e];
            if (scores != NULL)
                scores[t * E + e] = sc[e];
        }
        free(sc); free(key); free(order);
    }
    return status;
}

/* ------------------------------------------------------------------------ */
/* One SwiGLU expert.                                                         */
/* ------------------------------------------------------------------------ */

static double silu(double g)
{
    return g / (1.0 + exp(-g));
}

/*
 * expertSwiGLU [EP, "What is not yet" update, item 1]: the expert's FFN
 *   f(x) = W_down (silu(W_gate x) * (W_up x))
 * W_gate, W_up are [I][H] row-major (one row per intermediate unit), W_down is
 * [H][I] row-major (one row per output feature).  a has I entries of scratch.
 */
static void expert_swiglu(const double *xt, const uint16_t *w_gate, const uint16_t *w_up,
                          const uint16_t *w_down, int64_t H, int64_t I, double *a, double *out)
{
    for (int64_t i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int64_t h = 0; h < H; ++h) {
            g += bf16_value(w_gate[i * H + h]) * xt[h];
            u += bf16_value(w_up[i * H + h]) * xt[h];
        }
        a[i] = silu(g) * u;
    }
    for (int64_t r = 0; r < H; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; ++i)
            acc += bf16_value(w_down[r * I + i]) * a[i];
        out[r] = acc;
    }
}

/* Exported single-expert evaluation (used by the pins on tiny cases). */
int oracle_expert_swiglu(const double *xt, const uint16_t *w_gate, const uint16_t *w_up,
                         const uint16_t *w_down, int64_t H, int64_t I, double *out)
{
    if (xt == NULL || w_gate == NULL || w_up == NULL || w_down == NULL || out == NULL || H < 1 || I < 1)
        return ORACLE_EINVAL;
    double *a = (double *)malloc(sizeof(double) * (size_t)I);
    if (a == NULL)
        return ORACLE_EINVAL;
    expert_swiglu(xt, w_gate, w_up, w_down, H, I, a, out);
    free(a);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Routed MoE FFN: monolith and expert-parallel bands.                       */
/* ------------------------------------------------------------------------ */

/* The picks of one token, in the fold order: ascending (expert id, slot j). */
static void pick_order(const int32_t *ids_t, int32_t top_k, int32_t *slot_order)
{
    for (int32_t j = 0; j < top_k; ++j) {
        int32_t pos = j;
        while (pos > 0 && ids_t[slot_order[pos - 1]] > ids_t[j]) {
            slot_order[pos] = slot_order[pos - 1];
            --pos;
        }
        slot_order[pos] = j;
    }
}

static int check_picks(const int32_t *ids, int64_t n, int64_t E,
                       const uint16_t *const *w_gate, const uint16_t *const *w_up,
                       const uint16_t *const *w_down)
{
    for (int64_t q = 0; q < n; ++q) {
        int32_t e = ids[q];
        if (e < 0 || (int64_t)e >= E)
            return ORACLE_EBADID;
        if (w_gate[e] == NULL || w_up[e] == NULL || w_down[e] == NULL)
            return ORACLE_EINVAL;
    }
    return ORACLE_OK;
}

/*
 * Shared work of both forms.  band_start == NULL gives the routed monolith
 * (moeFFN / glmMoeFFN [EP, gate table]):
 *   y = fold over the picks of t in ascending (id, j) of w_j * f_{id_j}(x_t),
 * a sequential left fold that starts from its first term.
 *
 * With bands, each band r contributes the partial of the picks it owns
 * (expertParallelPartials [EP, "What landed"]):
 *   P_r = fold over the picks of t with id in band r, ascending (id, j),
 * starting from its first term; a band that owns none of t's picks contributes
 * nothing.  The partials are then summed in rank order [XS, "Per MoE layer";
 * TP3, "What stays exact"]: y = P_{r0} + P_{r1} + ... over the non-empty bands,
 * a left fold from the lowest rank.
 *
 * In both forms the GLM shared expert (the wrapper of [EP, gate table]) is
 * added last: y = routed + f_shared(x_t), when I_s > 0.
 */
static int moe_ffn(const void *x, int x_is_f32, int64_t T, int64_t H,
                   const int32_t *ids, const double *weights, int32_t top_k,
                   const uint16_t *const *w_gate, const uint16_t *const *w_up,
                   const uint16_t *const *w_down, int64_t E, int64_t I,
                   const uint16_t *ws_gate, const uint16_t *ws_up, const uint16_t *ws_down,
                   int64_t I_s, const int64_t *band_start, int32_t bands, double *y, int nthreads)
{
    if (T < 0 || H < 1 || E < 1 || I < 1 || top_k < 1 || I_s < 0)
        return ORACLE_EINVAL;
    if (T == 0)
        return ORACLE_OK;
    if (x == NULL || ids == NULL || weights == NULL || y == NULL || w_gate == NULL ||
        w_up == NULL || w_down == NULL)
        return ORACLE_EINVAL;
    if (I_s > 0 && (ws_gate == NULL || ws_up == NULL || ws_down == NULL))
        return ORACLE_EINVAL;
    if (band_start != NULL) {
        if (bands < 1 || bands > E || band_start[0] != 0 || band_start[bands] != E)
            return ORACLE_EPLAN;
        for (int32_t r = 0; r < bands; ++r)
            if (band_start[r + 1] < band_start[r])
                return ORACLE_EPLAN;
    }
    int st = check_picks(ids, T * top_k, E, w_gate, w_up, w_down);
    if (st != ORACLE_OK)
        return st;
    int64_t scratch_i = I > I_s ? I : I_s;
    int status = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t t = 0; t < T; ++t) {
        double *xt = (double *)malloc(sizeof(double) * (size_t)H);
        double *a = (double *)malloc(sizeof(double) * (size_t)scratch_i);
        double *f = (double *)malloc(sizeof(double) * (size_t)H);
        double *part = (double *)malloc(sizeof(double) * (size_t)H);
        int32_t *slot = (int32_t *)malloc(sizeof(int32_t) * (size_t)top_k);
        if (xt == NULL || a == NULL || f == NULL || part == NULL || slot == NULL) {
            free(xt); free(a); free(f); free(part); free(slot);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = ORACLE_EINVAL;
            continue;
        }
        const int32_t *ids_t = ids + t * top_k;
        const double *w_t = weights + t * top_k;
        double *yt = y + t * H;
        for (int64_t h = 0; h < H; ++h)
            xt[h] = activation_value(x, x_is_f32, t * H + h);
        pick_order(ids_t, top_k, slot);

        int32_t nbands = band_start != NULL ? bands : 1;
        int have_y = 0;                       /* y holds at least one band partial */
        for (int32_t r = 0; r < nbands; ++r) {
            int64_t lo = band_start != NULL ? band_start[r] : 0;
            int64_t hi = band_start != NULL ? band_start[r + 1] : E;
            int have_part = 0;                /* the band owns at least one pick */
            for (int32_t q = 0; q < top_k; ++q) {
                int32_t j = slot[q];
                int32_t e = ids_t[j];
                if (e < lo || e >= hi)
                    continue;
                expert_swiglu(xt, w_gate[e], w_up[e], w_down[e], H, I, a, f);
                for (int64_t h = 0; h < H; ++h) {
                    double c = w_t[j] * f[h];
                    part[h] = have_part ? part[h] + c : c;
                }
                have_part = 1;
            }
            if (!have_part)
                continue;
            for (int64_t h = 0; h < H; ++h)
                yt[h] = have_y ? yt[h] + part[h] : part[h];
            have_y = 1;
        }
        if (!have_y)
            for (int64_t h = 0; h < H; ++h)
                yt[h] = 0.0;
        if (I_s > 0) {
            expert_swiglu(xt, ws_gate, ws_up, ws_down, H, I_s, a, f);
            for (int64_t h = 0; h < H; ++h)
                yt[h] = yt[h] + f[h];
        }
        free(xt); free(a); free(f); free(part); free(slot);
    }
    return status;
}

int oracle_moe_ffn_monolith(const void *x, int x_is_f32, int64_t T, int64_t H,
                            const int32_t *ids, const double *weights, int32_t top_k,
                            const uint16_t *const *w_gate, const uint16_t *const *w_up,
                            const uint16_t *const *w_down, int64_t E, int64_t I,
                            const uint16_t *ws_gate, const uint16_t *ws_up,
                            const uint16_t *ws_down, int64_t I_s, double *y, int nthreads)
{
    return moe_ffn(x, x_is_f32, T, H, ids, weights, top_k, w_gate, w_up, w_down, E, I,
                   ws_gate, ws_up, ws_down, I_s, NULL, 0, y, nthreads);
}

int oracle_moe_ffn_expert_parallel(const void *x, int x_is_f32, int64_t T, int64_t H,
                                   const int32_t *ids, const double *weights, int32_t top_k,
                                   const uint16_t *const *w_gate, const uint16_t *const *w_up,
                                   const uint16_t *const *w_down, int64_t E, int64_t I,
                                   const uint16_t *ws_gate, const uint16_t *ws_up,
                                   const uint16_t *ws_down, int64_t I_s,
                                   const int64_t *band_start, int32_t bands, double *y,
                                   int nthreads)
{
    if (band_start == NULL)
        return ORACLE_EPLAN;
    return moe_ffn(x, x_is_f32, T, H, ids, weights, top_k, w_gate, w_up, w_down, E, I,
                   ws_gate, ws_up, ws_down, I_s, band_start, bands, y, nthreads);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
