/*
 * moe_oracle.c -- float64 CPU oracle for the forward pass of a top-k routed
 * mixture-of-experts SwiGLU FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker of the
 * CUDA library: only the tests, the smoke check and the timed CPU baseline
 * of the benchmark may load it.  It shares no code, header, table or helper
 * with the CUDA path; it reads the same raw input bits (bf16 or fp32) and
 * nothing else.
 *
 * Every value is widened to double on load (bf16 -> double and fp32 -> double
 * are exact), every sum is a plain left-to-right double sum, and there is no
 * blocking, fusion or reordering beyond what the method states.  The code
 * follows the pages step by step:
 *
 *   route      "Tutorial 11: Mixture of Experts (MoE)", section 2 "The Router"
 *              (route_topk: router logits, softmax over all experts, top-k,
 *              gather of the kept scores, optional renormalisation), and
 *              "Small MoE Architecture, in depth", section "A small MoE layer
 *              in PyTorch" (sigmoid scores, gates = the kept raw scores).
 *   permute    "Tutorial 11", section 3 "Expert Computation", Step 1 (sort the
 *              flattened expert ids; the grouped order) and "Small MoE
 *              Architecture, in depth" (per-expert counts by bincount).
 *   balance    "Small MoE Architecture, in depth", SmallMoE.forward and the
 *              paragraph on auxiliary-loss-free balancing after it (a
 *              per-expert bias added to the scores only when choosing the
 *              top k, and its update from the per-expert load after a step);
 *              "Mixture-of-Experts -- more capacity per byte of weight",
 *              section "What's wired today" (the Switch load-balancing term
 *              alpha * N * sum_e f_e * P_e and the statistics it needs).
 *   forward    "Tutorial 11", section 3 Steps 2-3 and section 4 "The Complete
 *              MoE Layer" (per-row expert SwiGLU, weighted sum over the k
 *              selected experts); the SwiGLU expert is down(silu(gate x) *
 *              up x) as in the Expert module of "Small MoE Architecture, in
 *              depth"; the always-on shared expert is added to every token as
 *              in the same module, scaled by sigmoid(w_s . x).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - top-k slot order: keys in descending order, ties to the lower expert
 *     index (the pages' argpartition leaves the order open; torch.topk sorts).
 *   - selection key: the logit for softmax scoring (softmax is monotone, so
 *     ranking logits ranks probabilities) and sigmoid(logit) for sigmoid.
 *   - "softmax over those four scores" (Small models, sparse experts, "How it
 *     works" step 3) equals full softmax followed by renormalisation of the k
 *     kept probabilities; that configuration is {softmax, norm_topk = 1}.
 *   - the shared expert's gate is sigmoid(w_s . x); its logit takes no part
 *     in the top-k selection.
 *   - silu(u) = u / (1 + exp(-u)); no biases in any linear layer.
 *   - the balance bias is added to the score s_e (softmax probability or
 *     sigmoid score, whichever the layer uses) to form the selection key;
 *     the gates are gathered from the unbiased scores.
 *   - the Switch statistics: f_e = counts[e] / T, the fraction of the T
 *     tokens dispatched to expert e, and P_e = the mean over the T tokens of
 *     the score s_e (the full score row, before selection).
 *
 * Pins: this file is checked, not trusted -- see tests/test_oracle_pins.py
 * (the route_topk worked example, a dense all-experts formulation, a
 * loop-over-experts formulation, E = 1 / k = 1 dense SwiGLU, invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_F32 = 1, ORACLE_F64 = 2 };
enum { ORACLE_SOFTMAX = 0, ORACLE_SIGMOID = 1 };

/* Layer shape and options.  T tokens of width d, E routed experts of hidden
 * width h, k experts per token, h_shared = 0 means no shared expert. */
typedef struct {
    int64_t T;
    int32_t d, E, h, k;
    int32_t norm_topk;
    int32_t score;
    int32_t h_shared;
    int32_t dtype;
} oracle_cfg;

/* Element i of a stored tensor, widened exactly to double.  (float64 inputs
 * exist only so that the pins can difference the layer finely.) */
static double elem(const void *base, int64_t i, int32_t dtype)
{
    if (dtype == ORACLE_F64)
        return ((const double *)base)[i];
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

static double silu(double u) { return u / (1.0 + exp(-u)); }

/* d silu(u) / du = sigmoid(u) * (1 + u * (1 - sigmoid(u))). */
static double dsilu(double u)
{
    double s = sigmoid(u);
    return s * (1.0 + u * (1.0 - s));
}

static int cfg_ok(const oracle_cfg *c)
{
    if (!c || c->T < 0 || c->d < 1 || c->E < 1 || c->h < 1) return 0;
    if (c->k < 1 || c->k > c->E) return 0;
    if (c->score != ORACLE_SOFTMAX && c->score != ORACLE_SIGMOID) return 0;
    if (c->dtype != ORACLE_BF16 && c->dtype != ORACLE_F32 && c->dtype != ORACLE_F64) return 0;
    if (c->h_shared < 0) return 0;
    return 1;
}

/* Router logits of one token: l_e = sum_i x_i * Wr[e, i] (a bias-free linear
 * layer, "Tutorial 11" section 2 step 1; the router of "Small MoE
 * Architecture, in depth" is nn.Linear(d, n_experts, bias=False)). */
static void router_logits(const oracle_cfg *c, const void *x, const void *wr,
                          int64_t t, double *logits)
{
    for (int32_t e = 0; e < c->E; ++e) {
        double s = 0.0;
        for (int32_t i = 0; i < c->d; ++i)
            s += elem(x, t * c->d + i, c->dtype) * elem(wr, (int64_t)e * c->d + i, c->dtype);
        logits[e] = s;
    }
}

/* Selection keys.  Without a balance bias: the logit under softmax (a
 * monotone map, so ranking logits ranks probabilities) and the sigmoid score
 * under sigmoid.  With a bias (SmallMoE.forward: topk of scores +
 * balance_bias): key_e = s_e + bias_e, the score plus the bias. */
static void selection_keys(const oracle_cfg *c, const double *logits, const double *scores,
                           const float *bias, double *keys)
{
    for (int32_t e = 0; e < c->E; ++e) {
        if (bias)
            keys[e] = scores[e] + (double)bias[e];
        else
            keys[e] = (c->score == ORACLE_SIGMOID) ? sigmoid(logits[e]) : logits[e];
    }
}

/* The k best experts, best first: repeatedly take the largest key not yet
 * taken, scanning experts in increasing index so that ties go to the lower
 * index.  O(k * E), plain on purpose. */
static void select_topk(const oracle_cfg *c, const double *keys, char *taken, int32_t *ids)
{
    memset(taken, 0, (size_t)c->E);
    for (int32_t j = 0; j < c->k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < c->E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || keys[e] > keys[best]) best = e;
        }
        taken[best] = 1;
        ids[j] = best;
    }
}

/* Scores over all experts: softmax with the maximum subtracted ("Tutorial 11"
 * section 2 step 2), or the element-wise sigmoid ("Small MoE Architecture, in
 * depth", forward: scores = sigmoid(router(x))). */
static void expert_scores(const oracle_cfg *c, const double *logits, double *scores)
{
    if (c->score == ORACLE_SIGMOID) {
        for (int32_t e = 0; e < c->E; ++e) scores[e] = sigmoid(logits[e]);
        return;
    }
    double m = logits[0];
    for (int32_t e = 1; e < c->E; ++e)
        if (logits[e] > m) m = logits[e];
    double z = 0.0;
    for (int32_t e = 0; e < c->E; ++e) z += exp(logits[e] - m);
    for (int32_t e = 0; e < c->E; ++e) scores[e] = exp(logits[e] - m) / z;
}

/* Routes one token: ids[0..k), gates[0..k), the full score row and the
 * shared-expert gate.  Gates are the selected scores ("Tutorial 11" section 2
 * step 4; with a balance bias still the unbiased scores, SmallMoE.forward),
 * divided by their sum when norm_topk is set (step 5; the worked example
 * under "Why Normalize Selected Probabilities?").  bias may be NULL. */
static void route_one(const oracle_cfg *c, const void *x, const void *wr, const void *w_sg,
                      const float *bias, int64_t t, double *logits, double *keys, double *scores,
                      char *taken, int32_t *ids, double *gates, double *shared_gate)
{
    router_logits(c, x, wr, t, logits);
    expert_scores(c, logits, scores);
    selection_keys(c, logits, scores, bias, keys);
    select_topk(c, keys, taken, ids);
    double sum = 0.0;
    for (int32_t j = 0; j < c->k; ++j) {
        gates[j] = scores[ids[j]];
        sum += gates[j];
    }
    if (c->norm_topk)
        for (int32_t j = 0; j < c->k; ++j) gates[j] /= sum;
    if (shared_gate) {
        double s = 0.0;
        if (c->h_shared > 0 && w_sg) {
            for (int32_t i = 0; i < c->d; ++i)
                s += elem(x, t * c->d + i, c->dtype) * elem(w_sg, i, c->dtype);
            *shared_gate = sigmoid(s);
        } else {
            *shared_gate = 0.0;
        }
    }
}

static int nthreads_used(int requested)
{
#ifdef _OPENMP
    if (requested > 0) return requested;
    return omp_get_max_threads();
#else
    (void)requested;
    return 1;
#endif
}

/* Routes tokens [t0, t1).  ids and gates are [T, k] (indexed by absolute
 * token), probs is an optional [T, E] score matrix, shared_gate an optional
 * [T] vector, bias an optional [E] fp32 balance bias.  Returns 0 on success,
 * -1 on a bad argument. */
int oracle_route(const oracle_cfg *c, const void *x, const void *wr, const void *w_sg,
                 const float *bias, int64_t t0, int64_t t1, int32_t *ids, double *gates,
                 double *probs, double *shared_gate, int nthreads)
{
    if (!cfg_ok(c) || !x || !wr || !ids || !gates || t0 < 0 || t1 > c->T || t0 > t1) return -1;
    int nt = nthreads_used(nthreads);
    int bad = 0;
#pragma omp parallel num_threads(nt)
    {
        double *logits = malloc(sizeof(double) * (size_t)c->E * 3);
        char *taken = malloc((size_t)c->E);
        if (!logits || !taken) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *keys = logits + c->E, *scores = logits + 2 * c->E;
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = t0; t < t1; ++t) {
                route_one(c, x, wr, w_sg, bias, t, logits, keys, scores, taken, ids + t * c->k,
                          gates + t * c->k, shared_gate ? shared_gate + t : NULL);
                if (probs)
                    for (int32_t e = 0; e < c->E; ++e) probs[t * c->E + e] = scores[e];
            }
        }
        free(logits);
        free(taken);
    }
    return bad ? -1 : 0;
}

/* Margin of the selection for tokens [t0, t1): the smallest gap between
 * adjacent keys (with the balance bias when given) among the top
 * min(k + 1, E) keys in descending order.  A
 * margin above the numerical error of a faster implementation means that it
 * must find the same experts in the same slot order. */
int oracle_topk_margin(const oracle_cfg *c, const void *x, const void *wr, const float *bias,
                       int64_t t0, int64_t t1, double *margin, int nthreads)
{
    if (!cfg_ok(c) || !x || !wr || !margin || t0 < 0 || t1 > c->T || t0 > t1) return -1;
    int nt = nthreads_used(nthreads);
    int32_t m = c->k + 1 <= c->E ? c->k + 1 : c->E;
    int bad = 0;
#pragma omp parallel num_threads(nt)
    {
        double *logits = malloc(sizeof(double) * (size_t)c->E * 3);
        char *taken = malloc((size_t)c->E);
        int32_t *order = malloc(sizeof(int32_t) * (size_t)m);
        if (!logits || !taken || !order) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *keys = logits + c->E, *scores = logits + 2 * c->E;
            oracle_cfg cm = *c;
            cm.k = m;
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = t0; t < t1; ++t) {
                router_logits(c, x, wr, t, logits);
                expert_scores(c, logits, scores);
                selection_keys(c, logits, scores, bias, keys);
                select_topk(&cm, keys, taken, order);
                double g = INFINITY;
                for (int32_t j = 0; j + 1 < m; ++j) {
                    double gap = keys[order[j]] - keys[order[j + 1]];
                    if (gap < g) g = gap;
                }
                margin[t - t0] = g;
            }
        }
        free(logits);
        free(taken);
        free(order);
    }
    return bad ? -1 : 0;
}

/* Groups the T*k assignments by expert.  Assignment r = t*k + j carries
 * expert ids[r].  counts[e] = number of assignments to e; offsets is the
 * exclusive prefix sum of counts (E + 1 entries); sorted_rows lists the
 * assignments expert by expert, each expert's in increasing r (a stable sort
 * by expert id, "Tutorial 11" section 3 Step 1); inv_rows is its inverse,
 * inv_rows[sorted_rows[i]] = i.  Returns -1 on an id outside [0, E). */
int oracle_permute(const oracle_cfg *c, const int32_t *ids, int32_t *counts, int32_t *offsets,
                   int32_t *sorted_rows, int32_t *inv_rows)
{
    if (!cfg_ok(c) || !ids || !counts || !offsets || !sorted_rows || !inv_rows) return -1;
    int64_t R = c->T * c->k;
    for (int64_t r = 0; r < R; ++r)
        if (ids[r] < 0 || ids[r] >= c->E) return -1;
    for (int32_t e = 0; e < c->E; ++e) {
        int32_t n = 0;
        for (int64_t r = 0; r < R; ++r) n += (ids[r] == e);
        counts[e] = n;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < c->E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t pos = 0;
    for (int32_t e = 0; e < c->E; ++e)
        for (int64_t r = 0; r < R; ++r)
            if (ids[r] == e) sorted_rows[pos++] = (int32_t)r;
    for (int64_t i = 0; i < R; ++i) inv_rows[sorted_rows[i]] = (int32_t)i;
    return 0;
}

/* One SwiGLU expert applied to token t, scaled by g and added to out[d]:
 * out += g * Wd . (silu(Wg . x) * (Wu . x)).  Wg, Wu are [hid, d] and Wd is
 * [d, hid], all row-major; `a` is scratch of length hid. */
static void swiglu_expert_add(const oracle_cfg *c, const void *x, int64_t t, const void *wg,
                              const void *wu, const void *wd, int64_t w_off_in, int64_t w_off_out,
                              int32_t hid, double g, double *a, double *out)
{
    for (int32_t n = 0; n < hid; ++n) {
        double u = 0.0, v = 0.0;
        for (int32_t i = 0; i < c->d; ++i) {
            double xi = elem(x, t * c->d + i, c->dtype);
            u += elem(wg, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
            v += elem(wu, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
        }
        a[n] = silu(u) * v;
    }
    for (int32_t i = 0; i < c->d; ++i) {
        double o = 0.0;
        for (int32_t n = 0; n < hid; ++n)
            o += elem(wd, w_off_out + (int64_t)i * hid + n, c->dtype) * a[n];
        out[i] += g * o;
    }
}

/* Full layer output for the listed tokens: y[i, :] is token tokens[i]'s
 * output row, y = sum_j gate_j * expert_{ids_j}(x) (+ sigmoid(w_s . x) *
 * shared(x) when h_shared > 0).  W_gate/W_up are [E, h, d], W_down [E, d, h];
 * the shared expert's weights are [h_shared, d], [h_shared, d], [d, h_shared]
 * and w_s is [d]; bias is the optional [E] balance bias.  Routing is recomputed per token, so any subset of tokens
 * can be evaluated on its own.  Returns the number of threads used, or -1. */
int oracle_forward(const oracle_cfg *c, const void *x, const void *wr, const void *wg,
                   const void *wu, const void *wd, const void *sh_g, const void *sh_u,
                   const void *sh_d, const void *w_sg, const float *bias, const int64_t *tokens,
                   int64_t n_tokens, double *y, int nthreads)
{
    if (!cfg_ok(c) || !x || !wr || !wg || !wu || !wd || !tokens || !y || n_tokens < 0) return -1;
    if (c->h_shared > 0 && (!sh_g || !sh_u || !sh_d || !w_sg)) return -1;
    for (int64_t i = 0; i < n_tokens; ++i)
        if (tokens[i] < 0 || tokens[i] >= c->T) return -1;
    int nt = nthreads_used(nthreads);
    int32_t hmax = c->h > c->h_shared ? c->h : c->h_shared;
    int bad = 0;
#pragma omp parallel num_threads(nt)
    {
        double *logits = malloc(sizeof(double) * ((size_t)c->E * 3 + (size_t)c->k + (size_t)hmax));
        char *taken = malloc((size_t)c->E);
        int32_t *ids = malloc(sizeof(int32_t) * (size_t)c->k);
        if (!logits || !taken || !ids) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *keys = logits + c->E, *scores = logits + 2 * c->E;
            double *gates = logits + 3 * c->E, *a = gates + c->k;
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n_tokens; ++i) {
                int64_t t = tokens[i];
                double sg = 0.0;
                route_one(c, x, wr, w_sg, bias, t, logits, keys, scores, taken, ids, gates, &sg);
                double *out = y + i * c->d;
                for (int32_t q = 0; q < c->d; ++q) out[q] = 0.0;
                for (int32_t j = 0; j < c->k; ++j) {
                    int64_t e = ids[j];
                    swiglu_expert_add(c, x, t, wg, wu, wd, e * c->h * c->d, e * c->d * c->h, c->h,
                                      gates[j], a, out);
                }
                if (c->h_shared > 0)
                    swiglu_expert_add(c, x, t, sh_g, sh_u, sh_d, 0, 0, c->h_shared, sg, a, out);
            }
        }
        free(logits);
        free(taken);
        free(ids);
    }
    return bad ? -1 : nt;
}

/* Balance-bias update after a step ("Small MoE Architecture, in depth",
 * SmallMoE.forward in training, and the paragraph on auxiliary-loss-free
 * balancing after it): the load of expert e is counts[e] (the bincount of
 * the chosen ids), and bias_e moves by lr * sign(mean load - load_e): down by
 * lr for an expert above the mean load, up by lr below it, unchanged at it.
 * The bias is a stored fp32 buffer: each new value is formed in double and
 * rounded once to fp32.  bias_out may alias bias_in. */
int oracle_update_bias(const oracle_cfg *c, const int32_t *counts, float lr, const float *bias_in,
                       float *bias_out)
{
    if (!cfg_ok(c) || !counts || !bias_in || !bias_out) return -1;
    double total = 0.0;
    for (int32_t e = 0; e < c->E; ++e) total += (double)counts[e];
    double mean = total / (double)c->E;
    for (int32_t e = 0; e < c->E; ++e) {
        double load = (double)counts[e];
        double sign = 0.0;
        if (mean > load) sign = 1.0;
        if (mean < load) sign = -1.0;
        bias_out[e] = (float)((double)bias_in[e] + (double)lr * sign);
    }
    return 0;
}

/* Mean score per expert over the T tokens, P_e = (1/T) sum_t s_e(t), with
 * s(t) the full score row of token t (softmax probabilities or sigmoid
 * scores, before selection): the router-probability statistic of the Switch
 * load-balancing term ("Mixture-of-Experts -- more capacity per byte of
 * weight", "What's wired today").  Scores are formed per token in parallel
 * and summed over tokens in increasing t.  T = 0 gives zeros. */
int oracle_score_mean(const oracle_cfg *c, const void *x, const void *wr, double *mean, int nthreads)
{
    if (!cfg_ok(c) || !x || !wr || !mean) return -1;
    for (int32_t e = 0; e < c->E; ++e) mean[e] = 0.0;
    if (c->T == 0) return 0;
    double *rows = malloc(sizeof(double) * (size_t)c->T * (size_t)c->E);
    if (!rows) return -1;
    int nt = nthreads_used(nthreads);
    int bad = 0;
#pragma omp parallel num_threads(nt)
    {
        double *logits = malloc(sizeof(double) * (size_t)c->E);
        if (!logits) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < c->T; ++t) {
                router_logits(c, x, wr, t, logits);
                expert_scores(c, logits, rows + t * c->E);
            }
        }
        free(logits);
    }
    if (!bad) {
        for (int32_t e = 0; e < c->E; ++e) {
            double s = 0.0;
            for (int64_t t = 0; t < c->T; ++t) s += rows[t * c->E + e];
            mean[e] = s / (double)c->T;
        }
    }
    free(rows);
    return bad ? -1 : 0;
}

/* The Switch load-balancing term ("Mixture-of-Experts -- more capacity per
 * byte of weight", "What's wired today"): loss = alpha * N * sum_e f_e * P_e
 * with N = E experts, f_e = counts[e] / T (the fraction of the T tokens
 * dispatched to expert e) and P_e = score_mean[e].  frac may be NULL.  T = 0
 * gives f = 0 and loss = 0. */
int oracle_balance_loss(const oracle_cfg *c, const int32_t *counts, const double *score_mean,
                        double alpha, double *frac, double *loss)
{
    if (!cfg_ok(c) || !counts || !score_mean || !loss) return -1;
    double sum = 0.0;
    for (int32_t e = 0; e < c->E; ++e) {
        double f = c->T > 0 ? (double)counts[e] / (double)c->T : 0.0;
        if (frac) frac[e] = f;
        sum += f * score_mean[e];
    }
    *loss = alpha * (double)c->E * sum;
    return 0;
}

/* ------------------------------------------------------------------ backward
 *
 * The gradient of the layer, written out by the chain rule through the same
 * steps as the forward pass above (the pages train this layer -- "Small
 * models, sparse experts", "Dispatch decides everything" reports training
 * tokens/s; "Small MoE Architecture, in depth", SmallMoE -- but print no
 * backward; the backward of a composition of these plain steps has one
 * definition).  Given the upstream gradient dy[T, d] of the output y:
 *
 *   expert j of token t (e = ids_j, gate g_j):
 *     u = Wg[e] x, v = Wu[e] x, a = silu(u) * v, o = Wd[e] a
 *     r  = Wd[e]^T dy            (dy . o = r . a, so dL/dg_j = r . a)
 *     da = g_j r, du = da * v * silu'(u), dv = da * silu(u)
 *     dx += Wg[e]^T du + Wu[e]^T dv
 *     dWd[e] += g_j dy a^T, dWg[e] += du x^T, dWu[e] += dv x^T
 *   shared expert (gate sg = sigmoid(w_s . x)): the same with sg in place of
 *     g_j, and dL/dsg = r_s . a_s, so dl_s = dL/dsg * sg * (1 - sg),
 *     dw_s += dl_s x, dx += dl_s w_s
 *   router: the kept raw scores q_j = s_{ids_j}; with renormalisation
 *     g_j = q_j / Q (Q = sum q), dq_j = (dg_j - sum_i dg_i g_i) / Q, else
 *     dq_j = dg_j; ds_{ids_j} = dq_j and 0 elsewhere; softmax:
 *     dl_e = s_e (ds_e - sum_e' s_e' ds_e'), sigmoid: dl_e = ds_e s_e (1 - s_e);
 *     dWr[e] += dl_e x, dx += sum_e dl_e Wr[e]
 *
 * The top-k selection (with or without the balance bias) is piecewise
 * constant, so it passes no gradient; the bias gets none.
 */

/* Gradient of the router logits of one token from the gradients dg of its k
 * gates (ids, gates, the full score row as route_one leaves them). */
static void router_backward(const oracle_cfg *c, const double *scores, const int32_t *ids,
                            const double *gates, const double *dg, double *ds, double *dl)
{
    double q = 0.0, dot = 0.0;
    for (int32_t j = 0; j < c->k; ++j) {
        q += scores[ids[j]];
        dot += dg[j] * gates[j];
    }
    for (int32_t e = 0; e < c->E; ++e) ds[e] = 0.0;
    for (int32_t j = 0; j < c->k; ++j)
        ds[ids[j]] = c->norm_topk ? (dg[j] - dot) / q : dg[j];
    if (c->score == ORACLE_SIGMOID) {
        for (int32_t e = 0; e < c->E; ++e) dl[e] = ds[e] * scores[e] * (1.0 - scores[e]);
        return;
    }
    double sd = 0.0;
    for (int32_t e = 0; e < c->E; ++e) sd += scores[e] * ds[e];
    for (int32_t e = 0; e < c->E; ++e) dl[e] = scores[e] * (ds[e] - sd);
}

/* u, v and a = silu(u) * v of one expert (rows w_off_in.. of Wg, Wu) on token t. */
static void expert_hidden(const oracle_cfg *c, const void *x, int64_t t, const void *wg, const void *wu,
                          int64_t w_off_in, int32_t hid, double *u, double *v, double *a)
{
    for (int32_t n = 0; n < hid; ++n) {
        double su = 0.0, sv = 0.0;
        for (int32_t i = 0; i < c->d; ++i) {
            double xi = elem(x, t * c->d + i, c->dtype);
            su += elem(wg, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
            sv += elem(wu, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
        }
        u[n] = su;
        v[n] = sv;
        a[n] = silu(su) * sv;
    }
}

/* r = Wd^T dy_t for one expert (Wd = rows w_off_out.. of [d, hid]). */
static void down_transpose(const oracle_cfg *c, const void *dy, int64_t t, const void *wd, int64_t w_off_out,
                           int32_t hid, double *r)
{
    for (int32_t n = 0; n < hid; ++n) {
        double s = 0.0;
        for (int32_t i = 0; i < c->d; ++i)
            s += elem(wd, w_off_out + (int64_t)i * hid + n, c->dtype) * elem(dy, t * c->d + i, c->dtype);
        r[n] = s;
    }
}

/* Backward of one expert on token t with gate g: returns dL/dg = r . a and
 * adds Wg^T du + Wu^T dv into dx_t. */
static double expert_backward_dx(const oracle_cfg *c, const void *x, const void *dy, int64_t t, const void *wg,
                                 const void *wu, const void *wd, int64_t w_off_in, int64_t w_off_out,
                                 int32_t hid, double g, double *u, double *v, double *a, double *r, double *dx_t)
{
    expert_hidden(c, x, t, wg, wu, w_off_in, hid, u, v, a);
    down_transpose(c, dy, t, wd, w_off_out, hid, r);
    double dgate = 0.0;
    for (int32_t n = 0; n < hid; ++n) dgate += r[n] * a[n];
    for (int32_t n = 0; n < hid; ++n) {
        double da = g * r[n];
        double du = da * v[n] * dsilu(u[n]);
        double dv = da * silu(u[n]);
        for (int32_t i = 0; i < c->d; ++i)
            dx_t[i] += elem(wg, w_off_in + (int64_t)n * c->d + i, c->dtype) * du +
                       elem(wu, w_off_in + (int64_t)n * c->d + i, c->dtype) * dv;
    }
    return dgate;
}

/* Weight gradients of hidden unit n of one expert from one token with gate
 * g: row n of dWg / dWu and column n of dWd (stride hid). */
static void expert_backward_w(const oracle_cfg *c, const void *x, const void *dy, int64_t t, const void *wg,
                              const void *wu, const void *wd, int64_t w_off_in, int64_t w_off_out, int32_t hid,
                              int32_t n, double g, double *dwg_row, double *dwu_row, double *dwd_col)
{
    double u = 0.0, v = 0.0, r = 0.0;
    for (int32_t i = 0; i < c->d; ++i) {
        double xi = elem(x, t * c->d + i, c->dtype);
        u += elem(wg, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
        v += elem(wu, w_off_in + (int64_t)n * c->d + i, c->dtype) * xi;
        r += elem(wd, w_off_out + (int64_t)i * hid + n, c->dtype) * elem(dy, t * c->d + i, c->dtype);
    }
    double a = silu(u) * v;
    double da = g * r;
    double du = da * v * dsilu(u);
    double dv = da * silu(u);
    for (int32_t i = 0; i < c->d; ++i) {
        double xi = elem(x, t * c->d + i, c->dtype);
        dwg_row[i] += du * xi;
        dwu_row[i] += dv * xi;
        dwd_col[(int64_t)i * hid] += g * elem(dy, t * c->d + i, c->dtype) * a;
    }
}

/* The layer's backward for all T tokens.  dy has the layer's dtype; every
 * output is float64 and overwritten: dx [T, d], dwr [E, d], dwg and dwu
 * [E, h, d], dwd [E, d, h]; with a shared expert dshg, dshu [h_shared, d],
 * dshd [d, h_shared] and dwsg [d] (else those may be NULL).  bias is the
 * optional balance bias (it changes the selection only).  Tokens are
 * independent in the first pass (dx and the router gradient, parallel over
 * tokens); each weight gradient is then a sum over tokens in increasing t,
 * parallel over experts and hidden units.  Returns 0, or -1 on a bad
 * argument or allocation failure. */
int oracle_backward(const oracle_cfg *c, const void *x, const void *wr, const void *wg, const void *wu,
                    const void *wd, const void *sh_g, const void *sh_u, const void *sh_d, const void *w_sg,
                    const float *bias, const void *dy, double *dx, double *dwr, double *dwg, double *dwu,
                    double *dwd, double *dshg, double *dshu, double *dshd, double *dwsg, int nthreads)
{
    if (!cfg_ok(c) || !x || !wr || !wg || !wu || !wd || !dy || !dx || !dwr || !dwg || !dwu || !dwd) return -1;
    const int shared = c->h_shared > 0;
    if (shared && (!sh_g || !sh_u || !sh_d || !w_sg || !dshg || !dshu || !dshd || !dwsg)) return -1;
    const int64_t T = c->T;
    const int32_t E = c->E, d = c->d, h = c->h, k = c->k, hs = c->h_shared;
    int nt = nthreads_used(nthreads);
    int32_t *ids = malloc(sizeof(int32_t) * (size_t)(T * k > 0 ? T * k : 1));
    double *gates = malloc(sizeof(double) * (size_t)(T * k > 0 ? T * k : 1));
    double *dl = malloc(sizeof(double) * (size_t)(T * E > 0 ? T * E : 1));
    double *sgs = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double *dls = malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    if (!ids || !gates || !dl || !sgs || !dls) {
        free(ids); free(gates); free(dl); free(sgs); free(dls);
        return -1;
    }
    int bad = 0;
    int32_t hmax = h > hs ? h : hs;
    /* pass 1: per token -- routing, the gate gradients, dx, the router's logit gradient */
#pragma omp parallel num_threads(nt)
    {
        double *buf = malloc(sizeof(double) * ((size_t)E * 5 + (size_t)k + 4 * (size_t)hmax));
        char *taken = malloc((size_t)E);
        if (!buf || !taken) {
#pragma omp atomic write
            bad = 1;
        } else {
            double *logits = buf, *keys = buf + E, *scores = buf + 2 * E, *ds = buf + 3 * E;
            double *dlt = buf + 4 * E, *dg = buf + 5 * E, *u = dg + k, *v = u + hmax, *a = v + hmax,
                   *r = a + hmax;
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                double sg = 0.0;
                route_one(c, x, wr, w_sg, bias, t, logits, keys, scores, taken, ids + t * k, gates + t * k,
                          &sg);
                double *dxt = dx + t * d;
                for (int32_t i = 0; i < d; ++i) dxt[i] = 0.0;
                for (int32_t j = 0; j < k; ++j) {
                    int64_t e = ids[t * k + j];
                    dg[j] = expert_backward_dx(c, x, dy, t, wg, wu, wd, e * h * d, e * d * h, h,
                                               gates[t * k + j], u, v, a, r, dxt);
                }
                router_backward(c, scores, ids + t * k, gates + t * k, dg, ds, dlt);
                for (int32_t e = 0; e < E; ++e) {
                    dl[t * E + e] = dlt[e];
                    for (int32_t i = 0; i < d; ++i) dxt[i] += dlt[e] * elem(wr, (int64_t)e * d + i, c->dtype);
                }
                sgs[t] = sg;
                dls[t] = 0.0;
                if (shared) {
                    double dsg = expert_backward_dx(c, x, dy, t, sh_g, sh_u, sh_d, 0, 0, hs, sg, u, v, a, r, dxt);
                    dls[t] = dsg * sg * (1.0 - sg);
                    for (int32_t i = 0; i < d; ++i) dxt[i] += dls[t] * elem(w_sg, i, c->dtype);
                }
            }
        }
        free(buf);
        free(taken);
    }
    if (!bad) {
        /* pass 2: weight gradients, each a sum over tokens in increasing t */
        memset(dwg, 0, sizeof(double) * (size_t)E * h * d);
        memset(dwu, 0, sizeof(double) * (size_t)E * h * d);
        memset(dwd, 0, sizeof(double) * (size_t)E * d * h);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
        for (int32_t e = 0; e < E; ++e)
            for (int32_t i = 0; i < d; ++i) {
                double s = 0.0;
                for (int64_t t = 0; t < T; ++t) s += dl[t * E + e] * elem(x, t * d + i, c->dtype);
                dwr[(int64_t)e * d + i] = s;
            }
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
        for (int64_t en = 0; en < (int64_t)E * h; ++en) {
            int32_t e = (int32_t)(en / h), n = (int32_t)(en % h);
            double *dwg_row = dwg + ((int64_t)e * h + n) * d, *dwu_row = dwu + ((int64_t)e * h + n) * d;
            double *dwd_col = dwd + (int64_t)e * d * h + n;
            for (int64_t t = 0; t < T; ++t)
                for (int32_t j = 0; j < k; ++j)
                    if (ids[t * k + j] == e)
                        expert_backward_w(c, x, dy, t, wg, wu, wd, (int64_t)e * h * d, (int64_t)e * d * h, h, n,
                                          gates[t * k + j], dwg_row, dwu_row, dwd_col);
        }
        if (shared) {
            memset(dshg, 0, sizeof(double) * (size_t)hs * d);
            memset(dshu, 0, sizeof(double) * (size_t)hs * d);
            memset(dshd, 0, sizeof(double) * (size_t)d * hs);
#pragma omp parallel for num_threads(nt) schedule(dynamic, 1)
            for (int32_t n = 0; n < hs; ++n)
                for (int64_t t = 0; t < T; ++t)
                    expert_backward_w(c, x, dy, t, sh_g, sh_u, sh_d, 0, 0, hs, n, sgs[t], dshg + (int64_t)n * d,
                                      dshu + (int64_t)n * d, dshd + n);
            for (int32_t i = 0; i < d; ++i) {
                double s = 0.0;
                for (int64_t t = 0; t < T; ++t) s += dls[t] * elem(x, t * d + i, c->dtype);
                dwsg[i] = s;
            }
        }
    }
    free(ids);
    free(gates);
    free(dl);
    free(sgs);
    free(dls);
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ 4-bit routed experts
 *
 * "Small MoE Architecture, in depth", section "Running experts that do not
 * fit: offloading and quantisation" (routed experts quantised more
 * aggressively than the shared expert and the router) and "Worked example:
 * the batch-1 budget on a device" (4-bit weights, about half a byte per
 * parameter).  The pages fix no format; the one read here: a weight matrix
 * [rows, cols] (cols a multiple of 64) is cut into groups of 64 consecutive
 * elements of a row; each group has the scale s = max|w| / 7 and each element
 * the code q = round(w / s) in [-7, 7] (round to nearest, ties to even),
 * stored as the nibble q + 8, two per byte (element 2i in the low nibble of
 * byte i).  A group of zeros has s = 0 and codes 0.  The value represented is
 * (nibble - 8) * s.  The code is decided in fp32 (s = fp32(max|w|) / 7 and
 * w / s both rounded to fp32), the precision of the kernel that quantises.
 */
int oracle_quantize_q4(const void *w, int32_t dtype, int64_t rows, int32_t cols, uint8_t *q, float *scales)
{
    if (!w || !q || !scales || rows < 0 || cols <= 0 || cols % 64) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F32) return -1;
    const int32_t groups = cols / 64;
    for (int64_t r = 0; r < rows; ++r) {
        for (int32_t g = 0; g < groups; ++g) {
            float m = 0.0f;
            for (int32_t i = 0; i < 64; ++i) {
                float v = (float)elem(w, r * cols + g * 64 + i, dtype);
                if (fabsf(v) > m) m = fabsf(v);
            }
            volatile float s = m / 7.0f;   /* one fp32 division, correctly rounded */
            scales[r * groups + g] = s;
            for (int32_t i = 0; i < 64; i += 2) {
                int code[2];
                for (int z = 0; z < 2; ++z) {
                    float v = (float)elem(w, r * cols + g * 64 + i + z, dtype);
                    if (s == 0.0f) {
                        code[z] = 0;
                    } else {
                        volatile float ratio = v / s;
                        float c = rintf(ratio);
                        if (c > 7.0f) c = 7.0f;
                        if (c < -7.0f) c = -7.0f;
                        code[z] = (int)c;
                    }
                }
                q[r * (cols / 2) + (g * 64 + i) / 2] = (uint8_t)((code[0] + 8) | ((code[1] + 8) << 4));
            }
        }
    }
    return 0;
}

/* The values a 4-bit matrix represents, (nibble - 8) * scale, in double. */
int oracle_dequantize_q4(const uint8_t *q, const float *scales, int64_t rows, int32_t cols, double *out)
{
    if (!q || !scales || !out || rows < 0 || cols <= 0 || cols % 64) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t c = 0; c < cols; ++c) {
            uint8_t b = q[r * (cols / 2) + c / 2];
            int nib = (c % 2 == 0) ? (b & 15) : (b >> 4);
            out[r * cols + c] = (double)(nib - 8) * (double)scales[r * (cols / 64) + c / 64];
        }
    return 0;
}
