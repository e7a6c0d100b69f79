/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for the forward
 * pass of a Mixture-of-Experts FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into liboracle_moe.so and
 * is used by the test-suite, by the smoke check and by the CPU-baseline leg
 * of the benchmark.  The CUDA library never links, includes or calls it, and
 * it shares no code, table or header with the CUDA library.
 *
 * Arithmetic is IEEE double throughout.  bf16 and fp32 inputs are widened
 * exactly to double; nothing is rounded in between.  Every loop is the plain
 * definition: no blocking, no fusion, no reordering.
 *
 * Sources (page title, section / equation):
 *  [VI]  "Mixture-of-Experts" (Vector Institute post), router section:
 *        router score h = x W_r, softmax over experts, top-k selection,
 *        Eq. moe-output (gates taken from the full softmax) and the
 *        renormalised-gate variant described right after it; Eq. balance
 *        (f_i, P_i, E * sum f_i P_i); the expert-capacity paragraph
 *        (limit c*k*T/E, overflow dropped).
 *  [RO]  "Fine-Tuning Mixture of Experts (MoE) Models: Router Optimization
 *        Techniques", "What Is It?" (h = x W_g, TopK, softmax over the
 *        selected logits, output = sum P_i E_i(x), SwiGLU expert),
 *        "How It Works" 1 (f_i, P_i, L_aux = N sum f_i P_i) and 2 (selection
 *        on score + b_i, gate from the unbiased score), "Why It Matters" 3
 *        (capacity; dropped tokens bypass the layer).
 *  [IS]  "Fine-tuning and serving MoE models" (intellisensei tutorial),
 *        "How an MoE layer actually works" (GELU expert Linear-GELU-Linear,
 *        fp32 router softmax, weighted index-add back to token order).
 *  [PK]  "Mixture of Experts" tutorial (prashantkul), "The capacity factor
 *        formula" and "Selective precision".
 *
 * Parity status of each function is pinned by tests (see the test-suite for
 * the pins): brute-force top-k, library softmax/sigmoid, closed-form balance
 * loss (1 under uniform routing, E under collapse), a second loop-over-experts
 * formulation, and the E=1 / k=E special cases reducing to a dense FFN and to
 * the full soft mixture.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- shapes and flags ------------------------------------------------ */
typedef struct {
    int32_t T;            /* tokens                                      */
    int32_t d;            /* d_model                                     */
    int32_t E;            /* routed experts                              */
    int32_t d_ff;         /* hidden width of one routed expert           */
    int32_t k;            /* experts selected per token                  */
    int32_t xw_dtype;     /* 0: x and expert weights are fp32,
                             1: they are bf16 (raw 16-bit patterns)      */
    int32_t act;          /* 0: GELU expert with biases, 1: SwiGLU       */
    int32_t score;        /* 0: softmax scores, 1: sigmoid scores        */
    int32_t renorm;       /* softmax only: 1 renormalise gates over the
                             selected experts, 0 keep full-softmax gates */
    int32_t capacity;     /* tokens one expert may keep; < 0: unlimited  */
    int32_t d_ff_shared;  /* hidden width of the shared expert; 0: none  */
    int32_t nthreads;     /* worker threads for the per-token loops      */
} oracle_dims;

/* Widen element i of a bf16 (dtype 1) or fp32 (dtype 0) array to double.
 * bf16 is the upper half of an fp32 pattern, so the widening is exact.   */
static double wide(const void *base, int dtype, size_t i)
{
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ---- capacity ----------------------------------------------------------
 * [VI] expert-capacity paragraph and [PK] "The capacity factor formula":
 * an expert keeps at most c * k * T / E assignments.  Rounded down; a
 * non-positive factor means no limit.                                     */
int32_t oracle_capacity(double c, int32_t k, int32_t T, int32_t E)
{
    if (!(c > 0.0)) return -1;
    return (int32_t)floor(c * (double)k * (double)T / (double)E);
}

/* ---- threading helper ------------------------------------------------- */
typedef void (*range_fn)(void *ctx, int64_t lo, int64_t hi);
typedef struct { range_fn fn; void *ctx; int64_t lo, hi; } range_job;

static void *range_thread(void *p)
{
    range_job *j = (range_job *)p;
    j->fn(j->ctx, j->lo, j->hi);
    return NULL;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void *ctx)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (n < nthreads) nthreads = (int)(n > 0 ? n : 1);
    if (nthreads == 1) { fn(ctx, 0, n); return; }
    pthread_t tid[256];
    range_job job[256];
    for (int i = 0; i < nthreads; ++i) {
        job[i].fn = fn; job[i].ctx = ctx;
        job[i].lo = n * i / nthreads; job[i].hi = n * (i + 1) / nthreads;
        pthread_create(&tid[i], NULL, range_thread, &job[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(tid[i], NULL);
}

/* ---- router ------------------------------------------------------------
 * For every token t:
 *   h_e   = sum_j x[t,j] * Wr[j,e]  (+ logit_bias[e])        [VI], [RO]
 *   softmax: p_e = exp(h_e - max h) / sum exp(h - max h)      [VI], [IS]
 *   sigmoid: s_e = 1 / (1 + exp(-h_e))
 *   selection key: softmax -> h_e (softmax is strictly increasing in h, so
 *   the k largest p are the k largest h); sigmoid -> s_e; plus sel_bias[e]
 *   when given, which steers the selection only ([RO] How It Works 2).
 *   idx = the k experts with the largest key, largest first; equal keys are
 *   ordered by the lower expert index.
 *   gate: softmax & renorm=0 -> p_idx (Eq. moe-output);
 *         softmax & renorm=1 -> p_idx / sum_{selected} p;
 *         sigmoid            -> s_idx / sum_{selected} s (bias never enters).
 *   pnorm_e (the per-token score whose token-mean is P_e): p_e for softmax,
 *   s_e / sum_all s for sigmoid.
 *   margin[t] = key of the k-th choice minus key of the (k+1)-th (HUGE_VAL
 *   when k == E): the distance from a different selection.
 * Outputs: idx [T,k], gate [T,k], logits [T,E] (h, or NULL), pnorm [T,E]
 * (or NULL), margin [T] (or NULL), sel_key [T,k] (key of each choice, or
 * NULL).                                                                   */
typedef struct {
    const oracle_dims *dm;
    const void *x; const float *Wr; const float *logit_bias; const float *sel_bias;
    int32_t *idx; double *gate; double *logits; double *pnorm; double *margin; double *sel_key;
    const int32_t *tokens;      /* optional subset of tokens (NULL: all) */
} route_ctx;

static void route_range(void *vctx, int64_t lo, int64_t hi)
{
    route_ctx *c = (route_ctx *)vctx;
    const oracle_dims *dm = c->dm;
    const int E = dm->E, d = dm->d, k = dm->k;
    double *h = (double *)malloc(sizeof(double) * E);
    double *sc = (double *)malloc(sizeof(double) * E);   /* p or s       */
    double *key = (double *)malloc(sizeof(double) * E);
    int *order = (int *)malloc(sizeof(int) * E);
    for (int64_t n = lo; n < hi; ++n) {
        int64_t t = c->tokens ? c->tokens[n] : n;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += wide(c->x, dm->xw_dtype, (size_t)t * d + j) * (double)c->Wr[(size_t)j * E + e];
            if (c->logit_bias) acc += (double)c->logit_bias[e];
            h[e] = acc;
        }
        double norm = 0.0;
        if (dm->score == 0) {
            double mx = h[0];
            for (int e = 1; e < E; ++e) if (h[e] > mx) mx = h[e];
            for (int e = 0; e < E; ++e) { sc[e] = exp(h[e] - mx); norm += sc[e]; }
            for (int e = 0; e < E; ++e) sc[e] /= norm;
            for (int e = 0; e < E; ++e) key[e] = h[e];
        } else {
            for (int e = 0; e < E; ++e) { sc[e] = 1.0 / (1.0 + exp(-h[e])); norm += sc[e]; }
            for (int e = 0; e < E; ++e) key[e] = sc[e];
        }
        if (c->sel_bias) for (int e = 0; e < E; ++e) key[e] += (double)c->sel_bias[e];
        /* selection: insertion sort of expert ids by (key desc, id asc) */
        for (int e = 0; e < E; ++e) {
            int pos = e;
            while (pos > 0 && key[order[pos - 1]] < key[e]) { order[pos] = order[pos - 1]; --pos; }
            order[pos] = e;
        }
        double selsum = 0.0;
        for (int s = 0; s < k; ++s) selsum += sc[order[s]];
        for (int s = 0; s < k; ++s) {
            int e = order[s];
            c->idx[n * k + s] = e;
            double g;
            if (dm->score == 0 && dm->renorm == 0) g = sc[e];
            else g = sc[e] / selsum;
            c->gate[n * k + s] = g;
            if (c->sel_key) c->sel_key[n * k + s] = key[e];
        }
        if (c->logits) for (int e = 0; e < E; ++e) c->logits[n * E + e] = h[e];
        if (c->pnorm) {
            for (int e = 0; e < E; ++e)
                c->pnorm[n * E + e] = (dm->score == 0) ? sc[e] : sc[e] / norm;
        }
        if (c->margin) c->margin[n] = (k < E) ? key[order[k - 1]] - key[order[k]] : HUGE_VAL;
    }
    free(h); free(sc); free(key); free(order);
}

int oracle_route(const oracle_dims *dm, int64_t ntok, const int32_t *tokens,
                 const void *x, const float *Wr, const float *logit_bias, const float *sel_bias,
                 int32_t *idx, double *gate, double *logits, double *pnorm, double *margin,
                 double *sel_key)
{
    if (!dm || dm->k < 1 || dm->k > dm->E || dm->d < 1) return 1;
    route_ctx c = { dm, x, Wr, logit_bias, sel_bias, idx, gate, logits, pnorm, margin, sel_key, tokens };
    parallel_for(ntok, dm->nthreads, route_range, &c);
    return 0;
}

/* ---- counts, capacity and permutation ----------------------------------
 * counts[e]  = number of (t, s) with idx[t,s] == e             ([RO] bincount)
 * Visit tokens in ascending t (slots in ascending s): rank = seen[e]++;
 * the assignment is kept when rank < capacity ([VI] capacity paragraph; the
 * first-come order is this implementation's reading).  Dropped assignments
 * contribute nothing ([RO] Why It Matters 3: they bypass the layer).
 * kept[e]    = min(counts[e], capacity)
 * offsets    = exclusive prefix sum of kept, offsets[E] = total kept rows
 * row_of[t,s]= offsets[e] + rank if kept, else -1
 * row_token[row] = t   (rows in (expert, token) order)                    */
int oracle_dispatch(const oracle_dims *dm, const int32_t *idx, int32_t *counts, int32_t *kept,
                    int32_t *offsets, int32_t *row_of, int32_t *row_token, int32_t *n_dropped)
{
    const int E = dm->E, k = dm->k;
    const int64_t T = dm->T;
    int32_t *seen = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T * k > 0 ? T * k : 1));
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < T; ++t)
        for (int s = 0; s < k; ++s) {
            int e = idx[t * k + s];
            if (e < 0 || e >= E) { free(seen); free(rank); return 1; }
            counts[e] += 1;
            rank[t * k + s] = seen[e]++;
        }
    int32_t dropped = 0;
    for (int e = 0; e < E; ++e) {
        kept[e] = (dm->capacity >= 0 && counts[e] > dm->capacity) ? dm->capacity : counts[e];
        dropped += counts[e] - kept[e];
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + kept[e];
    for (int64_t t = 0; t < T; ++t)
        for (int s = 0; s < k; ++s) {
            int e = idx[t * k + s];
            int32_t r = rank[t * k + s];
            if (dm->capacity >= 0 && r >= dm->capacity) { row_of[t * k + s] = -1; continue; }
            int32_t row = offsets[e] + r;
            row_of[t * k + s] = row;
            if (row_token) row_token[row] = (int32_t)t;
        }
    if (n_dropped) *n_dropped = dropped;
    free(seen); free(rank);
    return 0;
}

/* ---- balance statistics -------------------------------------------------
 * [VI] Eq. balance, [RO] How It Works 1, [IS] load_balancing_loss:
 *   f_e = counts_e / (T * k)    (router decisions, before any capacity drop;
 *                                dividing by k makes sum f = 1, so L = 1 under
 *                                uniform routing for every k)
 *   P_e = (1/T) sum_t pnorm[t,e]
 *   L   = E * sum_e f_e * P_e                                              */
int oracle_balance(const oracle_dims *dm, const int32_t *counts, const double *pnorm,
                   double *f, double *P, double *L)
{
    const int E = dm->E;
    const int64_t T = dm->T;
    double acc = 0.0;
    for (int e = 0; e < E; ++e) {
        f[e] = (double)counts[e] / ((double)T * (double)dm->k);
        double s = 0.0;
        for (int64_t t = 0; t < T; ++t) s += pnorm[t * E + e];
        P[e] = s / (double)T;
        acc += f[e] * P[e];
    }
    *L = (double)E * acc;
    return 0;
}

/* ---- one expert on one token -------------------------------------------
 * GELU expert ([IS] "How an MoE layer actually works"):
 *   a_j = sum_i W1[e,j,i] x_i + b1[e,j];  h_j = a_j * Phi(a_j)
 *        = 0.5 a_j (1 + erf(a_j / sqrt 2))  (exact-erf GELU, nn.GELU default)
 *   o_i = sum_j W2[e,i,j] h_j + b2[e,i]
 * SwiGLU expert ([RO] "What Is It?"):
 *   g_j = sum_i Wg[e,j,i] x_i;  u_j = sum_i Wu[e,j,i] x_i
 *   h_j = g_j / (1 + exp(-g_j)) * u_j;   o_i = sum_j Wd[e,i,j] h_j
 * Weight layouts follow nn.Linear: [out, in], stacked over experts.        */
typedef struct {
    const oracle_dims *dm;
    const void *x;
    const void *W1; const float *b1; const void *Wu; const void *W2; const float *b2;
    const void *Wsg; const void *Wsu; const void *Wsd;
} expert_weights;

static void expert_apply_one(const expert_weights *w, int64_t t, int e, double *hbuf, double *out)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d, dt = dm->xw_dtype;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const void *Wa = shared ? w->Wsg : w->W1;
    const void *Wb = shared ? w->Wsu : w->Wu;
    const void *Wo = shared ? w->Wsd : w->W2;
    const size_t ebase = shared ? 0 : (size_t)e;
    for (int j = 0; j < dff; ++j) {
        double a = 0.0;
        for (int i = 0; i < d; ++i)
            a += wide(Wa, dt, (ebase * dff + j) * d + i) * wide(w->x, dt, (size_t)t * d + i);
        if (dm->act == 0 && !shared) {
            if (w->b1) a += (double)w->b1[ebase * dff + j];
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else if (dm->act == 0) {
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else {
            double u = 0.0;
            for (int i = 0; i < d; ++i)
                u += wide(Wb, dt, (ebase * dff + j) * d + i) * wide(w->x, dt, (size_t)t * d + i);
            hbuf[j] = a / (1.0 + exp(-a)) * u;
        }
    }
    for (int i = 0; i < d; ++i) {
        double o = 0.0;
        for (int j = 0; j < dff; ++j)
            o += wide(Wo, dt, (ebase * d + i) * dff + j) * hbuf[j];
        if (dm->act == 0 && !shared && w->b2) o += (double)w->b2[ebase * d + i];
        out[i] = o;
    }
}

/* out[r,:] = scale[r] * E_{expert[r]}(x[token[r],:]); expert == E selects the
 * shared expert (GELU without biases when act == 0, SwiGLU otherwise).     */
typedef struct {
    expert_weights w;
    const int32_t *token; const int32_t *expert; const double *scale; double *out;
} apply_ctx;

static void apply_range(void *vctx, int64_t lo, int64_t hi)
{
    apply_ctx *c = (apply_ctx *)vctx;
    const oracle_dims *dm = c->w.dm;
    int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
    for (int64_t r = lo; r < hi; ++r) {
        double *o = c->out + (size_t)r * dm->d;
        expert_apply_one(&c->w, c->token[r], c->expert[r], hbuf, o);
        double sc = c->scale ? c->scale[r] : 1.0;
        for (int i = 0; i < dm->d; ++i) o[i] *= sc;
    }
    free(hbuf);
}

int oracle_expert_apply(const oracle_dims *dm, int64_t nrows, const int32_t *token,
                        const int32_t *expert, const double *scale, const void *x,
                        const void *W1, const float *b1, const void *Wu, const void *W2, const float *b2,
                        const void *Wsg, const void *Wsu, const void *Wsd, double *out)
{
    for (int64_t r = 0; r < nrows; ++r) {
        if (expert[r] < 0 || expert[r] > dm->E) return 1;
        if (expert[r] == dm->E && dm->d_ff_shared <= 0) return 1;
    }
    apply_ctx c = { { dm, x, W1, b1, Wu, W2, b2, Wsg, Wsu, Wsd }, token, expert, scale, out };
    parallel_for(nrows, dm->nthreads, apply_range, &c);
    return 0;
}

/* ---- the layer output for a list of tokens -------------------------------
 * [VI] Eq. moe-output, [RO] "What Is It?", [IS] forward():
 *   y_t = sum_{s : row_of[t,s] >= 0} gate[t,s] * E_{idx[t,s]}(x_t)
 *         (+ shared expert output, weight 1, when d_ff_shared > 0)
 * A dropped assignment (row_of < 0) adds nothing.                          */
typedef struct {
    expert_weights w;
    const int32_t *tokens; const int32_t *idx; const double *gate; const int32_t *row_of;
    double *y;
} layer_ctx;

static void layer_range(void *vctx, int64_t lo, int64_t hi)
{
    layer_ctx *c = (layer_ctx *)vctx;
    const oracle_dims *dm = c->w.dm;
    const int d = dm->d, k = dm->k;
    int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t n = lo; n < hi; ++n) {
        int64_t t = c->tokens[n];
        double *y = c->y + (size_t)n * d;
        for (int i = 0; i < d; ++i) y[i] = 0.0;
        for (int s = 0; s < k; ++s) {
            if (c->row_of && c->row_of[t * k + s] < 0) continue;
            expert_apply_one(&c->w, t, c->idx[t * k + s], hbuf, o);
            double g = c->gate[t * k + s];
            for (int i = 0; i < d; ++i) y[i] += g * o[i];
        }
        if (dm->d_ff_shared > 0) {
            expert_apply_one(&c->w, t, dm->E, hbuf, o);
            for (int i = 0; i < d; ++i) y[i] += o[i];
        }
    }
    free(hbuf); free(o);
}

int oracle_layer_tokens(const oracle_dims *dm, int64_t ntok, const int32_t *tokens,
                        const void *x, const int32_t *idx, const double *gate, const int32_t *row_of,
                        const void *W1, const float *b1, const void *Wu, const void *W2, const float *b2,
                        const void *Wsg, const void *Wsu, const void *Wsd, double *y)
{
    layer_ctx c = { { dm, x, W1, b1, Wu, W2, b2, Wsg, Wsu, Wsd }, tokens, idx, gate, row_of, y };
    parallel_for(ntok, dm->nthreads, layer_range, &c);
    return 0;
}

/* ---- auxiliary-loss-free bias update -------------------------------------
 * [RO] How It Works 2 and the dynamic-bias router module, step 5: after a
 * step, with L_e the assignments expert e received and L_target = T k / E,
 *   b_e <- b_e - gamma * sign(L_e - L_target)
 * (overloaded experts lose gamma, underloaded ones gain it, exactly loaded
 * ones keep their bias).  Arithmetic in double, result stored as float.     */
int oracle_bias_update(const oracle_dims *dm, const int32_t *counts, double gamma, float *bias)
{
    const double target = (double)dm->T * (double)dm->k / (double)dm->E;
    for (int e = 0; e < dm->E; ++e) {
        const double err = (double)counts[e] - target;
        const double sgn = err > 0.0 ? 1.0 : (err < 0.0 ? -1.0 : 0.0);
        bias[e] = (float)((double)bias[e] - gamma * sgn);
    }
    return 0;
}

/* ---- routing health ------------------------------------------------------
 * [RO] Best Practices 6: Shannon entropy H = -sum_e P_e log P_e of the layer's
 * mean routing distribution P (terms with P_e = 0 add 0); [IS] "Utilization
 * is a first-class metric": the max/min ratio of the per-expert counts
 * (HUGE_VAL when some expert received nothing), and the largest share
 * max_e counts_e / (T k).  out = {H, ratio, max share}.                     */
int oracle_routing_health(const oracle_dims *dm, const int32_t *counts, const double *P, double *out)
{
    double H = 0.0;
    int32_t mx = counts[0], mn = counts[0];
    for (int e = 0; e < dm->E; ++e) {
        if (P[e] > 0.0) H -= P[e] * log(P[e]);
        if (counts[e] > mx) mx = counts[e];
        if (counts[e] < mn) mn = counts[e];
    }
    out[0] = H;
    out[1] = mn > 0 ? (double)mx / (double)mn : HUGE_VAL;
    out[2] = (double)mx / ((double)dm->T * (double)dm->k);
    return 0;
}

/* ---- FP8 (e4m3) experts ----------------------------------------------------
 * [IS] "Serving: throughput does not scale the way you expect", its list of
 * consequences for capacity planning: quantize the experts to FP8 (or INT4),
 * since memory binds.  The pages give no recipe; the reading written out
 * here is W8A8 e4m3:
 *   e4m3 (OCP 8-bit floating point, E4M3): sign bit, 4 exponent bits with
 *   bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6;
 *   no infinities; S.1111.111 is NaN; the largest finite magnitude is 448.
 *   Expert weights: one e4m3 code per element and one fp32 scale per output
 *   channel (row of the nn.Linear [out, in] matrix): W[n][j] = code * scale[n].
 *   Activations (x, and the hidden activation H of each expert): one scale per
 *   row, from fp32 arithmetic on the row's values v:
 *     amax  = max_j |v_j|
 *     inv   = 448 / amax          (fp32 quotient; 0 when amax = 0)
 *     code  = e4m3 nearest to v_j * inv (fp32 product), ties to the even
 *             mantissa, magnitudes above 448 saturated to 448, sign kept
 *     scale = amax / 448          (fp32 quotient)
 *   H is held in bf16 (nearest, ties to even, from its exact value) before its
 *   row is quantized.  Everything else is the expert of the bf16 layer, in
 *   double, on the exactly dequantized values.                              */

/* Value of an e4m3 code (NaN for the two NaN codes).                        */
double oracle_e4m3_value(uint8_t c)
{
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    const double v = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest integer to a non-negative x, ties to even.                        */
static double round_half_even(double x)
{
    const double fl = floor(x), diff = x - fl;
    if (diff > 0.5) return fl + 1.0;
    if (diff < 0.5) return fl;
    return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;
}

/* e4m3 code nearest to q (see above).  Within a binade the e4m3 values are
 * the multiples of step = 2^(e-3) (2^-9 below 2^-6), so the magnitude is
 * rounded to a multiple of its binade's step; the division is exact.        */
uint8_t oracle_e4m3_round(float q)
{
    const double a = fabs((double)q);
    const uint8_t sign = signbit(q) ? 0x80 : 0x00;
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        const double n = round_half_even(a / ldexp(1.0, -9));      /* 0 .. 8 */
        return sign | (uint8_t)(n >= 8.0 ? 0x08 : (int)n);
    }
    int x;
    (void)frexp(a, &x);                      /* a = f * 2^x, f in [0.5, 1)  */
    int e = x - 1;                           /* 2^e <= a < 2^(e+1), -6..8   */
    double n = round_half_even(a / ldexp(1.0, e - 3));              /* 8 .. 16 */
    if (n >= 16.0) { e += 1; n = 8.0; }
    if (e > 8 || (e == 8 && n > 14.0)) return sign | 0x7E;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* Per-row quantization of rows x cols fp32 values (row stride ld).          */
int oracle_quantize_rows(const float *v, int64_t rows, int32_t cols, int64_t ld, uint8_t *codes,
                         float *scale)
{
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = v + r * ld;
        float amax = 0.0f;
        for (int j = 0; j < cols; ++j) {
            const float a = fabsf(row[j]);
            if (a > amax) amax = a;
        }
        const float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
        for (int j = 0; j < cols; ++j) {
            const float p = row[j] * inv;
            codes[r * (int64_t)cols + j] = oracle_e4m3_round(p);
        }
        scale[r] = amax / 448.0f;
    }
    return 0;
}

/* Nearest bf16 to h (ties to even), returned as a float (exact).            */
static float round_bf16(double h)
{
    if (h == 0.0 || !isfinite(h)) return (float)h;
    const double a = fabs(h);
    int x;
    (void)frexp(a, &x);                      /* 2^(x-1) <= a < 2^x          */
    int e = x - 1;
    if (e < -126) e = -126;                  /* bf16 subnormals: fixed step */
    const double step = ldexp(1.0, e - 7);   /* 8 significant bits          */
    const double r = round_half_even(a / step) * step;
    return (float)(h < 0 ? -r : r);
}

typedef struct {
    const oracle_dims *dm;
    const uint8_t *x8; const float *xs;                     /* [T, d], [T]       */
    const uint8_t *W1; const float *s1; const float *b1;    /* [E, d_ff, d] ...  */
    const uint8_t *Wu; const float *su;
    const uint8_t *W2; const float *s2; const float *b2;    /* [E, d, d_ff], [E, d] */
    const uint8_t *Wsg; const float *ssg;
    const uint8_t *Wsu; const float *ssu;
    const uint8_t *Wsd; const float *ssd;
} fp8_experts;

static double wq(const uint8_t *W, const float *s, size_t row, size_t cols, size_t j)
{
    return oracle_e4m3_value(W[row * cols + j]) * (double)s[row];
}

/* One FP8 expert on token t (e == E: the shared expert).  hbuf: d_ff doubles,
 * hf: d_ff floats, hc: d_ff bytes of scratch.                               */
static void expert_apply_fp8_one(const fp8_experts *w, int64_t t, int e, double *hbuf, float *hf,
                                 uint8_t *hc, double *out)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const uint8_t *Wa = shared ? w->Wsg : w->W1, *Wb = shared ? w->Wsu : w->Wu, *Wo = shared ? w->Wsd : w->W2;
    const float *sa = shared ? w->ssg : w->s1, *sb = shared ? w->ssu : w->su, *so = shared ? w->ssd : w->s2;
    const size_t eb = shared ? 0 : (size_t)e;
    const double xscale = (double)w->xs[t];
    for (int j = 0; j < dff; ++j) {
        double a = 0.0;
        for (int i = 0; i < d; ++i)
            a += wq(Wa, sa, eb * dff + j, d, i) * (oracle_e4m3_value(w->x8[(size_t)t * d + i]) * xscale);
        if (dm->act == 0) {
            if (!shared && w->b1) a += (double)w->b1[eb * dff + j];
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else {
            double u = 0.0;
            for (int i = 0; i < d; ++i)
                u += wq(Wb, sb, eb * dff + j, d, i) * (oracle_e4m3_value(w->x8[(size_t)t * d + i]) * xscale);
            hbuf[j] = a / (1.0 + exp(-a)) * u;
        }
        hf[j] = round_bf16(hbuf[j]);
    }
    float hs;
    oracle_quantize_rows(hf, 1, dff, dff, hc, &hs);
    for (int i = 0; i < d; ++i) {
        double o = 0.0;
        for (int j = 0; j < dff; ++j)
            o += wq(Wo, so, eb * d + i, dff, j) * (oracle_e4m3_value(hc[j]) * (double)hs);
        if (dm->act == 0 && !shared && w->b2) o += (double)w->b2[eb * d + i];
        out[i] = o;
    }
}

typedef struct {
    fp8_experts w;
    const int32_t *token; const int32_t *expert; const double *scale; double *out;
} apply8_ctx;

static void apply8_range(void *vctx, int64_t lo, int64_t hi)
{
    apply8_ctx *c = (apply8_ctx *)vctx;
    const oracle_dims *dm = c->w.dm;
    const int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    const size_t hn = (size_t)(hmax > 0 ? hmax : 1);
    double *hbuf = (double *)malloc(sizeof(double) * hn);
    float *hf = (float *)malloc(sizeof(float) * hn);
    uint8_t *hc = (uint8_t *)malloc(hn);
    for (int64_t r = lo; r < hi; ++r) {
        double *o = c->out + (size_t)r * dm->d;
        expert_apply_fp8_one(&c->w, c->token[r], c->expert[r], hbuf, hf, hc, o);
        const double sc = c->scale ? c->scale[r] : 1.0;
        for (int i = 0; i < dm->d; ++i) o[i] *= sc;
    }
    free(hbuf); free(hf); free(hc);
}

/* out[r,:] = scale[r] * E8_{expert[r]}(x8[token[r],:]) for FP8 experts;
 * expert == E selects the shared expert.                                    */
int oracle_expert_apply_fp8(const oracle_dims *dm, int64_t nrows, const int32_t *token,
                            const int32_t *expert, const double *scale, const uint8_t *x8, const float *xs,
                            const uint8_t *W1, const float *s1, const float *b1,
                            const uint8_t *Wu, const float *su,
                            const uint8_t *W2, const float *s2, const float *b2,
                            const uint8_t *Wsg, const float *ssg, const uint8_t *Wsu, const float *ssu,
                            const uint8_t *Wsd, const float *ssd, double *out)
{
    for (int64_t r = 0; r < nrows; ++r) {
        if (expert[r] < 0 || expert[r] > dm->E) return 1;
        if (expert[r] == dm->E && dm->d_ff_shared <= 0) return 1;
    }
    apply8_ctx c = { { dm, x8, xs, W1, s1, b1, Wu, su, W2, s2, b2, Wsg, ssg, Wsu, ssu, Wsd, ssd },
                     token, expert, scale, out };
    parallel_for(nrows, dm->nthreads, apply8_range, &c);
    return 0;
}

/* ---- Block-scaled FP8 (MX) experts ------------------------------------------
 * [IS] Serving section (quantized experts, FP8 or INT4, once memory binds).
 * The block-scaled reading follows the OCP microscaling (MX) FP8 layout: along
 * the contraction dimension of every matrix, each run of 32 consecutive
 * values shares one power-of-two scale 2^X, stored as the byte X + 127
 * (E8M0), and every value is stored as an e4m3 code:
 *   amax = max |v_j| over the block
 *   X    = floor(log2(amax)) - 8       (8: the exponent of e4m3's largest
 *                                       normal, 448 = 1.75 * 2^8), clamped to
 *                                       [-127, 127]; X = -127 for amax = 0
 *   code = e4m3 nearest to v_j / 2^X (ties to even, saturating at 448, sign
 *          kept); the division by a power of two is exact
 * so the block's largest magnitude maps into [256, 512) and values above 448
 * saturate.  x is quantized per token row along d_model, each weight matrix
 * per output row along its input dimension, and H (held in bf16 first) per
 * row along d_ff.  A product of two blocks is
 *   2^(Xa + Xw) * sum_j e4m3(a_j) e4m3(w_j),
 * summed over the blocks in double.                                         */

/* X of a block whose largest magnitude is amax > 0.                          */
static int mx_exponent(float amax)
{
    int x;
    (void)frexp((double)amax, &x);           /* amax = f 2^x, f in [0.5, 1)   */
    int X = (x - 1) - 8;
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    return X;
}

/* MX quantization of rows x cols fp32 values (row stride ld, cols a
 * multiple of 32): codes [rows, cols], scale bytes [rows, cols / 32].       */
int oracle_quantize_mx(const float *v, int64_t rows, int32_t cols, int64_t ld, uint8_t *codes, uint8_t *scales)
{
    if (cols <= 0 || cols % 32 != 0) return 1;
    const int nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = v + r * ld;
        for (int b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int j = 0; j < 32; ++j) {
                const float a = fabsf(row[b * 32 + j]);
                if (a > amax) amax = a;
            }
            const int X = amax > 0.0f ? mx_exponent(amax) : -127;
            scales[r * nb + b] = (uint8_t)(X + 127);
            for (int j = 0; j < 32; ++j) {
                const double q = ldexp((double)row[b * 32 + j], -X);
                codes[r * (int64_t)cols + b * 32 + j] = oracle_e4m3_round((float)q);
            }
        }
    }
    return 0;
}

/* sum over the n / 32 blocks of 2^(Xa + Xw) * sum_j e4m3(a_j) e4m3(w_j).      */
static double mx_dot(const uint8_t *a, const uint8_t *as, const uint8_t *w, const uint8_t *ws, int n)
{
    double s = 0.0;
    for (int b = 0; b < n / 32; ++b) {
        double blk = 0.0;
        for (int j = 0; j < 32; ++j) blk += oracle_e4m3_value(a[b * 32 + j]) * oracle_e4m3_value(w[b * 32 + j]);
        s += ldexp(blk, ((int)as[b] - 127) + ((int)ws[b] - 127));
    }
    return s;
}

typedef struct {
    const oracle_dims *dm;
    const uint8_t *x8, *xs;                                  /* [T, d], [T, d/32]             */
    const uint8_t *W1, *s1; const float *b1;                 /* [E, d_ff, d], [E, d_ff, d/32]  */
    const uint8_t *Wu, *su;
    const uint8_t *W2, *s2; const float *b2;                 /* [E, d, d_ff], [E, d, d_ff/32]  */
    const uint8_t *Wsg, *ssg, *Wsu, *ssu, *Wsd, *ssd;        /* shared expert, same layouts    */
} mx_experts;

/* One MX expert on token t (e == E: the shared expert).  hbuf: d_ff doubles,
 * hf: d_ff floats, hc: d_ff bytes, hs: d_ff / 32 bytes of scratch.          */
static void expert_apply_mx_one(const mx_experts *w, int64_t t, int e, double *hbuf, float *hf, uint8_t *hc,
                                uint8_t *hs, double *out)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const uint8_t *Wa = shared ? w->Wsg : w->W1, *Wb = shared ? w->Wsu : w->Wu, *Wo = shared ? w->Wsd : w->W2;
    const uint8_t *sa = shared ? w->ssg : w->s1, *sb = shared ? w->ssu : w->su, *so = shared ? w->ssd : w->s2;
    const size_t eb = shared ? 0 : (size_t)e;
    const uint8_t *xr = w->x8 + (size_t)t * d, *xsr = w->xs + (size_t)t * (d / 32);
    for (int j = 0; j < dff; ++j) {
        const size_t wr = eb * dff + j;
        double a = mx_dot(xr, xsr, Wa + wr * d, sa + wr * (d / 32), d);
        if (dm->act == 0) {
            if (!shared && w->b1) a += (double)w->b1[eb * dff + j];
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else {
            const double u = mx_dot(xr, xsr, Wb + wr * d, sb + wr * (d / 32), d);
            hbuf[j] = a / (1.0 + exp(-a)) * u;
        }
        hf[j] = round_bf16(hbuf[j]);
    }
    oracle_quantize_mx(hf, 1, dff, dff, hc, hs);
    for (int i = 0; i < d; ++i) {
        const size_t orow = eb * d + i;
        double o = mx_dot(hc, hs, Wo + orow * dff, so + orow * (dff / 32), dff);
        if (dm->act == 0 && !shared && w->b2) o += (double)w->b2[eb * d + i];
        out[i] = o;
    }
}

typedef struct {
    mx_experts w;
    const int32_t *token; const int32_t *expert; const double *scale; double *out;
} applymx_ctx;

static void applymx_range(void *vctx, int64_t lo, int64_t hi)
{
    applymx_ctx *c = (applymx_ctx *)vctx;
    const oracle_dims *dm = c->w.dm;
    const int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    const size_t hn = (size_t)(hmax > 0 ? hmax : 32);
    double *hbuf = (double *)malloc(sizeof(double) * hn);
    float *hf = (float *)malloc(sizeof(float) * hn);
    uint8_t *hc = (uint8_t *)malloc(hn);
    uint8_t *hs = (uint8_t *)malloc(hn / 32 + 1);
    for (int64_t r = lo; r < hi; ++r) {
        double *o = c->out + (size_t)r * dm->d;
        expert_apply_mx_one(&c->w, c->token[r], c->expert[r], hbuf, hf, hc, hs, o);
        const double sc = c->scale ? c->scale[r] : 1.0;
        for (int i = 0; i < dm->d; ++i) o[i] *= sc;
    }
    free(hbuf); free(hf); free(hc); free(hs);
}

/* out[r,:] = scale[r] * Emx_{expert[r]}(x8[token[r],:]) for MX experts;
 * expert == E selects the shared expert.  d, d_ff (and d_ff_shared) must be
 * multiples of 32.                                                          */
int oracle_expert_apply_mx(const oracle_dims *dm, int64_t nrows, const int32_t *token, const int32_t *expert,
                           const double *scale, const uint8_t *x8, const uint8_t *xs,
                           const uint8_t *W1, const uint8_t *s1, const float *b1,
                           const uint8_t *Wu, const uint8_t *su,
                           const uint8_t *W2, const uint8_t *s2, const float *b2,
                           const uint8_t *Wsg, const uint8_t *ssg, const uint8_t *Wsu, const uint8_t *ssu,
                           const uint8_t *Wsd, const uint8_t *ssd, double *out)
{
    if (dm->d % 32 != 0 || dm->d_ff % 32 != 0 || (dm->d_ff_shared > 0 && dm->d_ff_shared % 32 != 0)) return 2;
    for (int64_t r = 0; r < nrows; ++r) {
        if (expert[r] < 0 || expert[r] > dm->E) return 1;
        if (expert[r] == dm->E && dm->d_ff_shared <= 0) return 1;
    }
    applymx_ctx c = { { dm, x8, xs, W1, s1, b1, Wu, su, W2, s2, b2, Wsg, ssg, Wsu, ssu, Wsd, ssd },
                      token, expert, scale, out };
    parallel_for(nrows, dm->nthreads, applymx_range, &c);
    return 0;
}

/* ---- INT4 weight-only experts -----------------------------------------------
 * [IS] Serving: weight-only INT4 experts (torchao's INT4 weight-only path) once
 * memory binds.  The reading written out here: every expert weight matrix
 * [out, in] is stored as signed 4-bit integers q in [-8, 7], two per byte
 * (the low nibble holds the even input index; a nibble stores q + 8), with one
 * bf16 scale per output row and group of 128 consecutive inputs; a weight's
 * value is the bf16 nearest to q * s (ties to even).  Everything else is the
 * bf16 layer's expert (bf16 x, H exact), in double on the exact weight
 * values.                                                                    */

static double bf16_bits_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Value of input j of weight row `row` (cols inputs per row).                */
static double w4_value(const uint8_t *codes, const uint16_t *scales, size_t row, int cols, int j)
{
    const uint8_t byte = codes[row * (size_t)(cols / 2) + (size_t)(j / 2)];
    const int q = ((j & 1) ? (byte >> 4) : (byte & 15)) - 8;
    const double sc = bf16_bits_value(scales[row * (size_t)(cols / 128) + (size_t)(j / 128)]);
    return (double)round_bf16((double)q * sc);
}

typedef struct {
    const oracle_dims *dm;
    const uint16_t *x;                                       /* [T, d] bf16 bits              */
    const uint8_t *W1; const uint16_t *s1; const float *b1;  /* [E, d_ff, d/2], [E, d_ff, d/128] */
    const uint8_t *Wu; const uint16_t *su;
    const uint8_t *W2; const uint16_t *s2; const float *b2;  /* [E, d, d_ff/2], [E, d, d_ff/128] */
    const uint8_t *Wsg; const uint16_t *ssg; const uint8_t *Wsu; const uint16_t *ssu;
    const uint8_t *Wsd; const uint16_t *ssd;
} w4_experts;

/* One INT4 expert on token t (e == E: the shared expert); hbuf: d_ff doubles of scratch. */
static void expert_apply_w4_one(const w4_experts *w, int64_t t, int e, double *hbuf, double *out)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const uint8_t *Wa = shared ? w->Wsg : w->W1, *Wb = shared ? w->Wsu : w->Wu, *Wo = shared ? w->Wsd : w->W2;
    const uint16_t *sa = shared ? w->ssg : w->s1, *sb = shared ? w->ssu : w->su, *so = shared ? w->ssd : w->s2;
    const size_t eb = shared ? 0 : (size_t)e;
    const uint16_t *xr = w->x + (size_t)t * d;
    for (int j = 0; j < dff; ++j) {
        const size_t wr = eb * dff + j;
        double a = 0.0;
        for (int i = 0; i < d; ++i) a += w4_value(Wa, sa, wr, d, i) * bf16_bits_value(xr[i]);
        if (dm->act == 0) {
            if (!shared && w->b1) a += (double)w->b1[eb * dff + j];
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else {
            double u = 0.0;
            for (int i = 0; i < d; ++i) u += w4_value(Wb, sb, wr, d, i) * bf16_bits_value(xr[i]);
            hbuf[j] = a / (1.0 + exp(-a)) * u;
        }
    }
    for (int i = 0; i < d; ++i) {
        const size_t orow = eb * d + i;
        double o = 0.0;
        for (int j = 0; j < dff; ++j) o += w4_value(Wo, so, orow, dff, j) * hbuf[j];
        if (dm->act == 0 && !shared && w->b2) o += (double)w->b2[eb * d + i];
        out[i] = o;
    }
}

typedef struct {
    w4_experts w;
    const int32_t *token; const int32_t *expert; const double *scale; double *out;
} applyw4_ctx;

static void applyw4_range(void *vctx, int64_t lo, int64_t hi)
{
    applyw4_ctx *c = (applyw4_ctx *)vctx;
    const oracle_dims *dm = c->w.dm;
    const int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    const size_t hn = (size_t)(hmax > 0 ? hmax : 1);
    double *hbuf = (double *)malloc(sizeof(double) * hn);
    for (int64_t r = lo; r < hi; ++r) {
        double *o = c->out + (size_t)r * dm->d;
        expert_apply_w4_one(&c->w, c->token[r], c->expert[r], hbuf, o);
        const double sc = c->scale ? c->scale[r] : 1.0;
        for (int i = 0; i < dm->d; ++i) o[i] *= sc;
    }
    free(hbuf);
}

/* out[r,:] = scale[r] * Ew4_{expert[r]}(x[token[r],:]) for INT4 weight-only
 * experts (expert == E: the shared expert).  d, d_ff (and d_ff_shared) must
 * be multiples of 128; x is bf16 bits.                                       */
int oracle_expert_apply_w4(const oracle_dims *dm, int64_t nrows, const int32_t *token, const int32_t *expert,
                           const double *scale, const uint16_t *x,
                           const uint8_t *W1, const uint16_t *s1, const float *b1,
                           const uint8_t *Wu, const uint16_t *su,
                           const uint8_t *W2, const uint16_t *s2, const float *b2,
                           const uint8_t *Wsg, const uint16_t *ssg, const uint8_t *Wsu, const uint16_t *ssu,
                           const uint8_t *Wsd, const uint16_t *ssd, double *out)
{
    if (dm->d % 128 != 0 || dm->d_ff % 128 != 0 || (dm->d_ff_shared > 0 && dm->d_ff_shared % 128 != 0)) return 2;
    for (int64_t r = 0; r < nrows; ++r) {
        if (expert[r] < 0 || expert[r] > dm->E) return 1;
        if (expert[r] == dm->E && dm->d_ff_shared <= 0) return 1;
    }
    applyw4_ctx c = { { dm, x, W1, s1, b1, Wu, su, W2, s2, b2, Wsg, ssg, Wsu, ssu, Wsd, ssd },
                      token, expert, scale, out };
    parallel_for(nrows, dm->nthreads, applyw4_range, &c);
    return 0;
}

/* Value of every input of `rows` weight rows (the dequantized matrix, double). */
int oracle_w4_dequant(const uint8_t *codes, const uint16_t *scales, int64_t rows, int32_t cols, double *out)
{
    if (cols <= 0 || cols % 128 != 0) return 1;
    for (int64_t r = 0; r < rows; ++r)
        for (int j = 0; j < cols; ++j) out[r * cols + j] = w4_value(codes, scales, (size_t)r, cols, j);
    return 0;
}

/* ===========================================================================
 * Backward pass of the layer.
 *
 * The layer is trained ([RO] "The Fine-Tuning Router Challenge" and How It
 * Works 1: the router and experts learn from the task loss plus the
 * auxiliary balance loss).  For an upstream gradient dy [T, d] of the output
 * and an aux-loss weight alpha, this computes the gradient of
 *   ell = sum_t <dy_t, y_t> + alpha * L_aux,   L_aux = E sum_e f_e P_e
 * with respect to x, W_r, the logit offset beta, every routed expert's
 * weights and biases and the shared expert's weights.  It is the chain rule
 * applied to the forward definitions above, in double:
 *   - the expert selection (a sort of the keys) and the capacity ranks are
 *     piecewise constant: no gradient flows through which experts are chosen
 *     or dropped; f_e (counts) is constant in the same way, so L_aux is
 *     differentiated through P only ([RO] How It Works 1);
 *   - a kept slot s of token t with expert e adds g_s * E_e(x_t) to y_t, so
 *     dE_e = g_s dy_t and d g_s = <dy_t, E_e(x_t)>; a dropped slot adds
 *     nothing and its gate gets no gradient;
 *   - gate Jacobians: full-softmax gates g_s = p_{e_s}: dh = p (dp - <dp, p>)
 *     with dp_e the sum of dg over slots choosing e; renormalised softmax
 *     gates (a softmax over the selected logits): dh_sel = g (dg - <dg, g>);
 *     sigmoid gates g_s = s_{e_s} / S_sel: ds_sel = (dg - <dg, g>) / S_sel,
 *     dh = ds s (1 - s);
 *   - aux loss: dell / dpnorm_e(t) = alpha E f_e / T =: c_e; softmax pnorm = p
 *     gives dh += p (c - <c, p>); sigmoid pnorm = s / S_all gives
 *     ds = (c - <c, pnorm>) / S_all, dh += ds s (1 - s);
 *   - the selection bias never enters y or L_aux: no gradient;
 *   - GELU' (exact erf form) = Phi(a) + a phi(a); SiLU'(v) = sig(v) (1 + v (1 - sig(v))).
 * Weight gradients sum over tokens in ascending order; dx_t sums its slots in
 * slot order, then the shared expert, then the router term.
 * Outputs (double, any may be NULL except dx): dx [T,d], dWr [d,E], dbeta [E],
 * dW1 [E,d_ff,d], db1 [E,d_ff], dWu [E,d_ff,d], dW2 [E,d,d_ff], db2 [E,d],
 * dWsg [S,d], dWsu [S,d], dWsd [d,S].
 * ======================================================================== */
typedef struct {
    expert_weights w;
    const float *Wr;
    const int32_t *idx; const double *gate; const int32_t *row_of;
    const double *h; const double *pnorm; const double *cvec;   /* logits, pnorm, aux weights c_e */
    const double *dy;
    double *dx; double *dh;
    /* pass B */
    double *dW1, *db1, *dWu, *dW2, *db2, *dWsg, *dWsu, *dWsd;
} bwd_ctx;

static double gelu_grad(double a)
{
    return 0.5 * (1.0 + erf(a / sqrt(2.0))) + a * exp(-0.5 * a * a) / sqrt(2.0 * acos(-1.0));
}

/* Forward of expert e on token t keeping what the backward needs: pre-
 * activations a (GELU) or g and u (SwiGLU) in pre1 / pre2, the hidden h and
 * the output o.                                                            */
static void expert_fwd_keep(const expert_weights *w, int64_t t, int e, double *pre1, double *pre2, double *hbuf,
                            double *out)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d, dt = dm->xw_dtype;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const void *Wa = shared ? w->Wsg : w->W1;
    const void *Wb = shared ? w->Wsu : w->Wu;
    const void *Wo = shared ? w->Wsd : w->W2;
    const size_t eb = shared ? 0 : (size_t)e;
    for (int j = 0; j < dff; ++j) {
        double a = 0.0;
        for (int i = 0; i < d; ++i) a += wide(Wa, dt, (eb * dff + j) * d + i) * wide(w->x, dt, (size_t)t * d + i);
        if (dm->act == 0) {
            if (!shared && w->b1) a += (double)w->b1[eb * dff + j];
            pre1[j] = a;
            hbuf[j] = 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
        } else {
            double u = 0.0;
            for (int i = 0; i < d; ++i) u += wide(Wb, dt, (eb * dff + j) * d + i) * wide(w->x, dt, (size_t)t * d + i);
            pre1[j] = a;
            pre2[j] = u;
            hbuf[j] = a / (1.0 + exp(-a)) * u;
        }
    }
    for (int i = 0; i < d; ++i) {
        double o = 0.0;
        for (int j = 0; j < dff; ++j) o += wide(Wo, dt, (eb * d + i) * dff + j) * hbuf[j];
        if (dm->act == 0 && !shared && w->b2) o += (double)w->b2[eb * d + i];
        out[i] = o;
    }
}

/* Gradient of the expert's pre-activations from dz = dE_e/d(output):
 * dhid = Wo^T dz, then da (GELU) or dga, dua (SwiGLU) into d1 / d2.        */
static void expert_bwd_pre(const expert_weights *w, int e, const double *pre1, const double *pre2,
                           const double *dz, double *dhid, double *d1, double *d2)
{
    const oracle_dims *dm = w->dm;
    const int d = dm->d, dt = dm->xw_dtype;
    const int shared = (e == dm->E);
    const int dff = shared ? dm->d_ff_shared : dm->d_ff;
    const void *Wo = shared ? w->Wsd : w->W2;
    const size_t eb = shared ? 0 : (size_t)e;
    for (int j = 0; j < dff; ++j) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += wide(Wo, dt, (eb * d + i) * dff + j) * dz[i];
        dhid[j] = acc;
        if (dm->act == 0) {
            d1[j] = acc * gelu_grad(pre1[j]);
        } else {
            const double sg = 1.0 / (1.0 + exp(-pre1[j]));
            d1[j] = acc * pre2[j] * sg * (1.0 + pre1[j] * (1.0 - sg));
            d2[j] = acc * pre1[j] * sg;
        }
    }
}

static void bwd_token_range(void *vctx, int64_t lo, int64_t hi)
{
    bwd_ctx *c = (bwd_ctx *)vctx;
    const expert_weights *w = &c->w;
    const oracle_dims *dm = w->dm;
    const int d = dm->d, E = dm->E, k = dm->k, dt = dm->xw_dtype;
    const int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    const size_t hm = (size_t)(hmax > 0 ? hmax : 1);
    double *pre1 = (double *)malloc(sizeof(double) * hm), *pre2 = (double *)malloc(sizeof(double) * hm);
    double *hid = (double *)malloc(sizeof(double) * hm), *dhid = (double *)malloc(sizeof(double) * hm);
    double *d1 = (double *)malloc(sizeof(double) * hm), *d2 = (double *)malloc(sizeof(double) * hm);
    double *o = (double *)malloc(sizeof(double) * (size_t)d), *dz = (double *)malloc(sizeof(double) * (size_t)d);
    double *dg = (double *)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = lo; t < hi; ++t) {
        const double *dyt = c->dy + (size_t)t * d;
        double *dxt = c->dx + (size_t)t * d;
        for (int i = 0; i < d; ++i) dxt[i] = 0.0;
        /* routed slots (slot order), then the shared expert */
        for (int s = 0; s <= k; ++s) {
            int e;
            double g;
            if (s < k) {
                dg[s] = 0.0;
                if (c->row_of[t * k + s] < 0) continue;
                e = c->idx[t * k + s];
                g = c->gate[t * k + s];
            } else {
                if (dm->d_ff_shared <= 0) break;
                e = E;
                g = 1.0;
            }
            const int dff = (e == E) ? dm->d_ff_shared : dm->d_ff;
            expert_fwd_keep(w, t, e, pre1, pre2, hid, o);
            if (s < k) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += dyt[i] * o[i];
                dg[s] = acc;
            }
            for (int i = 0; i < d; ++i) dz[i] = g * dyt[i];
            expert_bwd_pre(w, e, pre1, pre2, dz, dhid, d1, d2);
            const void *Wa = (e == E) ? w->Wsg : w->W1;
            const void *Wb = (e == E) ? w->Wsu : w->Wu;
            const size_t eb = (e == E) ? 0 : (size_t)e;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dff; ++j) {
                    acc += wide(Wa, dt, (eb * dff + j) * d + i) * d1[j];
                    if (dm->act == 1) acc += wide(Wb, dt, (eb * dff + j) * d + i) * d2[j];
                }
                dxt[i] += acc;
            }
        }
        /* router: gates, then the aux loss, into dh_t */
        const double *h = c->h + (size_t)t * E;
        const double *pn = c->pnorm + (size_t)t * E;
        double *dh = c->dh + (size_t)t * E;
        for (int e = 0; e < E; ++e) dh[e] = 0.0;
        if (dm->score == 0) {
            /* p_e from the logits (pnorm is p for softmax scores) */
            if (dm->renorm == 0) {
                double dot = 0.0;
                for (int s = 0; s < k; ++s) dot += pn[c->idx[t * k + s]] * dg[s];
                for (int s = 0; s < k; ++s) {
                    const int e = c->idx[t * k + s];
                    dh[e] += pn[e] * dg[s];
                }
                for (int e = 0; e < E; ++e) dh[e] -= pn[e] * dot;
            } else {
                double dot = 0.0;
                for (int s = 0; s < k; ++s) dot += c->gate[t * k + s] * dg[s];
                for (int s = 0; s < k; ++s) dh[c->idx[t * k + s]] += c->gate[t * k + s] * (dg[s] - dot);
            }
            double cp = 0.0;
            for (int e = 0; e < E; ++e) cp += c->cvec[e] * pn[e];
            for (int e = 0; e < E; ++e) dh[e] += pn[e] * (c->cvec[e] - cp);
        } else {
            double ssel = 0.0, sall = 0.0, dot = 0.0;
            for (int s = 0; s < k; ++s) ssel += 1.0 / (1.0 + exp(-h[c->idx[t * k + s]]));
            for (int e = 0; e < E; ++e) sall += 1.0 / (1.0 + exp(-h[e]));
            for (int s = 0; s < k; ++s) dot += c->gate[t * k + s] * dg[s];
            for (int s = 0; s < k; ++s) {
                const int e = c->idx[t * k + s];
                const double se = 1.0 / (1.0 + exp(-h[e]));
                dh[e] += (dg[s] - dot) / ssel * se * (1.0 - se);
            }
            double cq = 0.0;
            for (int e = 0; e < E; ++e) cq += c->cvec[e] * pn[e];
            for (int e = 0; e < E; ++e) {
                const double se = 1.0 / (1.0 + exp(-h[e]));
                dh[e] += (c->cvec[e] - cq) / sall * se * (1.0 - se);
            }
        }
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int e = 0; e < E; ++e) acc += (double)c->Wr[(size_t)j * E + e] * dh[e];
            dxt[j] += acc;
        }
    }
    free(pre1); free(pre2); free(hid); free(dhid); free(d1); free(d2); free(o); free(dz); free(dg);
}

/* Pass B: weight gradients of expert e (e == E: the shared expert), tokens in
 * ascending order, one expert per worker.                                   */
static void bwd_expert_range(void *vctx, int64_t lo, int64_t hi)
{
    bwd_ctx *c = (bwd_ctx *)vctx;
    const expert_weights *w = &c->w;
    const oracle_dims *dm = w->dm;
    const int d = dm->d, E = dm->E, k = dm->k, dt = dm->xw_dtype;
    const int hmax = dm->d_ff > dm->d_ff_shared ? dm->d_ff : dm->d_ff_shared;
    const size_t hm = (size_t)(hmax > 0 ? hmax : 1);
    double *pre1 = (double *)malloc(sizeof(double) * hm), *pre2 = (double *)malloc(sizeof(double) * hm);
    double *hid = (double *)malloc(sizeof(double) * hm), *dhid = (double *)malloc(sizeof(double) * hm);
    double *d1 = (double *)malloc(sizeof(double) * hm), *d2 = (double *)malloc(sizeof(double) * hm);
    double *o = (double *)malloc(sizeof(double) * (size_t)d), *dz = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t e = lo; e < hi; ++e) {
        const int sh = (e == E);
        const int dff = sh ? dm->d_ff_shared : dm->d_ff;
        double *gA = sh ? c->dWsg : (c->dW1 ? c->dW1 + (size_t)e * dff * d : NULL);
        double *gB = sh ? c->dWsu : (c->dWu ? c->dWu + (size_t)e * dff * d : NULL);
        double *gO = sh ? c->dWsd : (c->dW2 ? c->dW2 + (size_t)e * d * dff : NULL);
        double *gb1 = (!sh && c->db1) ? c->db1 + (size_t)e * dff : NULL;
        double *gb2 = (!sh && c->db2) ? c->db2 + (size_t)e * d : NULL;
        if (gA) memset(gA, 0, sizeof(double) * (size_t)dff * d);
        if (gB) memset(gB, 0, sizeof(double) * (size_t)dff * d);
        if (gO) memset(gO, 0, sizeof(double) * (size_t)d * dff);
        if (gb1) memset(gb1, 0, sizeof(double) * (size_t)dff);
        if (gb2) memset(gb2, 0, sizeof(double) * (size_t)d);
        for (int64_t t = 0; t < dm->T; ++t) {
            double g = 1.0;
            if (!sh) {
                int s = 0;
                for (; s < k; ++s)
                    if (c->idx[t * k + s] == (int)e && c->row_of[t * k + s] >= 0) break;
                if (s == k) continue;
                g = c->gate[t * k + s];
            }
            expert_fwd_keep(w, t, (int)e, pre1, pre2, hid, o);
            const double *dyt = c->dy + (size_t)t * d;
            for (int i = 0; i < d; ++i) dz[i] = g * dyt[i];
            expert_bwd_pre(w, (int)e, pre1, pre2, dz, dhid, d1, d2);
            for (int i = 0; i < d; ++i) {
                if (gO) for (int j = 0; j < dff; ++j) gO[(size_t)i * dff + j] += dz[i] * hid[j];
                if (gb2 && dm->act == 0) gb2[i] += dz[i];
            }
            for (int j = 0; j < dff; ++j) {
                for (int i = 0; i < d; ++i) {
                    const double xi = wide(w->x, dt, (size_t)t * d + i);
                    if (gA) gA[(size_t)j * d + i] += d1[j] * xi;
                    if (gB && dm->act == 1) gB[(size_t)j * d + i] += d2[j] * xi;
                }
                if (gb1 && dm->act == 0) gb1[j] += d1[j];
            }
        }
    }
    free(pre1); free(pre2); free(hid); free(dhid); free(d1); free(d2); free(o); free(dz);
}

typedef struct { const oracle_dims *dm; const void *x; const double *dh; double *dWr; } dwr_ctx;

static void bwd_router_range(void *vctx, int64_t lo, int64_t hi)
{
    dwr_ctx *c = (dwr_ctx *)vctx;
    const oracle_dims *dm = c->dm;
    const int E = dm->E, d = dm->d;
    for (int64_t j = lo; j < hi; ++j)
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t t = 0; t < dm->T; ++t) acc += wide(c->x, dm->xw_dtype, (size_t)t * d + j) * c->dh[t * E + e];
            c->dWr[(size_t)j * E + e] = acc;
        }
}

int oracle_layer_backward(const oracle_dims *dm, const void *x, const float *Wr, const float *logit_bias,
                          const float *sel_bias, const void *W1, const float *b1, const void *Wu, const void *W2,
                          const float *b2, const void *Wsg, const void *Wsu, const void *Wsd,
                          const double *dy, double alpha,
                          double *dx, double *dWr, double *dbeta, double *dW1, double *db1, double *dWu,
                          double *dW2, double *db2, double *dWsg, double *dWsu, double *dWsd)
{
    if (!dm || !dx || dm->T < 0 || dm->k < 1 || dm->k > dm->E) return 1;
    const int64_t T = dm->T;
    const int E = dm->E, k = dm->k;
    const size_t tk = (size_t)(T * k > 0 ? T * k : 1);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * tk);
    double *gate = (double *)malloc(sizeof(double) * tk);
    double *h = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * E);
    double *pn = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * E);
    double *dh = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * E);
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *kept = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offs = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *row_of = (int32_t *)malloc(sizeof(int32_t) * tk);
    double *cvec = (double *)malloc(sizeof(double) * (size_t)E);
    int rc = oracle_route(dm, T, NULL, x, Wr, logit_bias, sel_bias, idx, gate, h, pn, NULL, NULL);
    if (!rc) rc = oracle_dispatch(dm, idx, counts, kept, offs, row_of, NULL, NULL);
    if (!rc) {
        for (int e = 0; e < E; ++e)
            cvec[e] = T > 0 ? alpha * (double)E * ((double)counts[e] / ((double)T * (double)k)) / (double)T : 0.0;
        bwd_ctx c = { { dm, x, W1, b1, Wu, W2, b2, Wsg, Wsu, Wsd }, Wr, idx, gate, row_of, h, pn, cvec, dy, dx, dh,
                      dW1, db1, dWu, dW2, db2, dWsg, dWsu, dWsd };
        parallel_for(T, dm->nthreads, bwd_token_range, &c);
        parallel_for(E + (dm->d_ff_shared > 0 ? 1 : 0), dm->nthreads, bwd_expert_range, &c);
        if (dWr) {
            dwr_ctx r = { dm, x, dh, dWr };
            parallel_for(dm->d, dm->nthreads, bwd_router_range, &r);
        }
        if (dbeta)
            for (int e = 0; e < E; ++e) {
                double acc = 0.0;
                for (int64_t t = 0; t < T; ++t) acc += dh[t * E + e];
                dbeta[e] = acc;
            }
    }
    free(idx); free(gate); free(h); free(pn); free(dh); free(counts); free(kept); free(offs); free(row_of); free(cvec);
    return rc;
}
