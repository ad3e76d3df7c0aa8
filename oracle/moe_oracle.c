/*
 * moe_oracle.c -- plain, slow, single-threaded fp64 CPU oracle of the
 * sparse Mixture-of-Experts block forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes is the definition printed in the article
 * "Qwen3MoeSparseMoeBlock performance optimisation in practice" (parallelising
 * a sparse mixture-of-experts system), section 1, the forward() listing and
 * the four-stage workflow above it:
 *   stage 1  router logits = x . W_router (+ per-expert bias), softmax over E
 *   stage 2  top-k experts per token by probability; the listing keeps the
 *            top-k probabilities as routing weights and does NOT renormalise
 *   stage 3  each selected expert processes its tokens
 *   stage 4  the expert outputs are summed per token, weighted by the routing
 *            weights (the prose of stage 4; the listing's index_add_ omits the
 *            multiply, the prose requires it)
 * The per-expert bias follows the gating formula G(x) = Softmax(W_g x + b_g)
 * of the Hunyuan-Large overview page, section 2.1.  The expert MLP is the
 * SwiGLU form down(silu(gate(x)) * up(x)) with silu(z) = z / (1 + exp(-z));
 * the routing weight multiplies the expert's output (after the down
 * projection).
 *
 * Readings where the pages are silent:
 *   - ties in probability: the lower expert index ranks first; the k slots of
 *     a token are ordered by descending probability;
 *   - the order of tokens inside one expert group: ascending flat assignment
 *     index t*k + j (a stable counting sort);
 *   - every sum runs in ascending index order, in fp64, with no intermediate
 *     rounding; bf16 inputs are widened exactly.
 *
 * Layouts (row-major, contiguous; bf16 given as raw uint16 bit patterns):
 *   x [T][d], W_router [d][E], bias [E] (fp32, may be NULL),
 *   W_gate [E][d][f], W_up [E][d][f], W_down [E][f][d].
 *
 * Optional variants, each off the article's path and pinned like the rest:
 * oracle_renormalize (renormalised top-k weights), oracle_shared_rows
 * (shared experts), oracle_round_tokens and oracle_masked_rows (token
 * rounding), and oracle_backward (the gradient of the block, for the
 * backward that recomputes the expert activations).
 *
 * Parity status: every function here is pinned by CPU tests against
 * independent computations (brute force, library routines, invariants and
 * special cases); nothing is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

/* Exact widening of one bf16 bit pattern: bf16 is the top half of an fp32. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One (probability, expert index) pair, for the top-k sort. */
typedef struct {
    double p;
    int32_t e;
} ranked_t;

/* Descending probability; equal probabilities: lower expert index first. */
static int by_prob_desc_then_index(const void* a, const void* b)
{
    const ranked_t* ra = (const ranked_t*)a;
    const ranked_t* rb = (const ranked_t*)b;
    if (ra->p > rb->p) return -1;
    if (ra->p < rb->p) return 1;
    return (ra->e > rb->e) - (ra->e < rb->e);
}

/*
 * Stages 1 and 2 for every token.
 *   logits_out [T][E]  (may be NULL)  x . W_router + bias, fp64
 *   probs_out  [T][E]  (may be NULL)  softmax over the E experts
 *   ids        [T][k]                 selected experts, descending probability
 *   weights    [T][k]                 their probabilities, not renormalised
 */
int oracle_route(const uint16_t* x, const uint16_t* w_router, const float* bias,
                 int64_t T, int64_t d, int64_t E, int64_t k,
                 double* logits_out, double* probs_out,
                 int32_t* ids, double* weights)
{
    if (!x || !w_router || !ids || !weights || T < 0 || d < 1 || E < 1 || k < 1 || k > E)
        return ORACLE_BAD_ARG;
    double* logit = (double*)malloc(sizeof(double) * E);
    double* prob = (double*)malloc(sizeof(double) * E);
    ranked_t* ranked = (ranked_t*)malloc(sizeof(ranked_t) * E);
    if (!logit || !prob || !ranked) {
        free(logit); free(prob); free(ranked);
        return ORACLE_NO_MEMORY;
    }
    for (int64_t t = 0; t < T; ++t) {
        /* router logits: sum over the hidden index i, ascending */
        for (int64_t e = 0; e < E; ++e) logit[e] = 0.0;
        for (int64_t i = 0; i < d; ++i) {
            double xi = bf16_to_double(x[t * d + i]);
            const uint16_t* wrow = w_router + i * E;
            for (int64_t e = 0; e < E; ++e) logit[e] += xi * bf16_to_double(wrow[e]);
        }
        if (bias)
            for (int64_t e = 0; e < E; ++e) logit[e] += (double)bias[e];

        /* softmax over experts, shifted by the maximum logit */
        double m = logit[0];
        for (int64_t e = 1; e < E; ++e) if (logit[e] > m) m = logit[e];
        double s = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            prob[e] = exp(logit[e] - m);
            s += prob[e];
        }
        for (int64_t e = 0; e < E; ++e) prob[e] /= s;

        /* top-k: sort all experts by (probability desc, index asc) */
        for (int64_t e = 0; e < E; ++e) {
            ranked[e].p = prob[e];
            ranked[e].e = (int32_t)e;
        }
        qsort(ranked, (size_t)E, sizeof(ranked_t), by_prob_desc_then_index);
        for (int64_t j = 0; j < k; ++j) {
            ids[t * k + j] = ranked[j].e;
            weights[t * k + j] = ranked[j].p;
        }
        if (logits_out) memcpy(logits_out + t * E, logit, sizeof(double) * E);
        if (probs_out) memcpy(probs_out + t * E, prob, sizeof(double) * E);
    }
    free(logit); free(prob); free(ranked);
    return ORACLE_OK;
}

/*
 * Optional variant (not in the article's listing, which keeps the top-k
 * probabilities as they are): renormalised routing weights,
 *   w[t][j] <- w[t][j] / sum_{m = 0..k-1} w[t][m]   (sum over m ascending),
 * so that each token's k weights sum to one.  In place.
 */
int oracle_renormalize(double* weights, int64_t T, int64_t k)
{
    if (!weights || T < 0 || k < 1) return ORACLE_BAD_ARG;
    for (int64_t t = 0; t < T; ++t) {
        double s = 0.0;
        for (int64_t j = 0; j < k; ++j) s += weights[t * k + j];
        for (int64_t j = 0; j < k; ++j) weights[t * k + j] /= s;
    }
    return ORACLE_OK;
}

/*
 * Grouping of the T*k assignments by expert (the "token reordering" step of
 * the article's section 2.2: sort_tokens_by_expert, then gather).
 *   counts  [E]    assignments per expert
 *   offsets [E+1]  exclusive prefix sum of counts; offsets[E] = T*k
 *   perm    [T*k]  perm[pos] = t*k + j of the assignment at grouped row pos
 *   inv     [T*k]  inv[t*k + j] = pos
 * Inside one expert group the assignments keep ascending flat order.
 */
int oracle_permute(const int32_t* ids, int64_t T, int64_t E, int64_t k,
                   int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv)
{
    if (!ids || !counts || !offsets || !perm || !inv || T < 0 || E < 1 || k < 1)
        return ORACLE_BAD_ARG;
    const int64_t n = T * k;
    for (int64_t a = 0; a < n; ++a)
        if (ids[a] < 0 || ids[a] >= E) return ORACLE_BAD_ARG;
    for (int64_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t a = 0; a < n; ++a) counts[ids[a]] += 1;
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* next = (int32_t*)malloc(sizeof(int32_t) * E);
    if (!next) return ORACLE_NO_MEMORY;
    for (int64_t e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t a = 0; a < n; ++a) {
        int32_t pos = next[ids[a]]++;
        perm[pos] = (int32_t)a;
        inv[a] = pos;
    }
    free(next);
    return ORACLE_OK;
}

/*
 * One expert's SwiGLU MLP on one token row (stage 3):
 *   g = x . W_gate[e],  u = x . W_up[e]          (sums over i ascending)
 *   h = silu(g) * u,    silu(z) = z / (1 + exp(-z))
 *   o = h . W_down[e]                            (sum over n ascending)
 */
static void expert_swiglu(const double* xrow, const uint16_t* wg, const uint16_t* wu,
                          const uint16_t* wd, int64_t d, int64_t f,
                          double* g, double* u, double* h, double* o)
{
    for (int64_t n = 0; n < f; ++n) { g[n] = 0.0; u[n] = 0.0; }
    for (int64_t i = 0; i < d; ++i) {
        const double xi = xrow[i];
        const uint16_t* grow = wg + i * f;
        const uint16_t* urow = wu + i * f;
        for (int64_t n = 0; n < f; ++n) {
            g[n] += xi * bf16_to_double(grow[n]);
            u[n] += xi * bf16_to_double(urow[n]);
        }
    }
    for (int64_t n = 0; n < f; ++n) h[n] = g[n] / (1.0 + exp(-g[n])) * u[n];
    for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
    for (int64_t n = 0; n < f; ++n) {
        const double hn = h[n];
        const uint16_t* drow = wd + n * d;
        for (int64_t c = 0; c < d; ++c) o[c] += hn * bf16_to_double(drow[c]);
    }
}

/*
 * Stages 3 and 4 for a chosen list of tokens, given the routing from
 * oracle_route:
 *   out   [n_rows][d]     out[r] = sum_{j ascending} w[t][j] * expert_{ids[t][j]}(x[t]),
 *                         t = rows[r]
 *   y_out [n_rows][k][d]  (may be NULL)  the weighted per-slot expert outputs
 *   h_out [n_rows][k][f]  (may be NULL)  silu(g) * u per slot
 * Every output row depends only on its own token, so any subset of tokens
 * gives exactly the rows a full evaluation would.
 */
int oracle_expert_rows(const uint16_t* x, const uint16_t* w_gate, const uint16_t* w_up,
                       const uint16_t* w_down, int64_t T, int64_t d, int64_t E, int64_t k,
                       int64_t f, const int32_t* ids, const double* weights,
                       int64_t n_rows, const int64_t* rows,
                       double* out, double* y_out, double* h_out)
{
    if (!x || !w_gate || !w_up || !w_down || !ids || !weights || !rows || !out ||
        T < 0 || d < 1 || E < 1 || k < 1 || f < 1 || n_rows < 0)
        return ORACLE_BAD_ARG;
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* g = (double*)malloc(sizeof(double) * f);
    double* u = (double*)malloc(sizeof(double) * f);
    double* h = (double*)malloc(sizeof(double) * f);
    double* o = (double*)malloc(sizeof(double) * d);
    if (!xrow || !g || !u || !h || !o) {
        free(xrow); free(g); free(u); free(h); free(o);
        return ORACLE_NO_MEMORY;
    }
    int status = ORACLE_OK;
    for (int64_t r = 0; r < n_rows && status == ORACLE_OK; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) { status = ORACLE_BAD_ARG; break; }
        for (int64_t i = 0; i < d; ++i) xrow[i] = bf16_to_double(x[t * d + i]);
        double* orow = out + r * d;
        for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            const int32_t e = ids[t * k + j];
            if (e < 0 || e >= E) { status = ORACLE_BAD_ARG; break; }
            expert_swiglu(xrow, w_gate + (int64_t)e * d * f, w_up + (int64_t)e * d * f,
                          w_down + (int64_t)e * f * d, d, f, g, u, h, o);
            const double wj = weights[t * k + j];
            for (int64_t c = 0; c < d; ++c) {
                const double yc = wj * o[c];
                orow[c] += yc;
                if (y_out) y_out[(r * k + j) * d + c] = yc;
            }
            if (h_out) memcpy(h_out + (r * k + j) * f, h, sizeof(double) * f);
        }
    }
    free(xrow); free(g); free(u); free(h); free(o);
    return status;
}

/*
 * Optional variant: shared experts, SwiGLU experts that every token passes
 * through with weight one, on top of its k routed experts (the "shared
 * expert" routing of the Hunyuan-Large overview page, section 2.1; the page
 * gives no formula, so the reading is: out[t] += sum_s shared_s(x[t])).
 *   w_gate_s, w_up_s [n_s][d][f_s], w_down_s [n_s][f_s][d]
 *   out [n_rows][d]  in/out: out[r] += sum_{s ascending} shared_s(x[rows[r]])
 *                    (call after oracle_expert_rows on the same rows)
 */
int oracle_shared_rows(const uint16_t* x, const uint16_t* w_gate_s, const uint16_t* w_up_s,
                       const uint16_t* w_down_s, int64_t T, int64_t d, int64_t n_s, int64_t f_s,
                       int64_t n_rows, const int64_t* rows, double* out)
{
    if (!x || !w_gate_s || !w_up_s || !w_down_s || !rows || !out || T < 0 || d < 1 || n_s < 1 ||
        f_s < 1 || n_rows < 0)
        return ORACLE_BAD_ARG;
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* g = (double*)malloc(sizeof(double) * f_s);
    double* u = (double*)malloc(sizeof(double) * f_s);
    double* h = (double*)malloc(sizeof(double) * f_s);
    double* o = (double*)malloc(sizeof(double) * d);
    if (!xrow || !g || !u || !h || !o) {
        free(xrow); free(g); free(u); free(h); free(o);
        return ORACLE_NO_MEMORY;
    }
    int status = ORACLE_OK;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) { status = ORACLE_BAD_ARG; break; }
        for (int64_t i = 0; i < d; ++i) xrow[i] = bf16_to_double(x[t * d + i]);
        for (int64_t sidx = 0; sidx < n_s; ++sidx) {
            expert_swiglu(xrow, w_gate_s + sidx * d * f_s, w_up_s + sidx * d * f_s,
                          w_down_s + sidx * f_s * d, d, f_s, g, u, h, o);
            for (int64_t c = 0; c < d; ++c) out[r * d + c] += o[c];
        }
    }
    free(xrow); free(g); free(u); free(h); free(o);
    return status;
}

/*
 * Optional variant: token rounding (the "token rounding" scheduling of the
 * SonicMoE comparison page, core difference 3: adjust the number of tokens
 * each expert receives so that the grouped GEMM needs no tile padding).  The
 * page's pseudocode is garbled; the reading implemented here, per expert e
 * and independently of the other experts, starting from the top-k routing:
 *   c = number of tokens routed to e, r = c mod R (R = the tile rows);
 *   r == 0        : unchanged;
 *   2 r <= R      : drop the r routed tokens with the smallest p[t][e]
 *                   (equal p: the larger token index is dropped first);
 *   2 r >  R      : add the a = R - r unrouted tokens with the largest
 *                   p[t][e] (equal p: the smaller token index first), if
 *                   T - c >= a; otherwise drop r as above.
 * Every count becomes a multiple of R.  A token's weight for each expert it
 * keeps or gains is its softmax probability p[t][e]; a token may end with
 * fewer or more than k experts.
 *   probs [T][E] fp64 (oracle_route's probs_out), ids [T][k]
 *   mask_out [T][E] (1: token t goes to expert e after rounding), counts_out [E]
 */
typedef struct {
    double p;
    int64_t t;
} cand_t;

/* ascending p; equal p: larger t first (the order in which tokens are dropped) */
static int drop_order(const void* a, const void* b)
{
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->p < y->p) return -1;
    if (x->p > y->p) return 1;
    return (x->t < y->t) - (x->t > y->t);
}

/* descending p; equal p: smaller t first (the order in which tokens are added) */
static int add_order(const void* a, const void* b)
{
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->p > y->p) return -1;
    if (x->p < y->p) return 1;
    return (x->t > y->t) - (x->t < y->t);
}

int oracle_round_tokens(const double* probs, const int32_t* ids, int64_t T, int64_t E, int64_t k, int64_t R,
                        uint8_t* mask_out, int32_t* counts_out)
{
    if (!probs || !ids || !mask_out || !counts_out || T < 0 || E < 1 || k < 1 || k > E || R < 1)
        return ORACLE_BAD_ARG;
    memset(mask_out, 0, (size_t)(T * E));
    for (int64_t a = 0; a < T * k; ++a) {
        const int32_t e = ids[a];
        if (e < 0 || e >= E) return ORACLE_BAD_ARG;
        mask_out[(a / k) * E + e] = 1;
    }
    cand_t* in = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T > 0 ? T : 1));
    cand_t* out = (cand_t*)malloc(sizeof(cand_t) * (size_t)(T > 0 ? T : 1));
    if (!in || !out) {
        free(in); free(out);
        return ORACLE_NO_MEMORY;
    }
    for (int64_t e = 0; e < E; ++e) {
        int64_t n_in = 0, n_out = 0;
        for (int64_t t = 0; t < T; ++t) {
            cand_t cd = {probs[t * E + e], t};
            if (mask_out[t * E + e]) in[n_in++] = cd; else out[n_out++] = cd;
        }
        const int64_t r = n_in % R;
        int64_t count = n_in;
        if (r != 0) {
            const int64_t add = R - r;
            if (2 * r > R && n_out >= add) {
                qsort(out, (size_t)n_out, sizeof(cand_t), add_order);
                for (int64_t i = 0; i < add; ++i) mask_out[out[i].t * E + e] = 1;
                count += add;
            } else {
                qsort(in, (size_t)n_in, sizeof(cand_t), drop_order);
                for (int64_t i = 0; i < r; ++i) mask_out[in[i].t * E + e] = 0;
                count -= r;
            }
        }
        counts_out[e] = (int32_t)count;
    }
    free(in); free(out);
    return ORACLE_OK;
}

/*
 * Stages 3 and 4 for a routing given as a mask (token rounding):
 *   out[r] = sum_{e ascending, mask[t][e] = 1} probs[t][e] * expert_e(x[t]), t = rows[r].
 */
int oracle_masked_rows(const uint16_t* x, const uint16_t* w_gate, const uint16_t* w_up,
                       const uint16_t* w_down, int64_t T, int64_t d, int64_t E, int64_t f,
                       const uint8_t* mask, const double* probs, int64_t n_rows, const int64_t* rows,
                       double* out)
{
    if (!x || !w_gate || !w_up || !w_down || !mask || !probs || !rows || !out || T < 0 || d < 1 ||
        E < 1 || f < 1 || n_rows < 0)
        return ORACLE_BAD_ARG;
    double* xrow = (double*)malloc(sizeof(double) * d);
    double* g = (double*)malloc(sizeof(double) * f);
    double* u = (double*)malloc(sizeof(double) * f);
    double* h = (double*)malloc(sizeof(double) * f);
    double* o = (double*)malloc(sizeof(double) * d);
    if (!xrow || !g || !u || !h || !o) {
        free(xrow); free(g); free(u); free(h); free(o);
        return ORACLE_NO_MEMORY;
    }
    int status = ORACLE_OK;
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) { status = ORACLE_BAD_ARG; break; }
        for (int64_t i = 0; i < d; ++i) xrow[i] = bf16_to_double(x[t * d + i]);
        double* orow = out + r * d;
        for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
        for (int64_t e = 0; e < E; ++e) {
            if (!mask[t * E + e]) continue;
            expert_swiglu(xrow, w_gate + e * d * f, w_up + e * d * f, w_down + e * f * d, d, f, g, u, h, o);
            const double we = probs[t * E + e];
            for (int64_t c = 0; c < d; ++c) orow[c] += we * o[c];
        }
    }
    free(xrow); free(g); free(u); free(h); free(o);
    return status;
}

/*
 * Backward of the block (the next row after the forward): the exact gradient
 * of L = sum_t sum_c dout[t][c] * out[t][c] with respect to x, W_router, the
 * router bias and the three expert weight tensors.  The SonicMoE comparison
 * page, section "core differences", item 1 (memory management), stores only
 * the gating outputs and the final expert outputs for the backward and
 * recomputes the rest; that changes what a GPU keeps, not the gradient, so
 * this oracle recomputes everything from the inputs, like the forward.
 *
 * For token t with routing (ids, w) from oracle_route (plus
 * oracle_renormalize when renormalize != 0), for each slot j, e = ids[t][j]:
 *   g, u, h = silu(g) * u, z = h . W_down[e]          (as the forward)
 *   dw_j     = dout[t] . z                            (gradient of the weight)
 *   dz       = w_j * dout[t]
 *   dW_down[e][n][c] += h[n] * dz[c]
 *   dh[n]    = sum_c dz[c] * W_down[e][n][c]
 *   du[n]    = dh[n] * silu(g[n])
 *   dg[n]    = dh[n] * u[n] * s(g[n]) * (1 + g[n] * (1 - s(g[n]))),  s = 1/(1+e^-x)
 *              (the derivative of silu(z) = z * s(z))
 *   dW_gate[e][i][n] += x[t][i] * dg[n],  dW_up[e][i][n] += x[t][i] * du[n]
 *   dx[t][i] += sum_n dg[n] * W_gate[e][i][n] + du[n] * W_up[e][i][n]
 * Router (the top-k choice itself is piecewise constant and passes no
 * gradient): with p the softmax of the logits,
 *   dp[e]      = dw_j for e = ids[t][j], 0 for the other experts
 *                (renormalised weights w_j = p_j / S, S = sum_m p_m over the
 *                 slots: dp[ids[t][m]] = (dw_m - sum_j dw_j * w_j) / S)
 *   dlogit[e]  = p[e] * (dp[e] - sum_i p[i] * dp[i])   (softmax Jacobian)
 *   dW_router[i][e] += x[t][i] * dlogit[e],  dbias[e] += dlogit[e]
 *   dx[t][i]  += sum_e dlogit[e] * W_router[i][e]
 * Every sum runs in ascending index order in fp64; tokens accumulate into
 * the weight gradients in ascending t, slots in ascending j.
 *
 * Outputs (fp64, overwritten): dx [T][d], dw_router [d][E], dbias [E],
 * dw_gate [E][d][f], dw_up [E][d][f], dw_down [E][f][d].  dout is [T][d].
 */
int oracle_backward(const uint16_t* x, const uint16_t* w_router, const float* bias,
                    const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                    int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int renormalize,
                    const double* dout, double* dx, double* dw_router, double* dbias,
                    double* dw_gate, double* dw_up, double* dw_down)
{
    if (!x || !w_router || !w_gate || !w_up || !w_down || !dout || !dx || !dw_router || !dbias ||
        !dw_gate || !dw_up || !dw_down || T < 0 || d < 1 || E < 1 || k < 1 || k > E || f < 1)
        return ORACLE_BAD_ARG;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * k + 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(T * k + 1));
    double* probs = (double*)malloc(sizeof(double) * (size_t)(T * E + 1));
    double* xrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* g = (double*)malloc(sizeof(double) * (size_t)f);
    double* u = (double*)malloc(sizeof(double) * (size_t)f);
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    double* z = (double*)malloc(sizeof(double) * (size_t)d);
    double* dz = (double*)malloc(sizeof(double) * (size_t)d);
    double* dh = (double*)malloc(sizeof(double) * (size_t)f);
    double* dg = (double*)malloc(sizeof(double) * (size_t)f);
    double* du = (double*)malloc(sizeof(double) * (size_t)f);
    double* dwj = (double*)malloc(sizeof(double) * (size_t)k);
    double* dp = (double*)malloc(sizeof(double) * (size_t)E);
    double* dl = (double*)malloc(sizeof(double) * (size_t)E);
    int rc = ORACLE_NO_MEMORY;
    if (!ids || !w || !probs || !xrow || !g || !u || !h || !z || !dz || !dh || !dg || !du || !dwj || !dp || !dl)
        goto done;
    rc = oracle_route(x, w_router, bias, T, d, E, k, NULL, probs, ids, w);
    if (rc != ORACLE_OK) goto done;
    if (renormalize) {
        rc = oracle_renormalize(w, T, k);
        if (rc != ORACLE_OK) goto done;
    }
    memset(dx, 0, sizeof(double) * (size_t)(T * d));
    memset(dw_router, 0, sizeof(double) * (size_t)(d * E));
    memset(dbias, 0, sizeof(double) * (size_t)E);
    memset(dw_gate, 0, sizeof(double) * (size_t)(E * d * f));
    memset(dw_up, 0, sizeof(double) * (size_t)(E * d * f));
    memset(dw_down, 0, sizeof(double) * (size_t)(E * f * d));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < d; ++i) xrow[i] = bf16_to_double(x[t * d + i]);
        const double* drow_out = dout + t * d;
        for (int64_t j = 0; j < k; ++j) {
            const int64_t e = ids[t * k + j];
            const double wj = w[t * k + j];
            const uint16_t* wg = w_gate + e * d * f;
            const uint16_t* wu = w_up + e * d * f;
            const uint16_t* wd = w_down + e * f * d;
            expert_swiglu(xrow, wg, wu, wd, d, f, g, u, h, z);
            double s = 0.0;
            for (int64_t c = 0; c < d; ++c) s += drow_out[c] * z[c];
            dwj[j] = s;
            for (int64_t c = 0; c < d; ++c) dz[c] = wj * drow_out[c];
            double* gdown = dw_down + e * f * d;
            for (int64_t n = 0; n < f; ++n) {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) {
                    gdown[n * d + c] += h[n] * dz[c];
                    acc += dz[c] * bf16_to_double(wd[n * d + c]);
                }
                dh[n] = acc;
            }
            for (int64_t n = 0; n < f; ++n) {
                const double sg = 1.0 / (1.0 + exp(-g[n]));
                du[n] = dh[n] * (g[n] * sg);
                dg[n] = dh[n] * u[n] * sg * (1.0 + g[n] * (1.0 - sg));
            }
            double* ggate = dw_gate + e * d * f;
            double* gup = dw_up + e * d * f;
            for (int64_t i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int64_t n = 0; n < f; ++n) {
                    ggate[i * f + n] += xrow[i] * dg[n];
                    gup[i * f + n] += xrow[i] * du[n];
                    acc += dg[n] * bf16_to_double(wg[i * f + n]) + du[n] * bf16_to_double(wu[i * f + n]);
                }
                dx[t * d + i] += acc;
            }
        }
        /* router: routing-weight gradients -> probabilities -> logits */
        for (int64_t e = 0; e < E; ++e) dp[e] = 0.0;
        if (renormalize) {
            double ssum = 0.0, dot = 0.0;
            for (int64_t j = 0; j < k; ++j) ssum += probs[t * E + ids[t * k + j]];
            for (int64_t j = 0; j < k; ++j) dot += dwj[j] * w[t * k + j];
            for (int64_t j = 0; j < k; ++j) dp[ids[t * k + j]] = (dwj[j] - dot) / ssum;
        } else {
            for (int64_t j = 0; j < k; ++j) dp[ids[t * k + j]] = dwj[j];
        }
        const double* p = probs + t * E;
        double pdp = 0.0;
        for (int64_t e = 0; e < E; ++e) pdp += p[e] * dp[e];
        for (int64_t e = 0; e < E; ++e) dl[e] = p[e] * (dp[e] - pdp);
        for (int64_t e = 0; e < E; ++e) dbias[e] += dl[e];
        for (int64_t i = 0; i < d; ++i) {
            double acc = 0.0;
            const uint16_t* wrow = w_router + i * E;
            for (int64_t e = 0; e < E; ++e) {
                dw_router[i * E + e] += xrow[i] * dl[e];
                acc += dl[e] * bf16_to_double(wrow[e]);
            }
            dx[t * d + i] += acc;
        }
    }
    rc = ORACLE_OK;
done:
    free(ids); free(w); free(probs); free(xrow); free(g); free(u); free(h); free(z); free(dz);
    free(dh); free(dg); free(du); free(dwj); free(dp); free(dl);
    return rc;
}

/*
 * The backward restricted to what a sampled check at full size needs; each
 * follows oracle_backward's arithmetic and summation order, so its results
 * equal the corresponding entries of oracle_backward's outputs.
 *
 * oracle_backward_rows: dx_rows[r] = dx[rows[r]] (fp64 [n_rows][d]).  dx[t]
 * depends only on token t (its routing, its k expert evaluations and its
 * router gradient), so each row is computed from that token alone.
 */
int oracle_backward_rows(const uint16_t* x, const uint16_t* w_router, const float* bias,
                         const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                         int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int renormalize,
                         const double* dout, int64_t n_rows, const int64_t* rows, double* dx_rows)
{
    if (!x || !w_router || !w_gate || !w_up || !w_down || !dout || !rows || !dx_rows || T < 0 || d < 1 ||
        E < 1 || k < 1 || k > E || f < 1 || n_rows < 0)
        return ORACLE_BAD_ARG;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* w = (double*)malloc(sizeof(double) * (size_t)k);
    double* probs = (double*)malloc(sizeof(double) * (size_t)E);
    double* xrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* g = (double*)malloc(sizeof(double) * (size_t)f);
    double* u = (double*)malloc(sizeof(double) * (size_t)f);
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    double* z = (double*)malloc(sizeof(double) * (size_t)d);
    double* dz = (double*)malloc(sizeof(double) * (size_t)d);
    double* dh = (double*)malloc(sizeof(double) * (size_t)f);
    double* dg = (double*)malloc(sizeof(double) * (size_t)f);
    double* du = (double*)malloc(sizeof(double) * (size_t)f);
    double* dwj = (double*)malloc(sizeof(double) * (size_t)k);
    double* dp = (double*)malloc(sizeof(double) * (size_t)E);
    double* dl = (double*)malloc(sizeof(double) * (size_t)E);
    int rc = ORACLE_NO_MEMORY;
    if (!ids || !w || !probs || !xrow || !g || !u || !h || !z || !dz || !dh || !dg || !du || !dwj || !dp || !dl)
        goto done;
    rc = ORACLE_OK;
    for (int64_t r = 0; r < n_rows && rc == ORACLE_OK; ++r) {
        const int64_t t = rows[r];
        if (t < 0 || t >= T) { rc = ORACLE_BAD_ARG; break; }
        rc = oracle_route(x + t * d, w_router, bias, 1, d, E, k, NULL, probs, ids, w);
        if (rc != ORACLE_OK) break;
        if (renormalize && (rc = oracle_renormalize(w, 1, k)) != ORACLE_OK) break;
        double* dxr = dx_rows + r * d;
        for (int64_t i = 0; i < d; ++i) { xrow[i] = bf16_to_double(x[t * d + i]); dxr[i] = 0.0; }
        const double* drow_out = dout + t * d;
        for (int64_t j = 0; j < k; ++j) {
            const int64_t e = ids[j];
            const uint16_t* wg = w_gate + e * d * f;
            const uint16_t* wu = w_up + e * d * f;
            const uint16_t* wd = w_down + e * f * d;
            expert_swiglu(xrow, wg, wu, wd, d, f, g, u, h, z);
            double s = 0.0;
            for (int64_t c = 0; c < d; ++c) s += drow_out[c] * z[c];
            dwj[j] = s;
            for (int64_t c = 0; c < d; ++c) dz[c] = w[j] * drow_out[c];
            for (int64_t n = 0; n < f; ++n) {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) acc += dz[c] * bf16_to_double(wd[n * d + c]);
                dh[n] = acc;
            }
            for (int64_t n = 0; n < f; ++n) {
                const double sg = 1.0 / (1.0 + exp(-g[n]));
                du[n] = dh[n] * (g[n] * sg);
                dg[n] = dh[n] * u[n] * sg * (1.0 + g[n] * (1.0 - sg));
            }
            for (int64_t i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int64_t n = 0; n < f; ++n)
                    acc += dg[n] * bf16_to_double(wg[i * f + n]) + du[n] * bf16_to_double(wu[i * f + n]);
                dxr[i] += acc;
            }
        }
        for (int64_t e = 0; e < E; ++e) dp[e] = 0.0;
        if (renormalize) {
            double ssum = 0.0, dot = 0.0;
            for (int64_t j = 0; j < k; ++j) ssum += probs[ids[j]];
            for (int64_t j = 0; j < k; ++j) dot += dwj[j] * w[j];
            for (int64_t j = 0; j < k; ++j) dp[ids[j]] = (dwj[j] - dot) / ssum;
        } else {
            for (int64_t j = 0; j < k; ++j) dp[ids[j]] = dwj[j];
        }
        double pdp = 0.0;
        for (int64_t e = 0; e < E; ++e) pdp += probs[e] * dp[e];
        for (int64_t e = 0; e < E; ++e) dl[e] = probs[e] * (dp[e] - pdp);
        for (int64_t i = 0; i < d; ++i) {
            double acc = 0.0;
            const uint16_t* wrow = w_router + i * E;
            for (int64_t e = 0; e < E; ++e) acc += dl[e] * bf16_to_double(wrow[e]);
            dxr[i] += acc;
        }
    }
done:
    free(ids); free(w); free(probs); free(xrow); free(g); free(u); free(h); free(z); free(dz);
    free(dh); free(dg); free(du); free(dwj); free(dp); free(dl);
    return rc;
}

/*
 * oracle_backward_expert: the weight gradients of one expert e_sel,
 * dw_gate_e, dw_up_e [d][f] and dw_down_e [f][d] (fp64, overwritten): the
 * contributions of the (token, slot) pairs routed to e_sel, tokens in
 * ascending order, exactly as oracle_backward accumulates dW[e_sel].
 */
int oracle_backward_expert(const uint16_t* x, const uint16_t* w_router, const float* bias,
                           const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down,
                           int64_t T, int64_t d, int64_t E, int64_t k, int64_t f, int renormalize,
                           const double* dout, int64_t e_sel, double* dw_gate_e, double* dw_up_e,
                           double* dw_down_e)
{
    if (!x || !w_router || !w_gate || !w_up || !w_down || !dout || !dw_gate_e || !dw_up_e || !dw_down_e ||
        T < 0 || d < 1 || E < 1 || k < 1 || k > E || f < 1 || e_sel < 0 || e_sel >= E)
        return ORACLE_BAD_ARG;
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T * k + 1));
    double* w = (double*)malloc(sizeof(double) * (size_t)(T * k + 1));
    double* xrow = (double*)malloc(sizeof(double) * (size_t)d);
    double* g = (double*)malloc(sizeof(double) * (size_t)f);
    double* u = (double*)malloc(sizeof(double) * (size_t)f);
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    double* z = (double*)malloc(sizeof(double) * (size_t)d);
    double* dz = (double*)malloc(sizeof(double) * (size_t)d);
    double* dh = (double*)malloc(sizeof(double) * (size_t)f);
    double* dg = (double*)malloc(sizeof(double) * (size_t)f);
    double* du = (double*)malloc(sizeof(double) * (size_t)f);
    int rc = ORACLE_NO_MEMORY;
    if (!ids || !w || !xrow || !g || !u || !h || !z || !dz || !dh || !dg || !du) goto done;
    rc = oracle_route(x, w_router, bias, T, d, E, k, NULL, NULL, ids, w);
    if (rc != ORACLE_OK) goto done;
    if (renormalize && (rc = oracle_renormalize(w, T, k)) != ORACLE_OK) goto done;
    memset(dw_gate_e, 0, sizeof(double) * (size_t)(d * f));
    memset(dw_up_e, 0, sizeof(double) * (size_t)(d * f));
    memset(dw_down_e, 0, sizeof(double) * (size_t)(f * d));
    const uint16_t* wg = w_gate + e_sel * d * f;
    const uint16_t* wu = w_up + e_sel * d * f;
    const uint16_t* wd = w_down + e_sel * f * d;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < k; ++j) {
            if (ids[t * k + j] != e_sel) continue;
            for (int64_t i = 0; i < d; ++i) xrow[i] = bf16_to_double(x[t * d + i]);
            const double* drow_out = dout + t * d;
            expert_swiglu(xrow, wg, wu, wd, d, f, g, u, h, z);
            for (int64_t c = 0; c < d; ++c) dz[c] = w[t * k + j] * drow_out[c];
            for (int64_t n = 0; n < f; ++n) {
                double acc = 0.0;
                for (int64_t c = 0; c < d; ++c) {
                    dw_down_e[n * d + c] += h[n] * dz[c];
                    acc += dz[c] * bf16_to_double(wd[n * d + c]);
                }
                dh[n] = acc;
            }
            for (int64_t n = 0; n < f; ++n) {
                const double sg = 1.0 / (1.0 + exp(-g[n]));
                du[n] = dh[n] * (g[n] * sg);
                dg[n] = dh[n] * u[n] * sg * (1.0 + g[n] * (1.0 - sg));
            }
            for (int64_t i = 0; i < d; ++i)
                for (int64_t n = 0; n < f; ++n) {
                    dw_gate_e[i * f + n] += xrow[i] * dg[n];
                    dw_up_e[i * f + n] += xrow[i] * du[n];
                }
        }
    }
    rc = ORACLE_OK;
done:
    free(ids); free(w); free(xrow); free(g); free(u); free(h); free(z); free(dz); free(dh); free(dg); free(du);
    return rc;
}
