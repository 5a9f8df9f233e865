/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of one MoE FFN layer forward.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or helper with the CUDA path and must never be used to produce a product
 * result.
 *
 * What it computes, step by step, in the order the pages describe the layer
 * (m.xxqk.cn Hy4-preview MoE explainer, section 2.2 "router mechanism": every
 * token is scored against every expert, the K best-scoring experts are
 * activated, they process the same token and their results are merged into the
 * layer output; ZAKER Hy4 Preview release news, MoE paragraph: 256 routed
 * experts plus 1 shared expert, 8 routed experts plus the shared one active per
 * token).  The pages leave the gate function, the renormalisation and the FFN
 * form open; the readings used here are: softmax gate over all router logits,
 * the top-k gate values renormalised to sum to 1, SwiGLU experts without bias
 * (down(silu(gate x) * up x)), shared experts added with weight 1.
 *
 * Every floating-point step runs in double precision on the exact widening of
 * the bf16 / fp32 inputs; nothing is rounded in between.  Loops are the plain
 * definition: no blocking, no reordering, no fusion.
 *
 * bf16 values are passed as their raw 16-bit patterns (uint16_t).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEM 2
#define ORACLE_MISSING_EXPERT 3

/* Exact widening of a bf16 bit pattern: the bf16 value is the fp32 whose high
 * 16 bits are the pattern and whose low 16 bits are zero. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Step 1 -- router score ("matching score" of a token against each expert,
 * explainer section 2.2):  logits[t][e] = sum_j x[t][j] * Wr[e][j] + bias[e].
 * x: [T][d] bf16, Wr: [E][d] fp32, bias: [E] fp32 or NULL, logits: [T][E]. */
int oracle_router_logits(const uint16_t *x, const float *Wr, const float *bias,
                         int T, int d, int E, double *logits) {
    if (T < 0 || d <= 0 || E <= 0 || (T > 0 && (!x || !Wr || !logits))) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += bf16_to_double(x[(size_t)t * d + j]) * (double)Wr[(size_t)e * d + j];
            if (bias) s += (double)bias[e];
            logits[(size_t)t * E + e] = s;
        }
    }
    return ORACLE_OK;
}

/* Steps 2-4 -- gate and top-k for one token row of logits.
 *   p = softmax over all E logits;
 *   experts ordered by (p descending, expert index ascending), first k kept;
 *   margin = l_(k) - l_(k+1)  (the k-th minus the (k+1)-th largest logit,
 *            +INFINITY when k == E);
 *   w_i = p_{e_i} / sum_{j<k} p_{e_j}.
 * The selection is done by k passes of a plain linear scan, each taking the
 * best not-yet-taken expert under the order above. */
static void route_row(const double *l, int E, int k, int32_t *idx, double *w,
                      double *margin, double *p, unsigned char *taken) {
    double lmax = l[0];
    for (int e = 1; e < E; ++e)
        if (l[e] > lmax) lmax = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(l[e] - lmax);
        z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;

    memset(taken, 0, (size_t)E);
    double psum = 0.0;
    for (int i = 0; i < k; ++i) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || p[e] > p[best]) best = e; /* strict '>' keeps the lower index on ties */
        }
        taken[best] = 1;
        idx[i] = best;
        psum += p[best];
    }
    for (int i = 0; i < k; ++i) w[i] = p[idx[i]] / psum;

    if (margin) {
        if (k == E) {
            *margin = INFINITY;
        } else {
            int next = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (next < 0 || p[e] > p[next]) next = e;
            }
            *margin = l[idx[k - 1]] - l[next];
        }
    }
}

/* Steps 2-4 for T tokens.  logits: [T][E]; idx: [T][k]; w: [T][k];
 * margin: [T] or NULL. */
int oracle_route(const double *logits, int T, int E, int k, int32_t *idx, double *w,
                 double *margin) {
    if (T < 0 || E <= 0 || k < 1 || k > E) return ORACLE_BAD_ARG;
    if (T == 0) return ORACLE_OK;
    if (!logits || !idx || !w) return ORACLE_BAD_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!p || !taken) {
#pragma omp atomic write
            err = ORACLE_NO_MEM;
        } else {
#pragma omp for schedule(static)
            for (int t = 0; t < T; ++t)
                route_row(logits + (size_t)t * E, E, k, idx + (size_t)t * k, w + (size_t)t * k,
                          margin ? margin + t : NULL, p, taken);
        }
        free(p);
        free(taken);
    }
    return err;
}

/* Step 5 -- group the T*k (token, choice) slots by expert.
 *   counts[e]  = number of slots s = t*k+i with idx[s] == e;
 *   offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e];
 *   perm[p]    = the slot stored at position p: within expert e's segment
 *                [offsets[e], offsets[e+1]) the slots appear in ascending
 *                slot order (a stable counting sort);
 *   pos[s]     = the position of slot s, i.e. perm[pos[s]] == s.
 * Written as the textbook counting sort: count, exclusive scan, then one
 * ascending pass that places every slot at its expert's next free position. */
int oracle_dispatch(const int32_t *idx, int T, int E, int k, int32_t *counts,
                    int32_t *offsets, int32_t *perm, int32_t *pos) {
    if (T < 0 || E <= 0 || k < 1 || !counts || !offsets) return ORACLE_BAD_ARG;
    const long n = (long)T * k;
    if (n > 0 && (!idx || !perm || !pos)) return ORACLE_BAD_ARG;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long s = 0; s < n; ++s) {
        if (idx[s] < 0 || idx[s] >= E) return ORACLE_BAD_ARG;
        counts[idx[s]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    if (!next) return ORACLE_NO_MEM;
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (long s = 0; s < n; ++s) {
        int32_t p = next[idx[s]]++;
        perm[p] = (int32_t)s;
        pos[s] = p;
    }
    free(next);
    return ORACLE_OK;
}

/* Step 6 -- one SwiGLU expert on one token (explainer section 2.1: each expert
 * is an FFN sub-network that stands in for the dense FFN):
 *   g[f] = sum_j Wg[f][j] x[j],  u[f] = sum_j Wu[f][j] x[j],
 *   h[f] = silu(g[f]) * u[f] = g[f] / (1 + exp(-g[f])) * u[f],
 *   y[i] = sum_f Wd[i][f] h[f].
 * Wg, Wu: [F][d] bf16; Wd: [d][F] bf16; x: [d] (already widened); h: [F]
 * scratch; y: [d] output. */
static void swiglu_expert(const uint16_t *Wg, const uint16_t *Wu, const uint16_t *Wd,
                          const double *x, int d, int F, double *h, double *y) {
    for (int f = 0; f < F; ++f) {
        double g = 0.0, u = 0.0;
        for (int j = 0; j < d; ++j) {
            g += bf16_to_double(Wg[(size_t)f * d + j]) * x[j];
            u += bf16_to_double(Wu[(size_t)f * d + j]) * x[j];
        }
        h[f] = g / (1.0 + exp(-g)) * u;
    }
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int f = 0; f < F; ++f) s += bf16_to_double(Wd[(size_t)i * F + f]) * h[f];
        y[i] = s;
    }
}

/* Steps 6-7 -- the layer output for a chosen list of tokens.
 *   y[t] = sum_{s<S} FFN_shared_s(x_t) + sum_{i<k} w[t][i] * FFN_{idx[t][i]}(x_t).
 * Expert weights are passed as arrays of per-expert pointers so that a caller
 * may supply only the experts that the chosen tokens use (a NULL pointer for an
 * expert that a chosen token needs is an error).
 *   x: [T][d] bf16 (all tokens); idx: [T][k]; w: [T][k];
 *   Wg[e], Wu[e]: [F][d] bf16; Wd[e]: [d][F] bf16 (e < E);
 *   Sg[s], Su[s], Sd[s]: the shared experts (s < S);
 *   tokens: [n_tok] token indices; y: [n_tok][d] output (row r is token tokens[r]). */
int oracle_moe_ffn_tokens(const uint16_t *x, int T, int d, int E, int k, int F, int S,
                          const int32_t *idx, const double *w,
                          const uint16_t *const *Wg, const uint16_t *const *Wu,
                          const uint16_t *const *Wd,
                          const uint16_t *const *Sg, const uint16_t *const *Su,
                          const uint16_t *const *Sd,
                          const int32_t *tokens, int n_tok, double *y) {
    if (T < 0 || d <= 0 || E <= 0 || k < 1 || k > E || F <= 0 || S < 0 || n_tok < 0)
        return ORACLE_BAD_ARG;
    if (n_tok == 0) return ORACLE_OK;
    if (!x || !idx || !w || !tokens || !y || !Wg || !Wu || !Wd) return ORACLE_BAD_ARG;
    if (S > 0 && (!Sg || !Su || !Sd)) return ORACLE_BAD_ARG;
    for (int r = 0; r < n_tok; ++r) {
        int t = tokens[r];
        if (t < 0 || t >= T) return ORACLE_BAD_ARG;
        for (int i = 0; i < k; ++i) {
            int e = idx[(size_t)t * k + i];
            if (e < 0 || e >= E) return ORACLE_BAD_ARG;
            if (!Wg[e] || !Wu[e] || !Wd[e]) return ORACLE_MISSING_EXPERT;
        }
    }
    for (int s = 0; s < S; ++s)
        if (!Sg[s] || !Su[s] || !Sd[s]) return ORACLE_MISSING_EXPERT;

    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *xt = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        double *ye = (double *)malloc(sizeof(double) * (size_t)d);
        if (!xt || !h || !ye) {
#pragma omp atomic write
            err = ORACLE_NO_MEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < n_tok; ++r) {
                const int t = tokens[r];
                double *yt = y + (size_t)r * d;
                for (int j = 0; j < d; ++j) xt[j] = bf16_to_double(x[(size_t)t * d + j]);
                for (int j = 0; j < d; ++j) yt[j] = 0.0;
                for (int s = 0; s < S; ++s) {
                    swiglu_expert(Sg[s], Su[s], Sd[s], xt, d, F, h, ye);
                    for (int j = 0; j < d; ++j) yt[j] += ye[j];
                }
                for (int i = 0; i < k; ++i) {
                    const int e = idx[(size_t)t * k + i];
                    const double wi = w[(size_t)t * k + i];
                    swiglu_expert(Wg[e], Wu[e], Wd[e], xt, d, F, h, ye);
                    for (int j = 0; j < d; ++j) yt[j] += wi * ye[j];
                }
            }
        }
        free(xt);
        free(h);
        free(ye);
    }
    return err;
}

/* The intermediate of step 6 for one (token, expert) pair, exposed so that
 * tests can compare per-stage values: h = silu(Wg x) * (Wu x) ([F]) and
 * y = Wd h ([d]). */
int oracle_expert_one(const uint16_t *xrow, int d, int F, const uint16_t *Wg,
                      const uint16_t *Wu, const uint16_t *Wd, double *h, double *y) {
    if (d <= 0 || F <= 0 || !xrow || !Wg || !Wu || !Wd || !h || !y) return ORACLE_BAD_ARG;
    double *xt = (double *)malloc(sizeof(double) * (size_t)d);
    if (!xt) return ORACLE_NO_MEM;
    for (int j = 0; j < d; ++j) xt[j] = bf16_to_double(xrow[j]);
    swiglu_expert(Wg, Wu, Wd, xt, d, F, h, y);
    free(xt);
    return ORACLE_OK;
}

/* Step 7 alone -- merge per-(slot, expert) outputs into the layer output:
 *   y[t] = sum_{s<S} Yrows[T*k + s*T + t] + sum_{i<k} w[t][i] * Yrows[pos[t*k+i]].
 * Yrows: [T*k + S*T][d] (any fp64 values); w: [T][k]; pos: [T*k]; y: [T][d]. */
int oracle_combine(const double *Yrows, const double *w, const int32_t *pos, int T, int k, int S,
                   int d, double *y) {
    if (T < 0 || k < 1 || S < 0 || d <= 0) return ORACLE_BAD_ARG;
    if (T == 0) return ORACLE_OK;
    if (!Yrows || !w || !pos || !y) return ORACLE_BAD_ARG;
    const long nslots = (long)T * k;
    for (long s = 0; s < nslots; ++s)
        if (pos[s] < 0 || pos[s] >= nslots) return ORACLE_BAD_ARG;
    for (int t = 0; t < T; ++t) {
        double *yt = y + (size_t)t * d;
        for (int j = 0; j < d; ++j) yt[j] = 0.0;
        for (int s = 0; s < S; ++s) {
            const double *row = Yrows + ((size_t)nslots + (size_t)s * T + t) * d;
            for (int j = 0; j < d; ++j) yt[j] += row[j];
        }
        for (int i = 0; i < k; ++i) {
            const double wi = w[(size_t)t * k + i];
            const double *row = Yrows + (size_t)pos[(size_t)t * k + i] * d;
            for (int j = 0; j < d; ++j) yt[j] += wi * row[j];
        }
    }
    return ORACLE_OK;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
