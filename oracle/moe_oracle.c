/*
 * moe_oracle.c -- plain fp64 CPU oracle for the sparse top-k MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header or table with the CUDA library; it reads the same input bytes
 * (bf16 or fp32, widened to double on every access) and computes every step
 * in double precision with plain loops, in the order the pages describe.
 *
 * Page references (title, section):
 *   [Mixtral explained]  "Mixtral 8x7B and MoE explained: sparse mixture of
 *                         experts, only 2 experts active per token"
 *   [MoE wiki]           "Mixture of experts" (wiki entry), "How it works"
 *   [Routing explained]  "MoE routing fully explained: the expert-mixture
 *                         structure Mixtral and DeepSeek use, load balancing,
 *                         capacity factor"
 *
 * Where the pages leave a step open, the reading taken is stated at the step.
 * Build: gcc -O2 -fopenmp -shared -fPIC (see oracle/build.py).  OpenMP only
 * splits independent outputs (tokens) across threads; each output's sum runs
 * in one fixed order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

typedef struct {
    int64_t T;           /* tokens */
    int32_t d, h, E, k;  /* model width, expert hidden width, experts, kept per token */
    int32_t n_shared;    /* shared experts (0 if none) */
    int32_t h_shared;    /* hidden width of each shared expert */
    int64_t cf_num, cf_den; /* capacity factor as a fraction; cf_den == 0 means no limit */
    int32_t dtype;       /* ORACLE_F32 or ORACLE_BF16 for x and expert weights */
    int32_t has_bias;    /* router bias present */
    int32_t overflow;    /* ORACLE_DROP or ORACLE_REROUTE */
} oracle_cfg;

#define ORACLE_DROP 0
#define ORACLE_REROUTE 1

/* Widen element i of a bf16 or fp32 array to double.  bf16 is the top half of
 * an IEEE binary32, so the widening is exact. */
static double elem(const void* p, int dtype, int64_t i) {
    float f;
    if (dtype == ORACLE_F32) {
        f = ((const float*)p)[i];
    } else {
        uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        memcpy(&f, &bits, sizeof f);
    }
    return (double)f;
}

/* Expert capacity [Routing explained, "Easy explanation" ¶5]: the buffer per
 * expert is about batch x top-k x capacity factor / number of experts.  The
 * "about" is read as the ceiling, taken in exact integer arithmetic on
 * cf = cf_num / cf_den.  No limit (cf_den == 0) gives T: a token never picks
 * the same expert twice, so no expert can receive more than T tokens. */
int64_t oracle_capacity(const oracle_cfg* c) {
    if (c->cf_den == 0) return c->T;
    int64_t num = c->T * (int64_t)c->k * c->cf_num;
    int64_t den = (int64_t)c->E * c->cf_den;
    return (num + den - 1) / den;
}

/* Router logits [Mixtral explained, "Easy explanation" ¶3; MoE wiki, "How it
 * works"]: a score for every expert, as in a classifier.  Linear router:
 * z[t][e] = sum_c x[t][c] * Wr[c][e] + b[e], c ascending. */
void oracle_logits(const oracle_cfg* c, const void* x, const float* Wr, const float* bias,
                   double* z) {
    const int64_t T = c->T;
    const int d = c->d, E = c->E;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int j = 0; j < d; ++j)
                s += elem(x, c->dtype, t * d + j) * (double)Wr[(int64_t)j * E + e];
            if (c->has_bias) s += (double)bias[e];
            z[t * E + e] = s;
        }
    }
}

/* Top-k and gates [Mixtral explained, "Easy explanation" ¶3]: keep the k
 * highest-scoring experts and softmax over those k alone.  Ties (equal
 * logits) go to the lower expert index, a reading the pages leave open.
 * idx[t][j] lists the kept experts in descending-logit order; gate[t][j] is
 * exp(z_j - z_max) / sum over the kept k of exp(z - z_max). */
void oracle_topk(const oracle_cfg* c, const double* z, int32_t* idx, double* gate) {
    const int64_t T = c->T;
    const int E = c->E, k = c->k;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double* zt = z + t * E;
        int32_t* it = idx + t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int q = 0; q < j; ++q) taken |= (it[q] == e);
                if (taken) continue;
                if (best < 0 || zt[e] > zt[best]) best = e; /* strict: lower index keeps a tie */
            }
            it[j] = best;
        }
        double zmax = zt[it[0]];
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += exp(zt[it[j]] - zmax);
        for (int j = 0; j < k; ++j) gate[t * k + j] = exp(zt[it[j]] - zmax) / den;
    }
}

/* Full softmax over all E experts [Routing explained, "Easy explanation" ¶2:
 * the router forms a probability distribution over every expert].  Used for
 * the load-balancing loss and the router entropy only. */
void oracle_probs(const oracle_cfg* c, const double* z, double* p) {
    const int64_t T = c->T;
    const int E = c->E;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double* zt = z + t * E;
        double zmax = zt[0];
        for (int e = 1; e < E; ++e) if (zt[e] > zmax) zmax = zt[e];
        double den = 0.0;
        for (int e = 0; e < E; ++e) den += exp(zt[e] - zmax);
        for (int e = 0; e < E; ++e) p[t * E + e] = exp(zt[e] - zmax) / den;
    }
}

/* Dispatch under capacity [Routing explained, "Easy explanation" ¶3 and ¶5]:
 * each expert takes at most C tokens per batch; the overflow is dropped.
 * Which assignments overflow is left open by the pages; the reading taken is
 * arrival order by token index: an expert's queue fills with its tokens in
 * increasing t and the rest are dropped.
 *   rank[t][j]  position of token t in expert idx[t][j]'s queue
 *   keep[t][j]  1 if rank < C
 *   routed[e]   assignments to e before the limit; kept[e] = min(routed[e], C) */
void oracle_dispatch(const oracle_cfg* c, const int32_t* idx, int64_t C,
                     int32_t* routed, int32_t* kept, int32_t* rank, int8_t* keep) {
    const int64_t T = c->T;
    const int E = c->E, k = c->k;
    for (int e = 0; e < E; ++e) routed[e] = 0;
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            int32_t r = routed[e]++;
            rank[t * k + j] = r;
            keep[t * k + j] = (r < C) ? 1 : 0;
        }
    }
    for (int e = 0; e < E; ++e) kept[e] = routed[e] < C ? routed[e] : (int32_t)C;
}

/* Overflow rerouted to a spare expert [Routing explained, "Easy explanation"
 * ¶3: the second of the three ways to treat tokens beyond an expert's
 * capacity].  Reading: after the arrival-order pass of oracle_dispatch, the
 * dropped assignments are visited in token order (t, then j); each moves to
 * the token's highest-scoring expert (ties: lower index) that the token does
 * not already use and that still has room, keeping its gate, and joins the end
 * of that expert's queue.  With no room anywhere it stays dropped.
 *   z[t][e]      router logits (bias included)
 *   kept[e]      in: min(routed, C); out: rows each expert serves
 *   rank, keep   in/out: updated for rerouted assignments
 *   expert[t][j] out: the expert serving assignment (t, j) */
void oracle_reroute(const oracle_cfg* c, const double* z, const int32_t* idx, int64_t C,
                    int32_t* kept, int32_t* rank, int8_t* keep, int32_t* expert) {
    const int64_t T = c->T;
    const int E = c->E, k = c->k;
    for (int64_t i = 0; i < T * k; ++i) expert[i] = idx[i];
    for (int64_t t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            if (keep[t * k + j]) continue;
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (kept[e] >= C) continue;
                int used = 0;
                for (int q = 0; q < k; ++q)
                    used |= (idx[t * k + q] == e) || (expert[t * k + q] == e);
                if (used) continue;
                if (best < 0 || z[t * E + e] > z[t * E + best]) best = e;
            }
            if (best < 0) continue;
            expert[t * k + j] = best;
            rank[t * k + j] = kept[best]++;
            keep[t * k + j] = 1;
        }
    }
}

/* Statistics.
 * Load-balancing loss [Routing explained, "Easy explanation" ¶4]: for each
 * expert multiply the share of tokens it actually received by the total
 * probability the router gave it, and sum.  Reading: share f_e = routed[e] /
 * (T k) (hard assignments before the capacity limit, so sum f = 1); mass
 * P_e = mean over tokens of the full softmax (sum P = 1); the sum is scaled by
 * E, so that perfectly even routing gives exactly 1.
 * Overflow rate and router entropy [Routing explained, "Main insights" ¶3]:
 * dropped / (T k), and the mean over tokens of -sum_e p ln p (nats).
 * out[0] = aux, out[1] = overflow rate, out[2] = mean entropy,
 * out[3 .. 3+E) = P_e.  T == 0 gives zeros. */
void oracle_stats(const oracle_cfg* c, const double* p, const int32_t* routed,
                  const int32_t* kept, double* out) {
    const int64_t T = c->T;
    const int E = c->E, k = c->k;
    for (int i = 0; i < 3 + E; ++i) out[i] = 0.0;
    if (T == 0) return;
    double ent = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        double ht = 0.0;
        for (int e = 0; e < E; ++e) {
            double q = p[t * E + e];
            if (q > 0.0) ht -= q * log(q);
        }
        ent += ht;
    }
    double aux = 0.0, dropped = 0.0;
    for (int e = 0; e < E; ++e) {
        double Pe = 0.0;
        for (int64_t t = 0; t < T; ++t) Pe += p[t * E + e];
        Pe /= (double)T;
        double fe = (double)routed[e] / ((double)T * k);
        aux += fe * Pe;
        dropped += (double)(routed[e] - kept[e]);
        out[3 + e] = Pe;
    }
    out[0] = (double)E * aux;
    out[1] = dropped / ((double)T * k);
    out[2] = ent / (double)T;
}

/* One expert's FFN for one token [Mixtral explained, "Easy explanation" ¶2:
 * widen d to h, then narrow back], in the SiLU-gated form
 * y = (silu(x w1) * (x w3)) w2 with silu(a) = a / (1 + e^-a).
 * w1, w3 are [d][h] and w2 is [h][d], row-major, as in y = x W; w_off13 and
 * w_off2 select the expert inside stacked arrays.  x is row x_off of x.
 * a, b are scratch of length h; the result goes to y[d]. */
static void ffn(int d, int h, int dtype, const void* x, int64_t x_off, const void* w1,
                const void* w3, const void* w2, int64_t w_off13, int64_t w_off2, double* y,
                double* a, double* b) {
    for (int i = 0; i < h; ++i) { a[i] = 0.0; b[i] = 0.0; }
    for (int j = 0; j < d; ++j) {
        const double xj = elem(x, dtype, x_off + j);
        const int64_t row = w_off13 + (int64_t)j * h;
        for (int i = 0; i < h; ++i) {
            a[i] += xj * elem(w1, dtype, row + i);
            b[i] += xj * elem(w3, dtype, row + i);
        }
    }
    for (int i = 0; i < h; ++i) a[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
    for (int o = 0; o < d; ++o) y[o] = 0.0;
    for (int i = 0; i < h; ++i) {
        const int64_t row = w_off2 + (int64_t)i * d;
        for (int o = 0; o < d; ++o) y[o] += a[i] * elem(w2, dtype, row + o);
    }
}

/* Single expert FFN on one row, exported for the oracle's own checks. */
void oracle_ffn(int d, int h, int dtype, const void* x_row, const void* w1, const void* w3,
                const void* w2, double* y) {
    double* a = (double*)malloc(sizeof(double) * (size_t)h);
    double* b = (double*)malloc(sizeof(double) * (size_t)h);
    ffn(d, h, dtype, x_row, 0, w1, w3, w2, 0, 0, y, a, b);
    free(a);
    free(b);
}

/* Layer output for selected tokens [Mixtral explained, "Easy explanation" ¶3;
 * MoE wiki, "How it works"; Routing explained, "Easy explanation" ¶4]:
 *   out[t] = sum over kept j of gate[t][j] * FFN_{expert[t][j]}(x_t)
 *          + sum over shared experts s of FFN^shared_s(x_t),
 * expert[t][j] being the router's choice idx[t][j], or the spare expert that
 * serves the assignment under the reroute policy.
 * A dropped assignment simply contributes nothing; the remaining gates are
 * not renormalised (the pages are silent; this is the reading taken).
 * Unselected experts are not evaluated at all.
 * rows[n_rows] lists the tokens to evaluate (NULL = all T); out is
 * [n_rows][d].  w1/w3 are [E][d][h], w2 [E][h][d]; the shared ones are
 * [S][d][hs] and [S][hs][d] (may be NULL when n_shared == 0). */
void oracle_layer_rows(const oracle_cfg* c, const void* x, const int32_t* expert,
                       const double* gate, const int8_t* keep, const void* w1,
                       const void* w3, const void* w2, const void* w1s, const void* w3s,
                       const void* w2s, const int64_t* rows, int64_t n_rows, double* out) {
    const int d = c->d, h = c->h, k = c->k, hs = c->h_shared, S = c->n_shared;
    const int hmax = h > hs ? h : hs;
    if (rows == NULL) n_rows = c->T;
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* b = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            const int64_t t = rows ? rows[r] : r;
            double* acc = out + r * d;
            for (int o = 0; o < d; ++o) acc[o] = 0.0;
            for (int j = 0; j < k; ++j) {
                if (!keep[t * k + j]) continue;
                const int64_t e = expert[t * k + j];
                ffn(d, h, c->dtype, x, t * d, w1, w3, w2, e * d * h, e * h * d, y, a, b);
                for (int o = 0; o < d; ++o) acc[o] += gate[t * k + j] * y[o];
            }
            for (int s = 0; s < S; ++s) {
                ffn(d, hs, c->dtype, x, t * d, w1s, w3s, w2s, (int64_t)s * d * hs,
                    (int64_t)s * hs * d, y, a, b);
                for (int o = 0; o < d; ++o) acc[o] += y[o];
            }
        }
        free(a);
        free(b);
        free(y);
    }
}

#ifdef _OPENMP
#include <omp.h>
#endif
/* Threads the oracle's parallel loops use (reported beside CPU timings). */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ backward
 *
 * Gradients of the layer [the pages motivate them: the softmax weighting of
 * the router and the load-balancing loss are what training acts on, Routing
 * explained, "Easy explanation" ¶2 and ¶4].  The loss taken is
 *   L = sum_t <G_t, out_t> + aux_coef * aux,
 * G = dL/dout being given.  Readings (the pages are silent on all of them):
 *   - the capacity decision and the top-k choice are piecewise constant, so
 *     the routed counts f_e carry no gradient; aux reaches the router through
 *     P_e only;
 *   - gates are not renormalised after a drop, so a dropped assignment still
 *     shapes the gates of the kept ones: its gate gradient is 0, but its logit
 *     receives the softmax-over-k terms of the others;
 *   - under the reroute policy an assignment keeps the gate of the expert the
 *     router chose, so the gate gradient goes to that expert's logit while the
 *     FFN evaluated (and differentiated) is the serving expert's.
 * With a = x w1, b = x w3, s = silu(a), u = s * b, y = u w2 and
 * silu'(a) = sig(a) (1 + a (1 - sig(a))):
 *   dy = g G_t,  dg = <G_t, y>,  dw2 += u^T dy,  du = w2 dy,
 *   da = du * b * silu'(a),  db = du * s,
 *   dw1 += x^T da,  dw3 += x^T db,  dx += w1 da + w3 db;
 *   softmax over the kept k:  dz[idx_j] += g_j (dg_j - sum_q g_q dg_q);
 *   aux = E sum_e f_e P_e, P_e = mean_t p_te:
 *     dz[t][e] += aux_coef (E / T) p_te (f_e - sum_i f_i p_ti);
 *   router z = x Wr + b:  dWr += x^T dz,  db_router += dz,  dx += Wr dz.
 * Shared experts take dy = G_t (gate 1) and have no gate gradient. */

/* One expert's FFN forward and backward for one token.  Adds into dw1, dw3
 * ([d][h] at w_off13), dw2 ([h][d] at w_off2) and dx ([d]); returns
 * <G_t, y>.  dw1 == NULL skips the weight gradients.  a, b, u, du are scratch
 * of length h; y of length d. */
static double ffn_backward(int d, int h, int dtype, const void* x, int64_t x_off,
                           const void* G, double g, const void* w1, const void* w3,
                           const void* w2, int64_t w_off13, int64_t w_off2, double* dw1,
                           double* dw3, double* dw2, double* dx, double* a, double* b,
                           double* u, double* du, double* y) {
    for (int i = 0; i < h; ++i) { a[i] = 0.0; b[i] = 0.0; }
    for (int c = 0; c < d; ++c) {
        const double xc = elem(x, dtype, x_off + c);
        const int64_t row = w_off13 + (int64_t)c * h;
        for (int i = 0; i < h; ++i) {
            a[i] += xc * elem(w1, dtype, row + i);
            b[i] += xc * elem(w3, dtype, row + i);
        }
    }
    for (int i = 0; i < h; ++i) u[i] = a[i] / (1.0 + exp(-a[i])) * b[i];
    for (int o = 0; o < d; ++o) y[o] = 0.0;
    for (int i = 0; i < h; ++i) {
        const int64_t row = w_off2 + (int64_t)i * d;
        for (int o = 0; o < d; ++o) y[o] += u[i] * elem(w2, dtype, row + o);
    }
    double dg = 0.0;
    for (int o = 0; o < d; ++o) dg += elem(G, dtype, x_off + o) * y[o];
    /* dy = g G_t, used through its entries below */
    for (int i = 0; i < h; ++i) {
        const int64_t row = w_off2 + (int64_t)i * d;
        double s = 0.0;
        for (int o = 0; o < d; ++o) {
            const double dyo = g * elem(G, dtype, x_off + o);
            if (dw1) dw2[row + o] += u[i] * dyo;
            s += elem(w2, dtype, row + o) * dyo;
        }
        du[i] = s;
    }
    for (int i = 0; i < h; ++i) {
        const double sig = 1.0 / (1.0 + exp(-a[i]));
        const double silu = a[i] * sig;
        const double da = du[i] * b[i] * sig * (1.0 + a[i] * (1.0 - sig));
        const double db = du[i] * silu;
        a[i] = da;  /* reuse the scratch: a <- da, b <- db */
        b[i] = db;
    }
    for (int c = 0; c < d; ++c) {
        const double xc = elem(x, dtype, x_off + c);
        const int64_t row = w_off13 + (int64_t)c * h;
        double s = 0.0;
        for (int i = 0; i < h; ++i) {
            if (dw1) {
                dw1[row + i] += xc * a[i];
                dw3[row + i] += xc * b[i];
            }
            s += elem(w1, dtype, row + i) * a[i] + elem(w3, dtype, row + i) * b[i];
        }
        dx[c] += s;
    }
    return dg;
}

/* Gradient of the router logits of token t (gate path and aux path).
 *   dgt[j]  <G_t, y_j> for kept assignments, 0 for dropped ones
 *   f[e]    routed[e] / (T k);  dzt[E] out */
static void router_logit_grad(const oracle_cfg* c, const double* zt, const int32_t* it,
                              const double* gt, const double* dgt, const double* f,
                              double aux_coef, double* dzt) {
    const int E = c->E, k = c->k;
    for (int e = 0; e < E; ++e) dzt[e] = 0.0;
    double m = 0.0;
    for (int j = 0; j < k; ++j) m += gt[j] * dgt[j];
    for (int j = 0; j < k; ++j) dzt[it[j]] += gt[j] * (dgt[j] - m);
    double zmax = zt[0];
    for (int e = 1; e < E; ++e) if (zt[e] > zmax) zmax = zt[e];
    double den = 0.0;
    for (int e = 0; e < E; ++e) den += exp(zt[e] - zmax);
    double q = 0.0;
    for (int e = 0; e < E; ++e) q += f[e] * exp(zt[e] - zmax) / den;
    const double scale = aux_coef * (double)E / (double)c->T;
    for (int e = 0; e < E; ++e) {
        const double p = exp(zt[e] - zmax) / den;
        dzt[e] += scale * p * (f[e] - q);
    }
}

/* The whole backward pass.  Inputs: the forward's logits z [T][E] (bias
 * included), router choice idx, serving expert, gates, keep flags and routed
 * counts; G [T][d] in the layer dtype.  Outputs (all overwritten, fp64):
 *   dx [T][d], dWr [d][E], db [E], dz [T][E],
 *   dw1, dw3 [E][d][h], dw2 [E][h][d], and (n_shared > 0) dw1s, dw3s
 *   [S][d][hs], dw2s [S][hs][d].
 * Tokens are visited in increasing order and every sum runs in one fixed
 * order; single-threaded (small cases only). */
void oracle_backward(const oracle_cfg* c, const void* x, const float* Wr, const double* z,
                     const int32_t* idx, const int32_t* expert, const double* gate,
                     const int8_t* keep, const int32_t* routed, const void* w1,
                     const void* w3, const void* w2, const void* w1s, const void* w3s,
                     const void* w2s, const void* G, double aux_coef, double* dx, double* dWr,
                     double* db, double* dz, double* dw1, double* dw3, double* dw2,
                     double* dw1s, double* dw3s, double* dw2s) {
    const int64_t T = c->T;
    const int d = c->d, h = c->h, E = c->E, k = c->k, S = c->n_shared, hs = c->h_shared;
    const int hmax = h > hs ? h : hs;
    memset(dx, 0, sizeof(double) * (size_t)(T * d));
    memset(dWr, 0, sizeof(double) * (size_t)d * E);
    memset(db, 0, sizeof(double) * (size_t)E);
    memset(dz, 0, sizeof(double) * (size_t)(T * E));
    memset(dw1, 0, sizeof(double) * (size_t)E * d * h);
    memset(dw3, 0, sizeof(double) * (size_t)E * d * h);
    memset(dw2, 0, sizeof(double) * (size_t)E * h * d);
    if (S > 0) {
        memset(dw1s, 0, sizeof(double) * (size_t)S * d * hs);
        memset(dw3s, 0, sizeof(double) * (size_t)S * d * hs);
        memset(dw2s, 0, sizeof(double) * (size_t)S * hs * d);
    }
    if (T == 0) return;
    double* a = (double*)malloc(sizeof(double) * (size_t)hmax);
    double* b = (double*)malloc(sizeof(double) * (size_t)hmax);
    double* u = (double*)malloc(sizeof(double) * (size_t)hmax);
    double* du = (double*)malloc(sizeof(double) * (size_t)hmax);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    double* f = (double*)malloc(sizeof(double) * (size_t)E);
    double* dg = (double*)malloc(sizeof(double) * (size_t)k);
    for (int e = 0; e < E; ++e) f[e] = (double)routed[e] / ((double)T * k);
    for (int64_t t = 0; t < T; ++t) {
        double* dxt = dx + t * d;
        for (int j = 0; j < k; ++j) {
            dg[j] = 0.0;
            if (!keep[t * k + j]) continue;
            const int64_t e = expert[t * k + j];
            dg[j] = ffn_backward(d, h, c->dtype, x, t * d, G, gate[t * k + j], w1, w3, w2,
                                 e * d * h, e * h * d, dw1, dw3, dw2, dxt, a, b, u, du, y);
        }
        for (int s = 0; s < S; ++s)
            (void)ffn_backward(d, hs, c->dtype, x, t * d, G, 1.0, w1s, w3s, w2s,
                               (int64_t)s * d * hs, (int64_t)s * hs * d, dw1s, dw3s, dw2s, dxt,
                               a, b, u, du, y);
        double* dzt = dz + t * E;
        router_logit_grad(c, z + t * E, idx + t * k, gate + t * k, dg, f, aux_coef, dzt);
        for (int cc = 0; cc < d; ++cc) {
            const double xc = elem(x, c->dtype, t * d + cc);
            double s = 0.0;
            for (int e = 0; e < E; ++e) {
                dWr[(int64_t)cc * E + e] += xc * dzt[e];
                s += (double)Wr[(int64_t)cc * E + e] * dzt[e];
            }
            dxt[cc] += s;
        }
        for (int e = 0; e < E; ++e) db[e] += dzt[e];
    }
    free(a); free(b); free(u); free(du); free(y); free(f); free(dg);
}

/* dx and dz rows of selected tokens (no weight gradients), for checks of
 * large batches: each row needs only its own token, the routed counts and
 * the token's experts.  rows[n_rows] lists the tokens; dx_rows [n_rows][d],
 * dz_rows [n_rows][E]. */
void oracle_backward_rows(const oracle_cfg* c, const void* x, const float* Wr, const double* z,
                          const int32_t* idx, const int32_t* expert, const double* gate,
                          const int8_t* keep, const int32_t* routed, const void* w1,
                          const void* w3, const void* w2, const void* w1s, const void* w3s,
                          const void* w2s, const void* G, double aux_coef, const int64_t* rows,
                          int64_t n_rows, double* dx_rows, double* dz_rows) {
    const int64_t T = c->T;
    const int d = c->d, h = c->h, E = c->E, k = c->k, S = c->n_shared, hs = c->h_shared;
    const int hmax = h > hs ? h : hs;
    double* f = (double*)malloc(sizeof(double) * (size_t)E);
    for (int e = 0; e < E; ++e) f[e] = T > 0 ? (double)routed[e] / ((double)T * k) : 0.0;
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* b = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* u = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* du = (double*)malloc(sizeof(double) * (size_t)hmax);
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
        double* dg = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            const int64_t t = rows[r];
            double* dxt = dx_rows + r * d;
            for (int cc = 0; cc < d; ++cc) dxt[cc] = 0.0;
            for (int j = 0; j < k; ++j) {
                dg[j] = 0.0;
                if (!keep[t * k + j]) continue;
                const int64_t e = expert[t * k + j];
                dg[j] = ffn_backward(d, h, c->dtype, x, t * d, G, gate[t * k + j], w1, w3, w2,
                                     e * d * h, e * h * d, NULL, NULL, NULL, dxt, a, b, u, du, y);
            }
            for (int s = 0; s < S; ++s)
                (void)ffn_backward(d, hs, c->dtype, x, t * d, G, 1.0, w1s, w3s, w2s,
                                   (int64_t)s * d * hs, (int64_t)s * hs * d, NULL, NULL, NULL,
                                   dxt, a, b, u, du, y);
            double* dzt = dz_rows + r * E;
            router_logit_grad(c, z + t * E, idx + t * k, gate + t * k, dg, f, aux_coef, dzt);
            for (int cc = 0; cc < d; ++cc) {
                double s = 0.0;
                for (int e = 0; e < E; ++e) s += (double)Wr[(int64_t)cc * E + e] * dzt[e];
                dxt[cc] += s;
            }
        }
        free(a); free(b); free(u); free(du); free(y); free(dg);
    }
    free(f);
}

/* A block of one expert's weight gradients, for checks of large batches.
 * Expert `e` of the routed set (shared == 0; tokens whose kept assignment is
 * served by e, with their gates) or shared expert `e` (shared == 1; every
 * token, gate 1).  For hidden indices hi[ni] and model indices ci[nc]:
 *   out1[a][b] = dw1[ci[b]][hi[a]],  out3[a][b] = dw3[ci[b]][hi[a]],
 *   out2[a][b] = dw2[hi[a]][ci[b]]    (each [ni][nc]).
 * Tokens are visited in increasing order. */
void oracle_wgrad_block(const oracle_cfg* c, const void* x, const int32_t* expert,
                        const double* gate, const int8_t* keep, const void* w1, const void* w3,
                        const void* w2, const void* G, int shared, int e, const int32_t* hi,
                        int ni, const int32_t* ci, int nc, double* out1, double* out3,
                        double* out2) {
    const int64_t T = c->T;
    const int d = c->d, k = c->k;
    const int h = shared ? c->h_shared : c->h;
    const int64_t off13 = (int64_t)e * d * h, off2 = (int64_t)e * h * d;
    for (int i = 0; i < ni * nc; ++i) { out1[i] = 0.0; out3[i] = 0.0; out2[i] = 0.0; }
#pragma omp parallel for schedule(static)
    for (int q = 0; q < ni; ++q) {
        const int i = hi[q];
        for (int64_t t = 0; t < T; ++t) {
            for (int j = 0; j < (shared ? 1 : k); ++j) {
                double g = 1.0;
                if (!shared) {
                    if (!keep[t * k + j] || expert[t * k + j] != e) continue;
                    g = gate[t * k + j];
                }
                double a = 0.0, b = 0.0, du = 0.0;
                for (int cc = 0; cc < d; ++cc) {
                    const double xc = elem(x, c->dtype, t * d + cc);
                    a += xc * elem(w1, c->dtype, off13 + (int64_t)cc * h + i);
                    b += xc * elem(w3, c->dtype, off13 + (int64_t)cc * h + i);
                }
                for (int o = 0; o < d; ++o)
                    du += elem(w2, c->dtype, off2 + (int64_t)i * d + o) * g *
                          elem(G, c->dtype, t * d + o);
                const double sig = 1.0 / (1.0 + exp(-a));
                const double u = a * sig * b;
                const double da = du * b * sig * (1.0 + a * (1.0 - sig));
                const double dbv = du * a * sig;
                for (int r = 0; r < nc; ++r) {
                    const double xc = elem(x, c->dtype, t * d + ci[r]);
                    out1[q * nc + r] += xc * da;
                    out3[q * nc + r] += xc * dbv;
                    out2[q * nc + r] += u * g * elem(G, c->dtype, t * d + ci[r]);
                }
            }
        }
    }
}
