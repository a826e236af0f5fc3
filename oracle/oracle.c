/*
 * oracle.c -- plain, slow, float64 CPU oracle for the RAT+ dilated-inference hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU-baseline leg
 * call this code; the library under recurrence_augmented_dilated_b200/ never does, and the two
 * share no source, header, table or helper.  Every routine is the written-out definition of
 * what it computes, with no blocking, fusion or reordering: loops in the order of the maths.
 *
 * Sources (page title, section):
 *   [RAT+ Deep Dive]  "RAT+ Deep Dive: A New KV Cache Compression Paradigm ...", section 2.1
 *                     "Full-Sequence Recurrence" (forget-gate recurrence over the whole
 *                     sequence, L = T, computed by an associative scan in prefill);
 *                     section 3.1 table (attention FLOPs T/D); section 6 "Head-Wise Hybrid".
 *   [RAT+ abstract]   "RAT+: Train Dense, Infer Sparse -- Recurrence Augmented Attention for
 *                     Dilated Inference", abstract (dilation D cuts attention FLOPs and KV cache
 *                     by D; optional local windows; hybrid layer/head compositions).
 *   [RAT abstract]    "RAT: Bridging RNN Efficiency and Attention Accuracy via Chunk-based
 *                     Sequence Modeling", abstract (recurrence inside chunks, attention across
 *                     chunk ends).
 *   [RoFormer]        rotary position embedding, cited by the RAT+ page; rotate-half pairing.
 *
 * The recurrence formula itself is lost from the blog's section 2.1: the text keeps only that
 * the recurrence uses a forget gate which depends on the input and decays memory as an LSTM
 * does; the form used here is the standard gated EMA  h_t = g_t * h_{t-1} + (1 - g_t) * x_t with
 * g_t = sigmoid(a_t), elementwise per channel, the same gate for keys and values.
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *   - the gate logit tensor is one (B,H,T,d) tensor shared by K and V;
 *   - h_{-1} = h0 (zero unless given);
 *   - key set of query t:  S(t) = { j : t - We < j <= t }  U  { j : j <= t - We, j mod D = D-1 },
 *     with We = max(W, 1): the query always sees its own recurrence output, the dilated keys
 *     are the chunk ends (positions D-1, 2D-1, ...) older than the window, the union is disjoint;
 *   - RoPE is applied to the recurrence output k~ (not to the raw k) and to q, at the absolute
 *     position pos0 + t, rotate-half pairing (c, c + d/2), theta_c = base^(-2c/d);
 *   - softmax scale is 1/sqrt(d) unless the caller gives one.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC oracle.c -o liboracle.so -lm  (see build.py).
 * OpenMP parallelism is over independent (batch, head) slices only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------------------- */
/* Forget gate.  g = sigmoid(a) = 1/(1+e^{-a});  1-g = 1/(1+e^{a}) (computed directly so that
 * it keeps full relative precision when g is close to 1).                [RAT+ Deep Dive 2.1] */
static double forget_gate(double a) { return 1.0 / (1.0 + exp(-a)); }
static double one_minus_gate(double a) { return 1.0 / (1.0 + exp(a)); }

/*
 * Full-sequence forget-gate recurrence, one tensor at a time.               [RAT+ Deep Dive 2.1]
 *   x, a, y : [BH][T][d]      h0, hT : [BH][d] (either may be NULL; NULL h0 means zeros)
 *   h_{-1} = h0;   h_t = g_t * h_{t-1} + (1 - g_t) * x_t;   y_t = h_t;   hT = h_{T-1}.
 * A sequential loop over t: the definition itself, no scan.
 */
void rat_oracle_recurrence(long BH, long T, long d, const double *x, const double *a,
                           const double *h0, double *y, double *hT)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        for (long c = 0; c < d; ++c) {
            double h = h0 ? h0[bh * d + c] : 0.0;
            for (long t = 0; t < T; ++t) {
                long idx = (bh * T + t) * d + c;
                double g = forget_gate(a[idx]);
                double omg = one_minus_gate(a[idx]);
                h = g * h + omg * x[idx];
                y[idx] = h;
            }
            if (hT) hT[bh * d + c] = h;
        }
    }
}

/*
 * Chunk-local recurrence of the predecessor RAT ("RAT+ Deep Dive" section 2.1: in the original
 * RAT the recurrence of a token stays inside its own block of L positions; the RAT paper's
 * abstract: recurrence within each chunk).  Same step as above, but the state is
 * set to zero before every absolute position p = pos0 + t with p mod L == 0 (L > 0), so each
 * block of L positions starts from an empty state.  h0 is the state before pos0 (dropped when
 * pos0 itself starts a block).
 */
void rat_oracle_recurrence_reset(long BH, long T, long d, const double *x, const double *a,
                                 const double *h0, double *y, double *hT, long pos0, long L)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        for (long c = 0; c < d; ++c) {
            double h = h0 ? h0[bh * d + c] : 0.0;
            for (long t = 0; t < T; ++t) {
                long idx = (bh * T + t) * d + c;
                if ((pos0 + t) % L == 0) h = 0.0;        /* a new block starts here */
                double g = forget_gate(a[idx]);
                double omg = one_minus_gate(a[idx]);
                h = g * h + omg * x[idx];
                y[idx] = h;
            }
            if (hT) hT[bh * d + c] = h;
        }
    }
}

/*
 * Fixed-window recurrence of RAT+ ("RAT+ Deep Dive" section 2.1: every token's recurrence looks
 * back a fixed L* = 64 tokens, independent of the dilation).  Read as: the state at t is the
 * forget-gate recurrence started from zero at position t - Lw + 1 and run to t,
 *   y_t = sum_{s = t-Lw+1}^{t} ( prod_{r = s+1}^{t} g_r ) (1 - g_s) x_s,
 * evaluated here by that restarted sequential loop for every t (O(T Lw) per channel).  Rows
 * before the sequence come from prev_x / prev_a ([BH][Lw][d]: the Lw positions just before row 0,
 * oldest first) when given; without them the window is clipped at row 0.
 */
void rat_oracle_recurrence_window(long BH, long T, long d, const double *x, const double *a,
                                  const double *prev_x, const double *prev_a, long Lw, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        for (long c = 0; c < d; ++c) {
            for (long t = 0; t < T; ++t) {
                double h = 0.0;
                for (long s = t - Lw + 1; s <= t; ++s) {
                    double xs, as;
                    if (s >= 0) {
                        xs = x[(bh * T + s) * d + c];
                        as = a[(bh * T + s) * d + c];
                    } else if (prev_x && s >= -Lw) {
                        xs = prev_x[(bh * Lw + (Lw + s)) * d + c];
                        as = prev_a[(bh * Lw + (Lw + s)) * d + c];
                    } else {
                        continue;           /* before the known sequence: clipped */
                    }
                    h = forget_gate(as) * h + one_minus_gate(as) * xs;
                }
                y[(bh * T + t) * d + c] = h;
            }
        }
    }
}

/*
 * Backward of the forget-gate recurrence above (its reverse-mode derivative), for one of x = k
 * or x = v.  With dy_t = dL/dy_t the upstream gradient of the outputs y_t = h_t and dhT =
 * dL/dh_{T-1} an extra gradient of the final state (NULL: none), the total gradient of the
 * state runs backwards,
 *   mu_{T-1} = dy_{T-1} + dhT,      mu_t = dy_t + g_{t+1} mu_{t+1},
 * and gives  dL/dx_t = (1 - g_t) mu_t,   dL/dg_t = mu_t (h_{t-1} - x_t)  (h_{-1} = h0),
 *            dL/dh0 = g_0 mu_0.
 * h is recomputed by the forward loop; dg is the gradient with respect to the gate value g
 * (the caller applies dg/da = g (1 - g) and sums the k and v parts, which share the gate).
 */
void rat_oracle_recurrence_backward(long BH, long T, long d, const double *x, const double *a,
                                    const double *h0, const double *dy, const double *dhT,
                                    double *dx, double *dg, double *dh0)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *h = (double *)malloc((size_t)(T + 1) * sizeof(double));  /* h[t+1] = h_t */
        for (long c = 0; c < d; ++c) {
            h[0] = h0 ? h0[bh * d + c] : 0.0;
            for (long t = 0; t < T; ++t) {
                long idx = (bh * T + t) * d + c;
                h[t + 1] = forget_gate(a[idx]) * h[t] + one_minus_gate(a[idx]) * x[idx];
            }
            double mu = dhT ? dhT[bh * d + c] : 0.0;     /* gradient arriving from t + 1 */
            for (long t = T - 1; t >= 0; --t) {
                long idx = (bh * T + t) * d + c;
                mu += dy[idx];                               /* total dL/dh_t */
                dx[idx] = one_minus_gate(a[idx]) * mu;
                dg[idx] = mu * (h[t] - x[idx]);
                mu *= forget_gate(a[idx]);                   /* dL/dh_{t-1} through h_t */
            }
            if (dh0) dh0[bh * d + c] = mu;
        }
        free(h);
    }
}

/*
 * Backward of the fixed-window recurrence (rat_oracle_recurrence_window: y_t is the recurrence
 * restarted from zero at t - Lw + 1), for one of x = k or x = v.  Each output y_t is its own
 * restarted recurrence over the window W(t) = [max(t - Lw + 1, lo), t] (lo = -Lw with history
 * rows, else 0), so by the rule of rat_oracle_recurrence_backward applied to that recurrence alone,
 * with upstream gradient dy_t at its last row and nothing else,
 *   nu = dy_t at s = t,   then for s = t, t-1, ..., start:
 *     dL/dx_s += (1 - g_s) nu,   dL/dg_s += nu (h^t_{s-1} - x_s),   nu <- g_s nu,
 * where h^t is the restarted state (h^t_{start-1} = 0), recomputed for every t.  The sums over t
 * are the gradients; O(T Lw^2) per channel.  dprev_x / dprev_g ([BH][Lw][d], or NULL) receive
 * the gradients of the history rows prev_x / prev_a (given only with them).
 */
void rat_oracle_recurrence_window_backward(long BH, long T, long d, const double *x,
                                           const double *a, const double *prev_x,
                                           const double *prev_a, long Lw, const double *dy,
                                           double *dx, double *dg, double *dprev_x,
                                           double *dprev_g)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *hs = (double *)malloc((size_t)(Lw + 1) * sizeof(double));  /* hs[i] = state before row start+i */
        double *xs = (double *)malloc((size_t)Lw * sizeof(double));
        double *gs = (double *)malloc((size_t)Lw * sizeof(double));
        double *os = (double *)malloc((size_t)Lw * sizeof(double));
        for (long c = 0; c < d; ++c) {
            for (long t = 0; t < T; ++t) {
                dx[(bh * T + t) * d + c] = 0.0;
                dg[(bh * T + t) * d + c] = 0.0;
            }
            if (dprev_x)
                for (long i = 0; i < Lw; ++i) {
                    dprev_x[(bh * Lw + i) * d + c] = 0.0;
                    dprev_g[(bh * Lw + i) * d + c] = 0.0;
                }
            for (long t = 0; t < T; ++t) {
                long start = t - Lw + 1;
                long lo = prev_x ? -Lw : 0;
                if (start < lo) start = lo;
                long n = t - start + 1;
                /* the window's inputs, oldest first, and its restarted forward states */
                hs[0] = 0.0;
                for (long i = 0; i < n; ++i) {
                    long s = start + i;
                    double xv, av;
                    if (s >= 0) {
                        xv = x[(bh * T + s) * d + c];
                        av = a[(bh * T + s) * d + c];
                    } else {
                        xv = prev_x[(bh * Lw + (Lw + s)) * d + c];
                        av = prev_a[(bh * Lw + (Lw + s)) * d + c];
                    }
                    xs[i] = xv;
                    gs[i] = forget_gate(av);
                    os[i] = one_minus_gate(av);
                    hs[i + 1] = gs[i] * hs[i] + os[i] * xv;
                }
                double nu = dy[(bh * T + t) * d + c];         /* dL/dh^t_s, from s = t down */
                for (long i = n - 1; i >= 0; --i) {
                    long s = start + i;
                    double ddx = os[i] * nu, ddg = nu * (hs[i] - xs[i]);
                    if (s >= 0) {
                        dx[(bh * T + s) * d + c] += ddx;
                        dg[(bh * T + s) * d + c] += ddg;
                    } else if (dprev_x) {
                        dprev_x[(bh * Lw + (Lw + s)) * d + c] += ddx;
                        dprev_g[(bh * Lw + (Lw + s)) * d + c] += ddg;
                    }
                    nu *= gs[i];
                }
            }
        }
        free(hs);
        free(xs);
        free(gs);
        free(os);
    }
}

/*
 * Backward of the chunk-local recurrence (RAT: the state restarts before every absolute
 * position pos0 + t that is a multiple of L; "RAT+ Deep Dive" section 2.1), for one of x = k or
 * x = v.  Forward: hs_t = 0 if (pos0 + t) mod L == 0, else h_{t-1} (h_{-1} = h0), then
 * h_t = g_t hs_t + (1 - g_t) x_t.  Reverse-mode derivative: the total gradient of h_t is
 *   mu_t = dy_t + [pos0 + t + 1 is not a block start] g_{t+1} mu_{t+1},  mu_{T-1} = dy_{T-1} + dhT,
 * and  dL/dx_t = (1 - g_t) mu_t,  dL/dg_t = mu_t (hs_t - x_t),
 *      dL/dh0 = [pos0 is not a block start] g_0 mu_0   (h0 reaches only rows before a restart).
 * hs is recomputed by the forward loop; dg as in rat_oracle_recurrence_backward.
 */
void rat_oracle_recurrence_backward_reset(long BH, long T, long d, const double *x,
                                          const double *a, const double *h0, const double *dy,
                                          const double *dhT, long pos0, long L, double *dx,
                                          double *dg, double *dh0)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        double *hs = (double *)malloc((size_t)(T + 1) * sizeof(double));  /* state entering t */
        for (long c = 0; c < d; ++c) {
            double h = h0 ? h0[bh * d + c] : 0.0;
            for (long t = 0; t < T; ++t) {
                long idx = (bh * T + t) * d + c;
                if ((pos0 + t) % L == 0) h = 0.0;                /* a block starts at row t */
                hs[t] = h;
                h = forget_gate(a[idx]) * h + one_minus_gate(a[idx]) * x[idx];
            }
            double mu = dhT ? dhT[bh * d + c] : 0.0;         /* gradient arriving from t + 1 */
            for (long t = T - 1; t >= 0; --t) {
                long idx = (bh * T + t) * d + c;
                mu += dy[idx];                               /* total dL/dh_t */
                dx[idx] = one_minus_gate(a[idx]) * mu;
                dg[idx] = mu * (hs[t] - x[idx]);
                /* dL/dh_{t-1}: through h_t, unless the state was restarted at row t */
                mu = (pos0 + t) % L == 0 ? 0.0 : mu * forget_gate(a[idx]);
            }
            if (dh0) dh0[bh * d + c] = mu;
        }
        free(hs);
    }
}

/*
 * Rotary position embedding, rotate-half pairing, in place.                  [RoFormer]
 *   x : [BH][T][d];  position of row t is pos0 + t;  for c < d/2:
 *   theta_c = base^(-2c/d),  phi = (pos0 + t) * theta_c,
 *   (x_c, x_{c+d/2}) <- (x_c cos phi - x_{c+d/2} sin phi,  x_{c+d/2} cos phi + x_c sin phi).
 */
void rat_oracle_rope(long BH, long T, long d, double *x, long pos0, double base)
{
    long half = d / 2;
#pragma omp parallel for schedule(static)
    for (long bh = 0; bh < BH; ++bh) {
        for (long t = 0; t < T; ++t) {
            double *row = x + (bh * T + t) * d;
            for (long c = 0; c < half; ++c) {
                double theta = pow(base, -2.0 * (double)c / (double)d);
                double phi = (double)(pos0 + t) * theta;
                double cs = cos(phi), sn = sin(phi);
                double x1 = row[c], x2 = row[c + half];
                row[c] = x1 * cs - x2 * sn;
                row[c + half] = x2 * cs + x1 * sn;
            }
        }
    }
}

/* Effective window: a query always sees at least itself.                                     */
static long eff_window(long W) { return W > 1 ? W : 1; }

/*
 * Membership of key j in the key set of query t (the definition, as a predicate), with
 * n_sink attention sinks: the first n_sink positions, always attended (StreamingLLM layers,
 * "RAT+ Deep Dive" section 6 layer-wise hybrid).  n_sink = 0 is the RAT+ key set.
 *                                                     [RAT+ abstract; RAT+ Deep Dive 3.1, 6]
 */
int rat_oracle_in_key_set_sinks(long t, long j, long D, long W, long n_sink)
{
    long We = eff_window(W);
    if (j < 0 || j > t) return 0;
    if (j > t - We) return 1;            /* local window, the query's own position included */
    if (j < n_sink) return 1;            /* attention sink                                   */
    return (j % D) == (D - 1);           /* dilated key: a chunk end older than the window  */
}

int rat_oracle_in_key_set(long t, long j, long D, long W)
{
    return rat_oracle_in_key_set_sinks(t, j, D, W, 0);
}

/* |S(t)|: number of keys query t attends to, counted by enumerating the set.                */
long rat_oracle_key_count_sinks(long t, long D, long W, long n_sink)
{
    long n = 0;
    for (long j = 0; j <= t; ++j) n += rat_oracle_in_key_set_sinks(t, j, D, W, n_sink);
    return n;
}

long rat_oracle_key_count(long t, long D, long W) { return rat_oracle_key_count_sinks(t, D, W, 0); }

/*
 * S(t) listed in the order the loops below use: the window t-We < j <= t, then the chunk ends
 * j = D-1, 2D-1, ... with j <= t-We, then the sinks j < n_sink older than the window that are not
 * chunk ends (each key once).  Returns |S(t)|.
 */
static long list_keys(long t, long D, long We, long n_sink, long *keys)
{
    long n = 0;
    for (long j = (t - We + 1 > 0 ? t - We + 1 : 0); j <= t; ++j) keys[n++] = j;
    for (long j = D - 1; j <= t - We; j += D) keys[n++] = j;
    for (long j = 0; j < n_sink && j <= t - We; ++j)
        if (j % D != D - 1) keys[n++] = j;
    return n;
}

/*
 * Causal dilated attention with an optional local window and a per-(batch,head) dilation.
 *                                   [RAT+ abstract; RAT+ Deep Dive 3.1 table, 6 Head-Wise Hybrid]
 *   q, k, v : [BH][T][d]  (q and k already rotated if RoPE is in use; k, v are the recurrence
 *                          outputs k~, v~)
 *   Dbh     : [BH]        dilation of each (batch, head) slice
 *   rows    : [nrows]     query positions to evaluate (NULL: all T rows, nrows = T)
 *   o       : [BH][nrows][d]
 *   lse     : [BH][nrows] or NULL: log2 of sum_j exp(s_j), the softmax denominator in base-2
 *             units (what the backward needs to rebuild the weights)
 * For each query t:  s_j = scale * <q_t, k_j>  for j in S(t);
 *                    o_t = sum_j exp(s_j - max s) v_j / sum_j exp(s_j - max s).
 * S(t) is enumerated as its two parts: the window t-We < j <= t, then the chunk ends
 * j = D-1, 2D-1, ... with j <= t - We.
 */
void rat_oracle_dilated_attention(long BH, long T, long d, const double *q, const double *k,
                                  const double *v, const int *Dbh, long W, long n_sink,
                                  double scale, const long *rows, long nrows, double *o,
                                  double *lse)
{
    long We = eff_window(W);
    if (!rows) nrows = T;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        long D = Dbh[bh];
        long *keys = (long *)malloc(sizeof(long) * (size_t)(T + 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(T + 1));
        for (long r = 0; r < nrows; ++r) {
            long t = rows ? rows[r] : r;
            long n = list_keys(t, D, We, n_sink, keys);
            const double *qt = q + (bh * T + t) * d;
            double mx = -INFINITY;
            for (long m = 0; m < n; ++m) {
                const double *kj = k + (bh * T + keys[m]) * d;
                double dot = 0.0;
                for (long c = 0; c < d; ++c) dot += qt[c] * kj[c];
                s[m] = scale * dot;
                if (s[m] > mx) mx = s[m];
            }
            double *ot = o + (bh * nrows + r) * d;
            for (long c = 0; c < d; ++c) ot[c] = 0.0;
            double l = 0.0;
            for (long m = 0; m < n; ++m) {
                double p = exp(s[m] - mx);
                const double *vj = v + (bh * T + keys[m]) * d;
                l += p;
                for (long c = 0; c < d; ++c) ot[c] += p * vj[c];
            }
            for (long c = 0; c < d; ++c) ot[c] /= l;
            /* log2 of the softmax denominator sum_j 2^(s_j log2 e): (max s + ln l) / ln 2 */
            if (lse) lse[bh * nrows + r] = (mx + log(l)) / log(2.0);
        }
        free(keys);
        free(s);
    }
}

/*
 * Dilated attention with top-k chunk selection ("RAT+ Deep Dive" section 4: dilation combined
 * with top-k block selection, dilation reaching the whole sequence and the selected blocks adding
 * dense local detail).  Read as: the blocks are the dilation's chunks c = [cD, cD + D - 1]; a chunk wholly
 * older than the window (cD + D - 1 <= t - We) is scored by its chunk-end key,
 * s_c = scale * <q_t, k_{cD+D-1}>; the top_k highest-scoring chunks (ties: the earlier chunk)
 * are attended at every position, on top of S(t) (and the sinks), each key once.
 * Arguments as rat_oracle_dilated_attention (all rows), plus top_k >= 0.
 */
void rat_oracle_topk_attention(long BH, long T, long d, const double *q, const double *k,
                               const double *v, const int *Dbh, long W, long n_sink, long top_k,
                               double scale, double *o)
{
    long We = eff_window(W);
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        long D = Dbh[bh];
        long *keys = (long *)malloc(sizeof(long) * (size_t)(T + 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(T + 1));
        double *cs = (double *)malloc(sizeof(double) * (size_t)(T / D + 1));
        char *taken = (char *)malloc((size_t)(T / D + 1));
        for (long t = 0; t < T; ++t) {
            long n = list_keys(t, D, We, n_sink, keys);
            const double *qt = q + (bh * T + t) * d;
            long nc = t - We + 1 >= D ? (t - We + 1) / D : 0;       /* candidate chunks */
            for (long c = 0; c < nc; ++c) {
                const double *kj = k + (bh * T + c * D + D - 1) * d;
                double dot = 0.0;
                for (long x = 0; x < d; ++x) dot += qt[x] * kj[x];
                cs[c] = scale * dot;
                taken[c] = 0;
            }
            for (long r = 0; r < top_k && r < nc; ++r) {            /* r-th best: a plain scan */
                long best = -1;
                for (long c = 0; c < nc; ++c)
                    if (!taken[c] && (best < 0 || cs[c] > cs[best])) best = c;
                taken[best] = 1;
                for (long j = best * D; j < best * D + D - 1; ++j)
                    if (j >= n_sink) keys[n++] = j;                 /* sinks are listed already */
            }
            double mx = -INFINITY;
            for (long m = 0; m < n; ++m) {
                const double *kj = k + (bh * T + keys[m]) * d;
                double dot = 0.0;
                for (long x = 0; x < d; ++x) dot += qt[x] * kj[x];
                s[m] = scale * dot;
                if (s[m] > mx) mx = s[m];
            }
            double *ot = o + (bh * T + t) * d, l = 0.0;
            for (long x = 0; x < d; ++x) ot[x] = 0.0;
            for (long m = 0; m < n; ++m) {
                double p = exp(s[m] - mx);
                const double *vj = v + (bh * T + keys[m]) * d;
                l += p;
                for (long x = 0; x < d; ++x) ot[x] += p * vj[x];
            }
            for (long x = 0; x < d; ++x) ot[x] /= l;
        }
        free(keys);
        free(s);
        free(cs);
        free(taken);
    }
}

/*
 * Backward of the dilated attention above (its reverse-mode derivative), for upstream
 * gradients dO of the outputs.  Per query t, with p_j the softmax weights over S(t) and
 * o_t = sum_j p_j v_j:
 *   dv_j += p_j dO_t;   dp_j = <dO_t, v_j>;   ds_j = p_j (dp_j - <dO_t, o_t>);
 *   dq_t  = scale * sum_j ds_j k_j;   dk_j += scale * ds_j q_t.
 * q, k as used by the attention (already rotated); dq, dk, dv are accumulated into arrays the
 * caller zeroes.  o_t is recomputed here from the definition.
 */
void rat_oracle_dilated_attention_backward(long BH, long T, long d, const double *q,
                                           const double *k, const double *v, const double *dO,
                                           const int *Dbh, long W, long n_sink, double scale,
                                           double *dq, double *dk, double *dv)
{
    long We = eff_window(W);
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {           /* slices are independent: no shared writes */
        long D = Dbh[bh];
        long *keys = (long *)malloc(sizeof(long) * (size_t)(T + 1));
        double *p = (double *)malloc(sizeof(double) * (size_t)(T + 1));
        double *ot = (double *)malloc(sizeof(double) * (size_t)d);
        for (long t = 0; t < T; ++t) {
            long n = list_keys(t, D, We, n_sink, keys);
            const double *qt = q + (bh * T + t) * d;
            const double *gt = dO + (bh * T + t) * d;
            double mx = -INFINITY;
            for (long m = 0; m < n; ++m) {
                const double *kj = k + (bh * T + keys[m]) * d;
                double dot = 0.0;
                for (long c = 0; c < d; ++c) dot += qt[c] * kj[c];
                p[m] = scale * dot;
                if (p[m] > mx) mx = p[m];
            }
            double l = 0.0;
            for (long m = 0; m < n; ++m) {
                p[m] = exp(p[m] - mx);
                l += p[m];
            }
            for (long c = 0; c < d; ++c) ot[c] = 0.0;
            for (long m = 0; m < n; ++m) {
                p[m] /= l;
                const double *vj = v + (bh * T + keys[m]) * d;
                for (long c = 0; c < d; ++c) ot[c] += p[m] * vj[c];
            }
            double delta = 0.0;                          /* <dO_t, o_t> */
            for (long c = 0; c < d; ++c) delta += gt[c] * ot[c];
            double *dqt = dq + (bh * T + t) * d;
            for (long m = 0; m < n; ++m) {
                long j = keys[m];
                const double *kj = k + (bh * T + j) * d;
                const double *vj = v + (bh * T + j) * d;
                double dp = 0.0;
                for (long c = 0; c < d; ++c) dp += gt[c] * vj[c];
                double ds = p[m] * (dp - delta);
                double *dkj = dk + (bh * T + j) * d;
                double *dvj = dv + (bh * T + j) * d;
                for (long c = 0; c < d; ++c) {
                    dqt[c] += scale * ds * kj[c];
                    dkj[c] += scale * ds * qt[c];
                    dvj[c] += p[m] * gt[c];
                }
            }
        }
        free(keys);
        free(p);
        free(ot);
    }
}

/*
 * Compressed KV cache build, on raw element bytes (bit-exact gather).      [RAT+ abstract]
 *   x    : [B][H][T][d] elements of esize bytes: the recurrence outputs of positions
 *          pos0 .. pos0+T-1
 *   Dh   : [H] per-head dilation;  cap_h = floor(Tcap / D_h);  off_h = sum_{h' < h} cap_h'
 *   dil  : [B][sum_h cap_h][d]   entry i of head h = position i*D_h + D_h - 1
 *   ring : [B][H][W][d]          position p lives in slot p mod W  (ring may be NULL if W == 0)
 * Every position p of this chunk with p mod D_h = D_h - 1 and p / D_h < cap_h is stored in
 * dil; every position among the last W of the sequence so far is stored in ring.
 */
void rat_oracle_kv_compress(long B, long H, long T, long d, long esize, const uint8_t *x,
                            const int *Dh, long W, long Tcap, long pos0, uint8_t *dil,
                            uint8_t *ring)
{
    long total_cap = 0;
    for (long h = 0; h < H; ++h) total_cap += Tcap / Dh[h];
    long row_bytes = d * esize;
    for (long b = 0; b < B; ++b) {
        long off = 0;
        for (long h = 0; h < H; ++h) {
            long D = Dh[h], cap = Tcap / D;
            for (long t = 0; t < T; ++t) {
                long p = pos0 + t;
                const uint8_t *src = x + ((b * H + h) * T + t) * row_bytes;
                if (p % D == D - 1 && p / D < cap)
                    memcpy(dil + (b * total_cap + off + p / D) * row_bytes, src, (size_t)row_bytes);
                if (W > 0 && p >= pos0 + T - W)
                    memcpy(ring + ((b * H + h) * W + p % W) * row_bytes, src, (size_t)row_bytes);
            }
            off += cap;
        }
    }
}

/*
 * One decode step for a new token at absolute position t, per (batch, head) slice.
 *                                           [RAT+ Deep Dive 2.1; RAT+ abstract; RoFormer]
 *   q, k, v, a   : [BH][d]          the new token's query, key, value, gate logit
 *   hk, hv       : [BH][d]          recurrence state (before RoPE), updated in place
 *   khist, vhist : [BH][Tcap][d]    every earlier k~ (rotated) and v~; row t is written here
 *   Dbh          : [BH]             dilation per slice
 *   o            : [BH][d]
 * State update h = g*h + (1-g)*x for k and v; k~_t = RoPE(h_k, t) (if rope_base > 0); the
 * query is RoPE(q, t); attention over S(t) exactly as in the prefill definition.
 */
void rat_oracle_decode_step(long BH, long d, long t, const int *Dbh, long W, long n_sink,
                            double scale,
                            double rope_base, const double *q, const double *k, const double *v,
                            const double *a, double *hk, double *hv, double *khist,
                            double *vhist, long Tcap, double *o)
{
    long We = eff_window(W);
    long half = d / 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < BH; ++bh) {
        long D = Dbh[bh];
        double *kt = khist + (bh * Tcap + t) * d;
        double *vt = vhist + (bh * Tcap + t) * d;
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        for (long c = 0; c < d; ++c) {
            long idx = bh * d + c;
            double g = forget_gate(a[idx]), omg = one_minus_gate(a[idx]);
            hk[idx] = g * hk[idx] + omg * k[idx];
            hv[idx] = g * hv[idx] + omg * v[idx];
            kt[c] = hk[idx];
            vt[c] = hv[idx];
            qr[c] = q[idx];
        }
        if (rope_base > 0.0) {
            for (long c = 0; c < half; ++c) {
                double theta = pow(rope_base, -2.0 * (double)c / (double)d);
                double phi = (double)t * theta, cs = cos(phi), sn = sin(phi);
                double x1 = kt[c], x2 = kt[c + half];
                kt[c] = x1 * cs - x2 * sn;
                kt[c + half] = x2 * cs + x1 * sn;
                x1 = qr[c];
                x2 = qr[c + half];
                qr[c] = x1 * cs - x2 * sn;
                qr[c + half] = x2 * cs + x1 * sn;
            }
        }
        long nmax = We + t / D + n_sink + 2;
        long *keys = (long *)malloc(sizeof(long) * (size_t)nmax);
        double *s = (double *)malloc(sizeof(double) * (size_t)nmax);
        long n = list_keys(t, D, We, n_sink, keys);
        double mx = -INFINITY;
        for (long m = 0; m < n; ++m) {
            const double *kj = khist + (bh * Tcap + keys[m]) * d;
            double dot = 0.0;
            for (long c = 0; c < d; ++c) dot += qr[c] * kj[c];
            s[m] = scale * dot;
            if (s[m] > mx) mx = s[m];
        }
        double *ot = o + bh * d, l = 0.0;
        for (long c = 0; c < d; ++c) ot[c] = 0.0;
        for (long m = 0; m < n; ++m) {
            double p = exp(s[m] - mx);
            const double *vj = vhist + (bh * Tcap + keys[m]) * d;
            l += p;
            for (long c = 0; c < d; ++c) ot[c] += p * vj[c];
        }
        for (long c = 0; c < d; ++c) ot[c] /= l;
        free(keys);
        free(s);
        free(qr);
    }
}

/* Number of OpenMP threads the oracle will use (for reporting the CPU baseline's cores).     */
#ifdef _OPENMP
#include <omp.h>
int rat_oracle_threads(void) { return omp_get_max_threads(); }
void rat_oracle_set_threads(int n) { omp_set_num_threads(n); }
#else
int rat_oracle_threads(void) { return 1; }
void rat_oracle_set_threads(int n) { (void)n; }
#endif
