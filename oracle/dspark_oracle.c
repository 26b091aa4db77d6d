/*
 * dspark_oracle.c -- plain, slow, single-threaded fp64 restatement of the
 * per-round token path of DSpark (arXiv:2607.05147).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it.  It shares no code, header, table or helper
 * with the CUDA library and includes nothing from it.
 *
 * Sources (web pages about the paper), cited below by tag:
 *   [PL] paperlayer.ai, "DSpark: Confidence-Scheduled Speculative Decoding with
 *        Semi-Autoregressive Generation" (section-by-section summary):
 *        §2 Background, §3.1 Semi-autoregressive generation, §3.2
 *        Confidence-scheduled verification, Appendix A (counterexample:
 *        selection bias without early stopping).
 *   [KB] menfem.com knowledge-base entry on the same paper: "Key
 *        Contributions" and "Methodology".
 *   [WK] llm-wiki.hwlabs.dev study 116 on DSpark: the draft-generation
 *        figure of the semi-autoregressive Markov head section, and the
 *        confidence-scheduling section.
 *
 * Arithmetic: every input (fp32, or bf16 values carried exactly in fp32) is
 * widened to double; all sums run sequentially in index order; exp() is the C
 * library's.  No blocking, fusion or reordering beyond the definitions.
 *
 * Readings where the pages are silent:
 *   - the Markov bias at position i is U[x_{i-1}] W with x_0 the last committed
 *     token, also at i = 1;
 *   - temperature T scales draft and target logits alike; T = 0 means greedy
 *     (argmax, lowest index on ties) with the exact-match accept rule;
 *   - inverse-CDF sampling takes the smallest v with u < C_v;
 *   - accept iff u < p_t(x)/p_d(x), i.e. with probability min(1, ratio);
 *   - the scheduler objective is Theta(n) = (B + sum of admitted S) / t(n);
 *     it stops at the first strict decrease (cross-multiplied compare);
 *   - candidates are laid out position-major and sorted stably by S
 *     descending, so ties go to the lower position, then the lower request;
 *   - an all-zero residual falls back to sampling from p_t.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ------------------------------------------------------------------------ */
/* Markov transition bias: [PL] §3.1 (a low-rank transition matrix conditions
 * each position on the previously sampled token); [KB] Methodology (rank-256
 * factorization); [WK] draft-generation figure (final logits L[i] + Delta[i]).
 * delta[v] = sum_k U[a][k] * W[k][v], with U stored [V][r] and W stored [r][V]. */
static void markov_bias_row(const float *U, const float *W, int V, int r, int a,
                            double *delta)
{
    for (int v = 0; v < V; ++v) delta[v] = 0.0;
    for (int k = 0; k < r; ++k) {
        double uk = (double)U[(size_t)a * r + k];
        const float *wk = W + (size_t)k * V;
        for (int v = 0; v < V; ++v) delta[v] += uk * (double)wk[v];
    }
}

/* Bias of draft position k (1-based) of one request, given its prefix
 * x_0 (last committed token) and xs[0..k-2] = x_1..x_{k-1}: [PL] §3.1 (the
 * sequential stage conditions each position on the tokens sampled before it;
 * a Markov head uses a low-rank transition matrix, an RNN head keeps a
 * recurrent state that summarises the whole prefix); [KB] Key Contributions
 * (Markov head: first-order dependency by a low-rank factorization; RNN head:
 * full within-block history).
 *   A == NULL (Markov head): Delta = U[x_{k-1}] W.
 *   A != NULL (RNN head, A stored [r][r]): the state h_0 = 0 and
 *     h_j[c] = tanh(sum_q h_{j-1}[q] A[q][c] + U[x_{j-1}][c]), j = 1..k;
 *     Delta = h_k W.  The pages give no equations for this head; this is
 *     the plainest recurrence over the same factors (a state of size r fed
 *     by the token's U row, read out through W).
 * h and hn are scratch rows of r doubles.  The state is recomputed from the
 * start of the block at every call (slow, and the same arithmetic wherever
 * the bias is needed). */
static void draft_bias(const float *U, const float *A, const float *W, int V, int r, int x0,
                       const int *xs, int k, double *h, double *hn, double *delta)
{
    if (A == NULL) {
        markov_bias_row(U, W, V, r, k == 1 ? x0 : xs[k - 2], delta);
        return;
    }
    for (int c = 0; c < r; ++c) h[c] = 0.0;
    for (int j = 1; j <= k; ++j) {
        int tok = (j == 1) ? x0 : xs[j - 2];
        for (int c = 0; c < r; ++c) {
            double a = 0.0;
            for (int q = 0; q < r; ++q) a += h[q] * (double)A[(size_t)q * r + c];
            a += (double)U[(size_t)tok * r + c];
            hn[c] = tanh(a);
        }
        for (int c = 0; c < r; ++c) h[c] = hn[c];
    }
    for (int v = 0; v < V; ++v) delta[v] = 0.0;
    for (int c = 0; c < r; ++c) {
        double hc = h[c];
        const float *wc = W + (size_t)c * V;
        for (int v = 0; v < V; ++v) delta[v] += hc * (double)wc[v];
    }
}

/* Index of the largest entry (lowest index on ties) and the gap to the
 * largest entry at any other index (the decision margin of an argmax). */
static int argmax_with_gap(const double *z, int V, double *gap)
{
    int best = 0;
    for (int v = 1; v < V; ++v)
        if (z[v] > z[best]) best = v;
    double second = -INFINITY;
    for (int v = 0; v < V; ++v)
        if (v != best && z[v] > second) second = z[v];
    *gap = (V > 1) ? z[best] - second : INFINITY;
    return best;
}

/* Inverse-CDF draw from non-negative weights e[0..V-1] with total tot:
 * the smallest v with u < C_v, C_v = (e_0 + ... + e_v) / tot.  margin is the
 * distance from u to the nearer end of the chosen interval.  If rounding
 * leaves u >= C_{V-1}, the last index with positive weight is taken. */
static int inverse_cdf(const double *e, int V, double tot, double u, double *margin)
{
    double run = 0.0, prev = 0.0;
    for (int v = 0; v < V; ++v) {
        run += e[v];
        double c = run / tot;
        if (u < c) {
            double m0 = u - prev, m1 = c - u;
            *margin = m0 < m1 ? m0 : m1;
            return v;
        }
        prev = c;
    }
    int last = V - 1;
    while (last > 0 && !(e[last] > 0.0)) --last;
    *margin = 0.0;
    return last;
}

/* Temperature softmax of one logit row: z = row / T, m = max z,
 * e_v = exp(z_v - m), returns Z = sum e_v.  T > 0. */
static double softmax_row(const double *row, int V, double T, double *e, double *m_out)
{
    double m = -INFINITY;
    for (int v = 0; v < V; ++v) {
        double z = row[v] / T;
        if (z > m) m = z;
    }
    double Z = 0.0;
    for (int v = 0; v < V; ++v) {
        e[v] = exp(row[v] / T - m);
        Z += e[v];
    }
    *m_out = m;
    return Z;
}

/* ------------------------------------------------------------------------ */
/* Stage 1, semi-autoregressive drafting: [PL] §3.1 (the parallel stage gives
 * all draft logits in one pass; the sequential stage samples left to right,
 * conditioning each position on the previously sampled token); [WK]
 * draft-generation figure (L[i] + Delta[i], then sample the draft token).
 *
 * L [B][G][V], U [V][r], W [r][V], A [r][r] or NULL (see draft_bias: NULL is
 * the Markov head, else the RNN head); x0 [B] last committed token per request;
 * temp [B]; u_draft [B][G] uniforms in [0,1).  force_x (nullable, [B][G]):
 * entries >= 0 replace the sampled token (used to follow another
 * implementation's decision after a reported near-tie).
 * Outputs per (b,i), with y = L + Delta and z = y / T: x, pd = p_d(x),
 * rowmax = max_v y_v (logit units, before the temperature), rowsum =
 * sum_v exp(z_v - max z), margin = decision margin.  For T = 0: x = argmax y,
 * pd = 1, rowmax = max y, rowsum = 1, margin = top-two gap. */
int dspark_oracle_draft_head(int B, int G, int V, int r, const float *L, const float *U,
                             const float *A, const float *W, const int *x0, const float *temp,
                             const double *u_draft, const int *force_x, int *x_out,
                             double *pd_out, double *rowmax_out, double *rowsum_out,
                             double *margin_out)
{
    if (B < 0 || G < 1 || V < 2 || r < 1) return ORACLE_ERR_ARG;
    double *delta = malloc(sizeof(double) * (size_t)V);
    double *y = malloc(sizeof(double) * (size_t)V);
    double *e = malloc(sizeof(double) * (size_t)V);
    double *h = malloc(sizeof(double) * (size_t)r * 2);
    if (!delta || !y || !e || !h) { free(delta); free(y); free(e); free(h); return ORACLE_ERR_NOMEM; }
    for (int b = 0; b < B; ++b) {
        if (x0[b] < 0 || x0[b] >= V) { free(delta); free(y); free(e); free(h); return ORACLE_ERR_ARG; }
        double T = (double)temp[b];
        for (int i = 0; i < G; ++i) {
            size_t o = (size_t)b * G + i;
            draft_bias(U, A, W, V, r, x0[b], x_out + (size_t)b * G, i + 1, h, h + r, delta);
            const float *Lrow = L + o * (size_t)V;
            for (int v = 0; v < V; ++v) y[v] = (double)Lrow[v] + delta[v];
            int x;
            if (T == 0.0) {
                double gap;
                x = argmax_with_gap(y, V, &gap);
                margin_out[o] = gap;
                rowmax_out[o] = y[x];
                rowsum_out[o] = 1.0;
                if (force_x && force_x[o] >= 0) x = force_x[o];
                pd_out[o] = 1.0;
            } else {
                double m, Z = softmax_row(y, V, T, e, &m), mg;
                x = inverse_cdf(e, V, Z, u_draft[o], &mg);
                margin_out[o] = mg;
                if (force_x && force_x[o] >= 0) x = force_x[o];
                double ymax = y[0];
                for (int v = 1; v < V; ++v)
                    if (y[v] > ymax) ymax = y[v];
                rowmax_out[o] = ymax;
                rowsum_out[o] = Z;
                pd_out[o] = e[x] / Z;
            }
            x_out[o] = x;
        }
    }
    free(delta); free(y); free(e); free(h);
    return ORACLE_OK;
}

/* The Markov-head drafting of [PL] §3.1 (the head of the headline path). */
int dspark_oracle_draft(int B, int G, int V, int r, const float *L, const float *U,
                        const float *W, const int *x0, const float *temp,
                        const double *u_draft, const int *force_x, int *x_out,
                        double *pd_out, double *rowmax_out, double *rowsum_out,
                        double *margin_out)
{
    return dspark_oracle_draft_head(B, G, V, r, L, U, NULL, W, x0, temp, u_draft, force_x, x_out, pd_out,
                                    rowmax_out, rowsum_out, margin_out);
}

/* The RNN head's states along drafted blocks (see draft_bias): for every
 * request b and position k = 1..G, h_k from x_0 and x_1..x_{k-1} of x [B][G].
 * Tokens index U [V][r]: any token outside [0, V) is an argument error.
 * Output h_out [B][G][r] (fp64). */
int dspark_oracle_rnn_states(int B, int G, int V, int r, const float *U, const float *Arec, const int *x0,
                             const int *x, double *h_out)
{
    if (B < 1 || G < 1 || V < 2 || r < 1 || !Arec) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        if (x0[b] < 0 || x0[b] >= V) return ORACLE_ERR_ARG;
        for (int k = 0; k + 1 < G; ++k)
            if (x[(size_t)b * G + k] < 0 || x[(size_t)b * G + k] >= V) return ORACLE_ERR_ARG;
    }
    double *h = malloc(sizeof(double) * (size_t)r);
    double *hn = malloc(sizeof(double) * (size_t)r);
    if (!h || !hn) { free(h); free(hn); return ORACLE_ERR_NOMEM; }
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < r; ++c) h[c] = 0.0;
        for (int k = 1; k <= G; ++k) {
            int tok = (k == 1) ? x0[b] : x[(size_t)b * G + k - 2];
            for (int c = 0; c < r; ++c) {
                double a = 0.0;
                for (int q = 0; q < r; ++q) a += h[q] * (double)Arec[(size_t)q * r + c];
                a += (double)U[(size_t)tok * r + c];
                hn[c] = tanh(a);
            }
            for (int c = 0; c < r; ++c) {
                h[c] = hn[c];
                h_out[((size_t)b * G + (k - 1)) * r + c] = hn[c];
            }
        }
    }
    free(h); free(hn);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Stage 2, confidence and prefix survival: [KB] Key Contributions (a
 * lightweight linear confidence head gives a per-position survival
 * probability); [PL] §3.2 (the head estimates the conditional survival of
 * each draft token; sequential temperature scaling calibrates the cumulative
 * products left to right); [WK] confidence-scheduling section (the survival
 * of position i is the probability that positions 1..i are all accepted).
 * c = sigmoid((w . h + bias) / tau_i), S_i = S_{i-1} c_i, S_0 = 1.
 * h [B][G][d], w [d], tau [G] or NULL (all ones). */
int dspark_oracle_confidence(int B, int G, int d, const float *h, const float *w,
                             double bias, const double *tau, double *c_out,
                             double *S_out)
{
    if (B < 0 || G < 1 || d < 1) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        double S = 1.0;
        for (int i = 0; i < G; ++i) {
            size_t o = (size_t)b * G + i;
            const float *hr = h + o * (size_t)d;
            double a = 0.0;
            for (int j = 0; j < d; ++j) a += (double)w[j] * (double)hr[j];
            a += bias;
            if (tau) a /= tau[i];
            double c = 1.0 / (1.0 + exp(-a));
            S *= c;
            c_out[o] = c;
            S_out[o] = S;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Throughput profile t(n): piecewise linear through the knots (n_j, t_j),
 * n_0 = 0, extended past the last knot with the last segment's slope
 * (constant if there is a single knot).  [PL] §1 and §3.2 (engine-specific
 * throughput profiles drive the verification length). */
static double profile_t(int P, const int *kn, const double *kt, double n)
{
    if (P == 1) return kt[0];
    int j = 0;
    while (j + 1 < P - 1 && n >= (double)kn[j + 1]) ++j;
    double slope = (kt[j + 1] - kt[j]) / (double)(kn[j + 1] - kn[j]);
    return kt[j] + (n - (double)kn[j]) * slope;
}

typedef struct { double s; int idx; } cand_t;

/* S descending; equal S keeps the position-major index order (stable). */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = pa, *b = pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

#define SCHED_ALL 0
#define SCHED_GREEDY_EARLY_STOP 1
#define SCHED_GLOBAL_ARGMAX 2 /* offline search of [PL] Appendix A: test-only negative control */

/* Stage 3, Algorithm 1 (hardware-aware prefix scheduler): [KB] Key
 * Contributions (greedy global sort of candidate tokens by cumulative
 * survival, incremental batch admission with early stopping that keeps
 * admissions causal); [PL] Appendix A (stop as soon as Theta_{n+1} < Theta_n;
 * admitting token k may only use information available before x_k is drawn;
 * with Theta_0 = 1.0 for one request and nothing admitted).
 *
 * S [B][G] survivals.  Candidates are indexed position-major, idx = i*B + b,
 * and sorted by S descending, ties by idx.  V_0 = B (every request emits at
 * least one token), Theta_0 = B / t(0); candidate n+1 is admitted unless
 * (V_n + S_(n+1)) t(n) < V_n t(n+1).  Admission also stops at `budget`
 * (budget < 0: none) and when every candidate is admitted.
 * mode ALL: every request gets ell = G.  mode GLOBAL_ARGMAX: the admitted
 * count maximises Theta over all n (no early stop).  force_n >= 0 replaces
 * the admitted count (used to follow another implementation after a
 * near-tie).  Outputs: ell [B], n_adm, theta (objective at the admitted
 * count), order [B*G] (sorted candidate indices), margin_theta (the
 * decision margin of the early stop, taken at the stop point: the relative
 * objective change |Theta_{n+1} - Theta_n| / Theta_n of the comparison that
 * ended admission; +inf when admission ended at the budget or with every
 * candidate admitted, or in the other modes), margin_gap (S gap across the
 * cut, +inf if nothing is cut), and margins (nullable, [B*G]): the relative
 * objective change of every comparison n the early stop made (n = 0..the
 * stop), NaN for comparisons not made -- the margin at another
 * implementation's stop point when it stopped earlier. */
int dspark_oracle_schedule(int B, int G, const double *S, int P, const int *knots_n,
                           const double *knots_t, int budget, int mode, int force_n,
                           int *ell_out, int *n_adm_out, double *theta_out,
                           int *order_out, double *margin_theta_out,
                           double *margin_gap_out, double *margins_out)
{
    if (B < 1 || G < 1 || P < 1 || knots_n[0] != 0) return ORACLE_ERR_ARG;
    int N = B * G;
    cand_t *c = malloc(sizeof(cand_t) * (size_t)N);
    if (!c) return ORACLE_ERR_NOMEM;
    for (int i = 0; i < G; ++i)
        for (int b = 0; b < B; ++b) {
            c[i * B + b].s = S[(size_t)b * G + i];
            c[i * B + b].idx = i * B + b;
        }
    qsort(c, (size_t)N, sizeof(cand_t), cand_cmp);
    if (order_out)
        for (int n = 0; n < N; ++n) order_out[n] = c[n].idx;
    if (margins_out)
        for (int n = 0; n < N; ++n) margins_out[n] = NAN;

    int limit = N;
    if (budget >= 0 && budget < limit) limit = budget;
    double Vn = (double)B;
    double theta = Vn / profile_t(P, knots_n, knots_t, 0.0);
    double mtheta = INFINITY;
    int n = 0;
    if (mode == SCHED_ALL) {
        n = N;
        for (int k = 0; k < N; ++k) Vn += c[k].s;
        theta = Vn / profile_t(P, knots_n, knots_t, (double)N);
    } else if (mode == SCHED_GREEDY_EARLY_STOP) {
        while (n < limit) {
            double t0 = profile_t(P, knots_n, knots_t, (double)n);
            double t1 = profile_t(P, knots_n, knots_t, (double)(n + 1));
            double Vn1 = Vn + c[n].s;
            double th1 = Vn1 / t1;
            double rel = fabs(th1 - theta) / theta;
            if (margins_out) margins_out[n] = rel;
            if (Vn1 * t0 < Vn * t1) { /* Theta_{n+1} < Theta_n: stop */
                mtheta = rel;
                break;
            }
            Vn = Vn1;
            theta = th1;
            ++n;
        }
    } else if (mode == SCHED_GLOBAL_ARGMAX) {
        double best = theta, run = Vn;
        int bestn = 0;
        for (int k = 0; k < limit; ++k) {
            run += c[k].s;
            double th = run / profile_t(P, knots_n, knots_t, (double)(k + 1));
            if (th > best) { best = th; bestn = k + 1; }
        }
        n = bestn;
        theta = best;
    } else {
        free(c);
        return ORACLE_ERR_ARG;
    }
    if (force_n >= 0 && force_n <= N) {
        n = force_n;
        Vn = (double)B;
        for (int k = 0; k < n; ++k) Vn += c[k].s;
        theta = Vn / profile_t(P, knots_n, knots_t, (double)n);
    }
    for (int b = 0; b < B; ++b) ell_out[b] = 0;
    for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;
    *n_adm_out = n;
    *theta_out = theta;
    *margin_theta_out = mtheta;
    *margin_gap_out = (n > 0 && n < N) ? fabs(c[n - 1].s - c[n].s) : INFINITY;
    free(c);
    return ORACLE_OK;
}

/* Static-threshold pruning, a scheduler variant ([KB] Key Contributions:
 * candidates ranked by cumulative survival; the threshold form prunes by a
 * fixed survival level instead of the objective): in the same sorted order as
 * above, admit the candidates with S >= threshold, at most `budget`
 * (budget < 0: none).  Because the order is by S descending, the admitted
 * candidates are exactly those with S >= threshold (up to the budget), and a
 * request's admitted positions are a prefix whenever its S is non-increasing.
 * Outputs ell [B], n_adm, order [B*G]. */
int dspark_oracle_schedule_threshold(int B, int G, const double *S, double threshold, int budget, int *ell_out,
                                     int *n_adm_out, int *order_out)
{
    if (B < 1 || G < 1) return ORACLE_ERR_ARG;
    int N = B * G;
    cand_t *c = malloc(sizeof(cand_t) * (size_t)N);
    if (!c) return ORACLE_ERR_NOMEM;
    for (int i = 0; i < G; ++i)
        for (int b = 0; b < B; ++b) {
            c[i * B + b].s = S[(size_t)b * G + i];
            c[i * B + b].idx = i * B + b;
        }
    qsort(c, (size_t)N, sizeof(cand_t), cand_cmp);
    if (order_out)
        for (int n = 0; n < N; ++n) order_out[n] = c[n].idx;
    int limit = N;
    if (budget >= 0 && budget < limit) limit = budget;
    int n = 0;
    while (n < limit && c[n].s >= threshold) ++n;
    for (int b = 0; b < B; ++b) ell_out[b] = 0;
    for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;
    *n_adm_out = n;
    free(c);
    return ORACLE_OK;
}

/* Dynamic top-K admission, the production scheduler's selection step ([PL]
 * §5.2 Production Scheduler: asynchronous; the capacity limit comes from
 * historical predictions, the current candidates are ranked by their latest
 * cumulative confidence, and a dynamic top-K selection keeps the confidence
 * ordering).  In the same sorted order as above, admit the first K candidates,
 * K = capacity clamped to [0, B*G], at most `budget` (budget < 0: none).  The
 * capacity itself is an input: the production form computes it from an
 * earlier round (the global search over the profile on that round's
 * survivals), so the count does not look at the current round at all.
 * Outputs ell [B], n_adm, order [B*G]. */
int dspark_oracle_schedule_topk(int B, int G, const double *S, int capacity, int budget, int *ell_out,
                                int *n_adm_out, int *order_out)
{
    if (B < 1 || G < 1) return ORACLE_ERR_ARG;
    int N = B * G;
    cand_t *c = malloc(sizeof(cand_t) * (size_t)N);
    if (!c) return ORACLE_ERR_NOMEM;
    for (int i = 0; i < G; ++i)
        for (int b = 0; b < B; ++b) {
            c[i * B + b].s = S[(size_t)b * G + i];
            c[i * B + b].idx = i * B + b;
        }
    qsort(c, (size_t)N, sizeof(cand_t), cand_cmp);
    if (order_out)
        for (int n = 0; n < N; ++n) order_out[n] = c[n].idx;
    int n = capacity < 0 ? 0 : (capacity > N ? N : capacity);
    if (budget >= 0 && budget < n) n = budget;
    for (int b = 0; b < B; ++b) ell_out[b] = 0;
    for (int k = 0; k < n; ++k) ell_out[c[k].idx % B] += 1;
    *n_adm_out = n;
    free(c);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Stage 4, exact rejection-sampling verification: [KB] Methodology (x_k is
 * accepted with probability min(1, p_t(x_k)/p_d(x_k)); the first rejection
 * discards every later token; the output stays distributed as the target);
 * [PL] §2 (the longest consistent prefix is kept, verification runs left to
 * right); [PL] Appendix A (with nothing admitted the target draws a fresh
 * token from p_t).  On a rejection at k* the replacement is drawn from the
 * normalised residual max(0, p_t - p_d) at k*; if every admitted token is
 * accepted a bonus token is drawn from p_t at row ell+1.
 *
 * Tlog [B][G+1][V] target logits (row k verifies x_k; row G+1 is the bonus
 * row), L, U, W, x0 as for drafting, x [B][G] draft tokens, temp [B],
 * u_accept [B][G], u_final [B], ell [B] admitted counts.  The draft
 * probabilities are recomputed here from L, U, W and x (fp64), not taken
 * from the drafting stage.  force_accept (nullable, [B][G]): entries 0/1
 * replace the accept decision at that position.
 * Outputs: acc [B] accepted count A, tokens [B][G+1] = x_1..x_A, y, then -1,
 * nout [B] = A+1, pt_x / pd_x [B][G] = p_t(x_k), p_d(x_k) for k <= ell (NaN
 * elsewhere; for T = 0 both are 1 when the argmax matches, else 0 / 1),
 * margin_acc [B][G] (|u - ratio|, or the top-two gap for T = 0; +inf beyond
 * ell), margin_fin [B], final_kind [B]: 0 residual, 1 bonus/fresh token,
 * 2 greedy, 3 residual that was all zero (drawn from p_t). */
int dspark_oracle_verify_head(int B, int G, int V, int r, const float *Tlog, const float *L,
                              const float *U, const float *Arec, const float *W, const int *x0, const int *x,
                              const float *temp, const double *u_accept,
                              const double *u_final, const int *ell,
                              const int *force_accept, int *acc_out, int *tokens_out,
                              int *nout_out, double *pt_x_out, double *pd_x_out,
                              double *margin_acc_out, double *margin_fin_out,
                              int *final_kind_out)
{
    if (B < 0 || G < 1 || V < 2 || r < 1) return ORACLE_ERR_ARG;
    double *hs = malloc(sizeof(double) * (size_t)r * 2);
    if (!hs) return ORACLE_ERR_NOMEM;
    double *delta = malloc(sizeof(double) * (size_t)V);
    double *yd = malloc(sizeof(double) * (size_t)V);
    double *yt = malloc(sizeof(double) * (size_t)V);
    double *ed = malloc(sizeof(double) * (size_t)V);
    double *et = malloc(sizeof(double) * (size_t)V);
    double *q = malloc(sizeof(double) * (size_t)V);
    if (!delta || !yd || !yt || !ed || !et || !q) {
        free(delta); free(yd); free(yt); free(ed); free(et); free(q); free(hs);
        return ORACLE_ERR_NOMEM;
    }
    int rc = ORACLE_OK;
    for (int b = 0; b < B && rc == ORACLE_OK; ++b) {
        double T = (double)temp[b];
        int lb = ell[b];
        if (lb < 0 || lb > G) { rc = ORACLE_ERR_ARG; break; }
        for (int k = 0; k < G; ++k) {
            size_t o = (size_t)b * G + k;
            pt_x_out[o] = NAN;
            pd_x_out[o] = NAN;
            margin_acc_out[o] = INFINITY;
        }
        /* Per admitted position: target and draft probability of x_k. */
        int A = 0, rejected = 0;
        for (int k = 1; k <= lb; ++k) {
            size_t o = (size_t)b * G + (k - 1);
            int xk = x[o];
            const float *Trow = Tlog + ((size_t)b * (G + 1) + (k - 1)) * (size_t)V;
            for (int v = 0; v < V; ++v) yt[v] = (double)Trow[v];
            int accept;
            if (T == 0.0) {
                double gap;
                int am = argmax_with_gap(yt, V, &gap);
                accept = (am == xk);
                /* The decision flips only if x_k and the argmax swap: margin is
                 * the distance between z[x_k] and the best other entry. */
                double best_other = -INFINITY;
                for (int v = 0; v < V; ++v)
                    if (v != xk && yt[v] > best_other) best_other = yt[v];
                margin_acc_out[o] = fabs(yt[xk] - best_other);
                pt_x_out[o] = accept ? 1.0 : 0.0;
                pd_x_out[o] = 1.0;
            } else {
                double mt, Zt = softmax_row(yt, V, T, et, &mt);
                draft_bias(U, Arec, W, V, r, x0[b], x + (size_t)b * G, k, hs, hs + r, delta);
                const float *Lrow = L + o * (size_t)V;
                for (int v = 0; v < V; ++v) yd[v] = (double)Lrow[v] + delta[v];
                double md, Zd = softmax_row(yd, V, T, ed, &md);
                double pt = et[xk] / Zt, pd = ed[xk] / Zd;
                double ratio = pt / pd;
                accept = u_accept[o] < ratio;
                margin_acc_out[o] = fabs(u_accept[o] - ratio);
                pt_x_out[o] = pt;
                pd_x_out[o] = pd;
            }
            if (force_accept && force_accept[o] >= 0) accept = force_accept[o] ? 1 : 0;
            if (!rejected) {
                if (accept) ++A;
                else rejected = 1;
            }
        }
        /* Final token from row k* = A + 1 (1-based). */
        int ks = A + 1;
        const float *Trow = Tlog + ((size_t)b * (G + 1) + (ks - 1)) * (size_t)V;
        for (int v = 0; v < V; ++v) yt[v] = (double)Trow[v];
        int yv, kind;
        double mfin;
        if (T == 0.0) {
            yv = argmax_with_gap(yt, V, &mfin);
            kind = 2;
        } else {
            double mt, Zt = softmax_row(yt, V, T, et, &mt);
            if (A < lb) {
                size_t o = (size_t)b * G + (ks - 1);
                draft_bias(U, Arec, W, V, r, x0[b], x + (size_t)b * G, ks, hs, hs + r, delta);
                const float *Lrow = L + o * (size_t)V;
                for (int v = 0; v < V; ++v) yd[v] = (double)Lrow[v] + delta[v];
                double md, Zd = softmax_row(yd, V, T, ed, &md);
                double Q = 0.0;
                for (int v = 0; v < V; ++v) {
                    double d = et[v] / Zt - ed[v] / Zd;
                    q[v] = d > 0.0 ? d : 0.0;
                    Q += q[v];
                }
                if (Q > 0.0) {
                    yv = inverse_cdf(q, V, Q, u_final[b], &mfin);
                    kind = 0;
                } else {
                    yv = inverse_cdf(et, V, Zt, u_final[b], &mfin);
                    kind = 3;
                }
            } else {
                yv = inverse_cdf(et, V, Zt, u_final[b], &mfin);
                kind = 1;
            }
        }
        int *tok = tokens_out + (size_t)b * (G + 1);
        for (int j = 0; j < G + 1; ++j) tok[j] = -1;
        for (int j = 0; j < A; ++j) tok[j] = x[(size_t)b * G + j];
        tok[A] = yv;
        acc_out[b] = A;
        nout_out[b] = A + 1;
        margin_fin_out[b] = mfin;
        final_kind_out[b] = kind;
    }
    free(delta); free(yd); free(yt); free(ed); free(et); free(q); free(hs);
    return rc;
}

/* Verification of Markov-head drafts (the headline path). */
int dspark_oracle_verify(int B, int G, int V, int r, const float *Tlog, const float *L,
                         const float *U, const float *W, const int *x0, const int *x,
                         const float *temp, const double *u_accept,
                         const double *u_final, const int *ell,
                         const int *force_accept, int *acc_out, int *tokens_out,
                         int *nout_out, double *pt_x_out, double *pd_x_out,
                         double *margin_acc_out, double *margin_fin_out,
                         int *final_kind_out)
{
    return dspark_oracle_verify_head(B, G, V, r, Tlog, L, U, NULL, W, x0, x, temp, u_accept, u_final, ell,
                                     force_accept, acc_out, tokens_out, nout_out, pt_x_out, pd_x_out,
                                     margin_acc_out, margin_fin_out, final_kind_out);
}
