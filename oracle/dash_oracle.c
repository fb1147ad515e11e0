/*
 * dash_oracle.c -- plain float64 CPU oracle for the DashAttention forward pass and its
 * backward pass (gradients of Q, K, V and the Stage 0 query qbar; orc_backward at the end).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file;
 * only the tests, the smoke check and the benchmark's CPU-baseline / reference legs use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Source of every formula: "DashAttention: Differentiable and Adaptive Sparse Hierarchical
 * Attention" (xllm-io paper review page), section 3 "core formulas":
 *   - alpha-entmax:   background formula  alpha-entmax(s) = [(alpha-1) s - tau 1]_+^{1/(alpha-1)}
 *   - Stage 0:        Eq. 4   (local SDPA of a learned per-KV-head query over each chunk)
 *   - Stage 1:        Eq. 6   (chunk logits, entmax routing, GQA average, union support)
 *   - Stage 2:        Eq. 9, Eq. 11-12 (prior-induced softmax, prior strength sigma, split lambda)
 *                     and Proposition 4.1 (equivalent additive bias d_{i,j}).
 * Stage 0 and Stage 2 wording is also confirmed by the gist.science technical summary,
 * "Methodology", Stage 0 / Stage 2.
 *
 * Readings where the pages are silent (the plainest reading each passage supports):
 *   chunks are contiguous from position 0, c(j) = floor(j/B); a query at position i routes only
 *   over complete chunks c < floor(i/B); its own chunk is the diagonal branch D_i = {c(i)B .. i}
 *   and carries bias 0; rows with floor(i/B) = 0 have no routed branch; 1/sqrt(d) scales the
 *   logits of all three stages, gamma only Stage 1; head h belongs to KV head floor(h/g_q);
 *   the bias uses the GQA-averaged weights w^(r), shared by all heads of the group.
 *
 * All arithmetic is double.  Inputs are float arrays (bf16 and fp32 values are exact in float),
 * read through element strides [batch, position, head]; the head dimension is contiguous.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int batch, seqlen, h_q, h_kv, d, chunk;
    double alpha, gamma, inv_sigma;
} orc_cfg;

/* ------------------------------------------------------------------------------------------ */
/* alpha-entmax (background formula).  x = (alpha-1)*s is passed in.                          */
/* ------------------------------------------------------------------------------------------ */

static double ent_mass(const double* x, int n, double t, double p)
{
    double f = 0.0;
    for (int c = 0; c < n; ++c) {
        double u = x[c] - t;
        if (u > 0.0) f += pow(u, p);
    }
    return f;
}

/* Threshold tau with sum_c [x_c - tau]_+^{1/(alpha-1)} = 1.
 * Step 1: bisection on [max x - 1, max x - n^{-(alpha-1)}]; the mass is >= 1 at the left end
 *         (the largest entry alone contributes 1) and <= 1 at the right end (each of the n
 *         entries contributes at most 1/n), and it is strictly decreasing in between.
 * Step 2: on the support found, solve exactly: alpha = 2 is linear, alpha = 1.5 is the smaller
 *         root of a quadratic, any other alpha takes Newton steps to double precision. */
double orc_entmax_threshold(const double* x, int n, double alpha)
{
    const double p = 1.0 / (alpha - 1.0);
    double mx = x[0];
    for (int c = 1; c < n; ++c) if (x[c] > mx) mx = x[c];
    double lo = mx - 1.0;
    double hi = mx - pow((double)n, -(alpha - 1.0));
    for (int it = 0; it < 200; ++it) {
        double t = 0.5 * (lo + hi);
        if (t <= lo || t >= hi) break;
        if (ent_mass(x, n, t, p) >= 1.0) lo = t; else hi = t;
    }
    /* support at the bisection threshold */
    int k = 0;
    double s1 = 0.0, s2 = 0.0;
    for (int c = 0; c < n; ++c)
        if (x[c] > lo) { ++k; s1 += x[c] - mx; s2 += (x[c] - mx) * (x[c] - mx); }
    double tau = lo;
    if (alpha == 2.0) {
        tau = mx + (s1 - 1.0) / k;
    } else if (alpha == 1.5) {
        /* k t^2 - 2 t s1 + s2 - 1 = 0 in t = tau - mx; smaller root */
        double disc = s1 * s1 - k * (s2 - 1.0);
        if (disc < 0.0) disc = 0.0;
        tau = mx + (s1 - sqrt(disc)) / k;
    } else {
        for (int it = 0; it < 100; ++it) {
            double f = -1.0, fp = 0.0;
            for (int c = 0; c < n; ++c) {
                double u = x[c] - tau;
                if (u > 0.0) { f += pow(u, p); fp -= p * pow(u, p - 1.0); }
            }
            if (fp == 0.0) break;
            double step = f / fp;
            tau -= step;
            if (fabs(step) < 1e-15) break;
        }
    }
    return tau;
}

/* p = alpha-entmax(s); returns the support size. */
int orc_entmax(const double* s, int n, double alpha, double* p)
{
    if (n <= 0) return 0;
    double* x = (double*)malloc(sizeof(double) * (size_t)n);
    for (int c = 0; c < n; ++c) x[c] = (alpha - 1.0) * s[c];
    double tau = orc_entmax_threshold(x, n, alpha);
    int k = 0;
    for (int c = 0; c < n; ++c) {
        double u = x[c] - tau;
        p[c] = u > 0.0 ? pow(u, 1.0 / (alpha - 1.0)) : 0.0;
        k += p[c] > 0.0;
    }
    free(x);
    return k;
}

/* ------------------------------------------------------------------------------------------ */
/* Stage 0 (Eq. 4): kbar = sum_{t in [t0,t1)} softmax_t(<qbar_r, k_t>/sqrt(d)) k_t             */
/* ------------------------------------------------------------------------------------------ */

static const float* at(const float* base, const long long st[3], int b, int j, int h)
{
    return base + (long long)b * st[0] + (long long)j * st[1] + (long long)h * st[2];
}

/* Summary of keys t0..t1-1 of sequence b, KV head r.  A complete chunk is t1 - t0 = B; the
 * running summary of an incomplete chunk (incremental decoding) is the same formula over the
 * keys written so far. */
void orc_chunk_summary(const orc_cfg* cf, const float* K, const long long ks[3], const float* qbar,
                       int b, int r, int t0, int t1, double* out)
{
    const int d = cf->d;
    const double scale = 1.0 / sqrt((double)d);
    double* a = (double*)malloc(sizeof(double) * (size_t)(t1 - t0));
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        const float* k = at(K, ks, b, t, r);
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += (double)qbar[r * d + e] * (double)k[e];
        a[t - t0] = dot * scale;
        if (a[t - t0] > m) m = a[t - t0];
    }
    double z = 0.0;
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    for (int t = t0; t < t1; ++t) {
        double wgt = exp(a[t - t0] - m);
        z += wgt;
        const float* k = at(K, ks, b, t, r);
        for (int e = 0; e < d; ++e) out[e] += wgt * (double)k[e];
    }
    for (int e = 0; e < d; ++e) out[e] /= z;
    free(a);
}

/* All complete-chunk summaries: kbar[b][r][c][d] for c < floor(n/B). */
void orc_stage0(const orc_cfg* cf, const float* K, const long long ks[3], const float* qbar,
                double* kbar, int nthreads)
{
    const int T = cf->seqlen / cf->chunk, d = cf->d;
    const long long total = (long long)cf->batch * cf->h_kv * T;
#ifdef _OPENMP
    #pragma omp parallel for schedule(dynamic, 4) num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
#endif
    for (long long u = 0; u < total; ++u) {
        int c = (int)(u % T);
        int r = (int)((u / T) % cf->h_kv);
        int b = (int)(u / ((long long)T * cf->h_kv));
        orc_chunk_summary(cf, K, ks, qbar, b, r, c * cf->chunk, (c + 1) * cf->chunk,
                          kbar + (((long long)b * cf->h_kv + r) * T + c) * d);
    }
    (void)nthreads;
}

/* ------------------------------------------------------------------------------------------ */
/* Stage 1 (Eq. 6) for one query position i, one KV head r:                                   */
/*   zbar_c^(h) = <q_i^(h), kbar_c^(r)>/sqrt(d), c < floor(i/B)                                */
/*   what^(h)  = alpha-entmax(gamma * zbar^(h))                                                */
/*   w^(r)     = sum_{h in G_r} what^(h) / g_q,   R = {c : w_c > 0} (union of head supports)  */
/* Proposition 4.1: mu = mean_{c in R} log w_c, bias_c = (log w_c - mu) / sigma.               */
/* q points at the g_q query vectors of the group, d apart.  kbar points at [c][d] for head r. */
/* Outputs per visible chunk: w, bias (0 off the support), margin = max_h (x_c^(h) - tau^(h)). */
/* Returns |R|.                                                                                */
/* ------------------------------------------------------------------------------------------ */

int orc_route_row(const orc_cfg* cf, const float* q, long long q_head_stride, const double* kbar,
                  int nvis, double* w, double* bias, double* margin)
{
    const int d = cf->d, g = cf->h_q / cf->h_kv;
    const double scale = 1.0 / sqrt((double)d), am1 = cf->alpha - 1.0;
    if (nvis <= 0) return 0;
    double* x = (double*)malloc(sizeof(double) * (size_t)nvis);
    for (int c = 0; c < nvis; ++c) { w[c] = 0.0; margin[c] = -INFINITY; bias[c] = 0.0; }
    for (int hh = 0; hh < g; ++hh) {
        const float* qh = q + (long long)hh * q_head_stride;
        for (int c = 0; c < nvis; ++c) {
            double dot = 0.0;
            for (int e = 0; e < d; ++e) dot += (double)qh[e] * kbar[(long long)c * d + e];
            x[c] = am1 * (cf->gamma * dot * scale);
        }
        double tau = orc_entmax_threshold(x, nvis, cf->alpha);
        for (int c = 0; c < nvis; ++c) {
            double u = x[c] - tau;
            if (u > margin[c]) margin[c] = u;
            if (u > 0.0) w[c] += pow(u, 1.0 / am1);
        }
    }
    int nR = 0;
    double mu = 0.0;
    for (int c = 0; c < nvis; ++c) {
        w[c] /= g;
        if (w[c] > 0.0) { ++nR; mu += log(w[c]); }
    }
    mu /= nR;
    for (int c = 0; c < nvis; ++c)
        bias[c] = w[c] > 0.0 ? (log(w[c]) - mu) * cf->inv_sigma : 0.0;
    free(x);
    return nR;
}

/* ------------------------------------------------------------------------------------------ */
/* Stage 2 for one query vector q at position i (sequence b, KV head r).                      */
/* Proposition 4.1 form: z_j = <q,k_j>/sqrt(d) + d_ij with d_ij = bias_{c(j)} on the routed    */
/* tokens R_i and 0 on the diagonal tokens D_i = {c(i)B .. i};  o = softmax(z) V over R u D.    */
/* ------------------------------------------------------------------------------------------ */

static void attend_bias_form(const orc_cfg* cf, const float* q, const float* K, const long long ks[3],
                             const float* V, const long long vs[3], int b, int r, int i,
                             int nvis, const double* w, const double* bias, double* o)
{
    const int d = cf->d, B = cf->chunk, ci = i / B;
    const double scale = 1.0 / sqrt((double)d);
    int ntok = 0;
    for (int c = 0; c < nvis; ++c) if (w[c] > 0.0) ntok += B;
    ntok += i - ci * B + 1;
    double* z = (double*)malloc(sizeof(double) * (size_t)ntok);
    int* idx = (int*)malloc(sizeof(int) * (size_t)ntok);
    int m = 0;
    for (int c = 0; c < nvis; ++c) {
        if (!(w[c] > 0.0)) continue;
        for (int j = c * B; j < (c + 1) * B; ++j) { idx[m] = j; z[m++] = bias[c]; }
    }
    for (int j = ci * B; j <= i; ++j) { idx[m] = j; z[m++] = 0.0; }
    double zmax = -INFINITY;
    for (int t = 0; t < m; ++t) {
        const float* k = at(K, ks, b, idx[t], r);
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)k[e];
        z[t] += dot * scale;
        if (z[t] > zmax) zmax = z[t];
    }
    double den = 0.0;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int t = 0; t < m; ++t) {
        double p = exp(z[t] - zmax);
        den += p;
        const float* v = at(V, vs, b, idx[t], r);
        for (int e = 0; e < d; ++e) o[e] += p * (double)v[e];
    }
    for (int e = 0; e < d; ++e) o[e] /= den;
    free(z); free(idx);
}

/* Eq. 9 with the prior of Eq. 11-12, written out independently of the bias form:
 *   w'_j = (1/B) w_{c(j)}^{1/sigma} / sum_{c in R} w_c^{1/sigma}           (j in R)
 *   lambda = sigmoid( KL(u_R || w'_R) + log(|R|/|D|) ),  u_R uniform over the tokens of R
 *   g_j = lambda w'_j on R, (1 - lambda)/|D| on D;   p_j = g_j exp(z_j) / sum_t g_t exp(z_t).
 * With no routed chunk lambda = 0 and the row is a plain softmax over D. */
static void attend_prior_form(const orc_cfg* cf, const float* q, const float* K, const long long ks[3],
                              const float* V, const long long vs[3], int b, int r, int i,
                              int nvis, const double* w, double* o)
{
    const int d = cf->d, B = cf->chunk, ci = i / B;
    const double scale = 1.0 / sqrt((double)d), is = cf->inv_sigma;
    int nRc = 0;
    double zsum = 0.0;
    for (int c = 0; c < nvis; ++c) if (w[c] > 0.0) { ++nRc; zsum += pow(w[c], is); }
    const int nR = nRc * B, nD = i - ci * B + 1;
    double lam = 0.0;
    if (nR > 0) {
        double kl = 0.0;
        for (int c = 0; c < nvis; ++c) {
            if (!(w[c] > 0.0)) continue;
            double wp = pow(w[c], is) / (B * zsum);
            kl += B * (1.0 / nR) * log((1.0 / nR) / wp);
        }
        double a = kl + log((double)nR / nD);
        lam = 1.0 / (1.0 + exp(-a));
    }
    /* log g_j + z_j, then a max-subtracted normalisation */
    const int ntok = nR + nD;
    double* lz = (double*)malloc(sizeof(double) * (size_t)ntok);
    int* idx = (int*)malloc(sizeof(int) * (size_t)ntok);
    int m = 0;
    for (int c = 0; c < nvis; ++c) {
        if (!(w[c] > 0.0)) continue;
        double lg = log(lam) + log(pow(w[c], is) / (B * zsum));
        for (int j = c * B; j < (c + 1) * B; ++j) { idx[m] = j; lz[m++] = lg; }
    }
    for (int j = ci * B; j <= i; ++j) { idx[m] = j; lz[m++] = log((1.0 - lam) / nD); }
    double mx = -INFINITY;
    for (int t = 0; t < m; ++t) {
        const float* k = at(K, ks, b, idx[t], r);
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)k[e];
        lz[t] += dot * scale;
        if (lz[t] > mx) mx = lz[t];
    }
    double den = 0.0;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int t = 0; t < m; ++t) {
        double p = exp(lz[t] - mx);
        den += p;
        const float* v = at(V, vs, b, idx[t], r);
        for (int e = 0; e < d; ++e) o[e] += p * (double)v[e];
    }
    for (int e = 0; e < d; ++e) o[e] /= den;
    free(lz); free(idx);
}

/* ------------------------------------------------------------------------------------------ */
/* Rows driver: the full forward for a list of query rows.                                     */
/*   Qrows [batch][nrows][h_q][d] (contiguous) holds the query vectors; pos[b*nrows + t] is the */
/*   position of row t of sequence b (prefill: its index in the sequence; decode: length - 1). */
/*   kbar [batch][h_kv][kbar_T][d] holds the complete-chunk summaries of Stage 0.               */
/* Outputs: O [batch][nrows][h_q][d]; optional counts [batch][h_kv][nrows] = |R|, and optional  */
/* w, bias, margin [batch][h_kv][nrows][kbar_T] (entries past floor(pos/B) are left at 0).     */
/* prior_form = 1 computes Stage 2 from Eq. 9 / 11-12 instead of Proposition 4.1.              */
/* O = NULL skips Stage 2 (routing statistics only).                                          */
/* ------------------------------------------------------------------------------------------ */

void orc_rows(const orc_cfg* cf, const float* Qrows, const int* pos, int nrows,
              const float* K, const long long ks[3], const float* V, const long long vs[3],
              const double* kbar, int kbar_T, int prior_form, double* O,
              int* counts, double* wout, double* bout, double* mout, int nthreads)
{
    const int d = cf->d, g = cf->h_q / cf->h_kv, hkv = cf->h_kv, B = cf->chunk;
    const long long total = (long long)cf->batch * nrows * hkv;
#ifdef _OPENMP
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
#endif
    for (long long u = 0; u < total; ++u) {
        const int r = (int)(u % hkv);
        const int t = (int)((u / hkv) % nrows);
        const int b = (int)(u / ((long long)hkv * nrows));
        const int i = pos[(long long)b * nrows + t];
        int nvis = i / B;
        if (nvis > kbar_T) nvis = kbar_T;
        const int cap = kbar_T > 0 ? kbar_T : 1;
        double* w = (double*)calloc((size_t)cap, sizeof(double));
        double* bias = (double*)calloc((size_t)cap, sizeof(double));
        double* margin = (double*)calloc((size_t)cap, sizeof(double));
        const float* q = Qrows + (((long long)b * nrows + t) * cf->h_q + (long long)r * g) * d;
        const double* kb = kbar + ((long long)b * hkv + r) * (long long)kbar_T * d;
        int nR = orc_route_row(cf, q, d, kb, nvis, w, bias, margin);
        for (int hh = 0; hh < g && O; ++hh) {
            double* o = O + (((long long)b * nrows + t) * cf->h_q + (long long)r * g + hh) * d;
            if (prior_form)
                attend_prior_form(cf, q + (long long)hh * d, K, ks, V, vs, b, r, i, nvis, w, o);
            else
                attend_bias_form(cf, q + (long long)hh * d, K, ks, V, vs, b, r, i, nvis, w, bias, o);
        }
        const long long rowoff = ((long long)b * hkv + r) * nrows + t;
        if (counts) counts[rowoff] = nR;
        for (int c = 0; c < nvis; ++c) {
            if (wout) wout[rowoff * kbar_T + c] = w[c];
            if (bout) bout[rowoff * kbar_T + c] = bias[c];
            if (mout) mout[rowoff * kbar_T + c] = margin[c];
        }
        free(w); free(bias); free(margin);
    }
    (void)nthreads;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------------ */
/* Backward pass.  The paper review page (section 3, after Eq. 9) states that the output is    */
/* differentiable in q, k, v and in the prior g, so that the gradient reaches the Stage 1      */
/* entmax scores and through them the Stage 0 summaries (the Stage 2 kernel row: the training  */
/* backward reuses the routed support, the entmax Jacobian being sparse).  The routed support  */
/* R itself is piecewise constant, so no gradient flows through the choice of R.               */
/*                                                                                             */
/* Chain, for the scalar L = sum dO . O, per (b, r) and position i (g heads h of group r):     */
/*   Stage 2 (Prop. 4.1): p = softmax(z + d) over R u D;  dv_j += p_j dO;  dp_j = dO . v_j;     */
/*     ds_j = p_j (dp_j - sum_t p_t dp_t);  dq += ds_j k_j / sqrt(d);  dk_j += ds_j q / sqrt(d); */
/*     dbias_c = sum over the group's heads and the tokens j of chunk c of ds_j.               */
/*   bias_c = (log w_c - mean_{R} log w) / sigma  =>  dlog w_c = (dbias_c - mean_R dbias)/sigma, */
/*     dw_c = dlog w_c / w_c;  w = mean_h what^(h)  =>  dwhat^(h)_c = dw_c / g.                 */
/*   alpha-entmax(theta), theta = gamma zbar: on the support the Jacobian is                   */
/*     diag(s) - s s^T / sum s with s_c = what_c^(2 - alpha)  (zero off the support), so        */
/*     dtheta = s * dwhat - s (s . dwhat) / sum s;  dzbar = gamma dtheta.                       */
/*   Eq. 6: dq += dzbar_c kbar_c / sqrt(d);  dkbar_c += dzbar_c q / sqrt(d).                    */
/*   Eq. 4: kbar_c = sum_t pi_t k_t, pi = softmax_t(<qbar, k_t>/sqrt(d)):                       */
/*     dk_t += pi_t dkbar_c + pi_t (k_t . dkbar_c - kbar_c . dkbar_c) qbar / sqrt(d);           */
/*     dqbar += sum_t pi_t (k_t . dkbar_c - kbar_c . dkbar_c) k_t / sqrt(d).                    */
/*                                                                                             */
/* Layouts (contiguous): Q, dO, dQ [batch][n][h_q][d]; K, V, dK, dV [batch][n][h_kv][d];        */
/* qbar, dqbar [h_kv][d] (dqbar sums over the batch).                                          */
/* ------------------------------------------------------------------------------------------ */

static void bwd_pair(const orc_cfg* cf, const float* Q, const float* K, const float* V, const float* qbar,
                     const float* dO, double* dQ, double* dK, double* dV, double* dqbar_part, int b, int r)
{
    const int n = cf->seqlen, d = cf->d, B = cf->chunk, hq = cf->h_q, hkv = cf->h_kv, g = hq / hkv;
    const int T = n / B;
    const double scale = 1.0 / sqrt((double)d), am1 = cf->alpha - 1.0;
    const long long ks[3] = {(long long)n * hkv * d, (long long)hkv * d, d};
    const int Tc = T > 0 ? T : 1;
    double* kbar = (double*)calloc((size_t)Tc * d, sizeof(double));
    double* dkbar = (double*)calloc((size_t)Tc * d, sizeof(double));
    double* what = (double*)calloc((size_t)g * Tc, sizeof(double));
    double* w = (double*)calloc((size_t)Tc, sizeof(double));
    double* bias = (double*)calloc((size_t)Tc, sizeof(double));
    double* dbias = (double*)calloc((size_t)Tc, sizeof(double));
    double* x = (double*)calloc((size_t)Tc, sizeof(double));
    double* zl = (double*)malloc(sizeof(double) * (size_t)(n + B));
    double* pl = (double*)malloc(sizeof(double) * (size_t)(n + B));
    int* idx = (int*)malloc(sizeof(int) * (size_t)(n + B));
    for (int c = 0; c < T; ++c)
        orc_chunk_summary(cf, K, ks, qbar, b, r, c * B, (c + 1) * B, kbar + (long long)c * d);

#define KV_AT(base, j) ((base) + (((long long)b * n + (j)) * hkv + r) * d)
#define Q_AT(base, i, hh) ((base) + (((long long)b * n + (i)) * hq + (long long)r * g + (hh)) * d)

    for (int i = 0; i < n; ++i) {
        const int ci = i / B;
        const int nvis = ci < T ? ci : T;
        /* Stage 1 forward: per-head weights, their average, the routed set and the biases */
        int nR = 0;
        double mu = 0.0;
        for (int c = 0; c < nvis; ++c) { w[c] = 0.0; dbias[c] = 0.0; }
        for (int hh = 0; hh < g && nvis > 0; ++hh) {
            const float* q = Q_AT(Q, i, hh);
            for (int c = 0; c < nvis; ++c) {
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += (double)q[e] * kbar[(long long)c * d + e];
                x[c] = am1 * cf->gamma * dot * scale;
            }
            const double tau = orc_entmax_threshold(x, nvis, cf->alpha);
            for (int c = 0; c < nvis; ++c) {
                const double u = x[c] - tau;
                what[(long long)hh * Tc + c] = u > 0.0 ? pow(u, 1.0 / am1) : 0.0;
                w[c] += what[(long long)hh * Tc + c] / g;
            }
        }
        for (int c = 0; c < nvis; ++c)
            if (w[c] > 0.0) { ++nR; mu += log(w[c]); }
        if (nR) mu /= nR;
        for (int c = 0; c < nvis; ++c) bias[c] = w[c] > 0.0 ? (log(w[c]) - mu) * cf->inv_sigma : 0.0;

        /* Stage 2 forward and backward, one head at a time */
        int m = 0;
        for (int c = 0; c < nvis; ++c)
            if (w[c] > 0.0)
                for (int j = c * B; j < (c + 1) * B; ++j) idx[m++] = j;
        const int mR = m;
        for (int j = ci * B; j <= i; ++j) idx[m++] = j;
        for (int hh = 0; hh < g; ++hh) {
            const float* q = Q_AT(Q, i, hh);
            const float* go = Q_AT(dO, i, hh);
            double* gq = Q_AT(dQ, i, hh);
            double zmax = -INFINITY;
            for (int t = 0; t < m; ++t) {
                const float* k = KV_AT(K, idx[t]);
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)k[e];
                zl[t] = dot * scale + (t < mR ? bias[idx[t] / B] : 0.0);
                if (zl[t] > zmax) zmax = zl[t];
            }
            double den = 0.0;
            for (int t = 0; t < m; ++t) { pl[t] = exp(zl[t] - zmax); den += pl[t]; }
            double delta = 0.0;
            for (int t = 0; t < m; ++t) {
                pl[t] /= den;
                const float* v = KV_AT(V, idx[t]);
                double dp = 0.0;
                for (int e = 0; e < d; ++e) dp += (double)go[e] * (double)v[e];
                zl[t] = dp;                                   /* zl now holds dp_t */
                delta += pl[t] * dp;
            }
            for (int t = 0; t < m; ++t) {
                const int j = idx[t];
                const double ds = pl[t] * (zl[t] - delta);
                const float* k = KV_AT(K, j);
                double* gk = KV_AT(dK, j);
                double* gv = KV_AT(dV, j);
                for (int e = 0; e < d; ++e) {
                    gv[e] += pl[t] * (double)go[e];
                    gk[e] += ds * (double)q[e] * scale;
                    gq[e] += ds * (double)k[e] * scale;
                }
                if (t < mR) dbias[j / B] += ds;
            }
        }

        /* Stage 1 backward through the bias, the GQA mean and each head's entmax */
        if (nR > 0) {
            double mdb = 0.0;
            for (int c = 0; c < nvis; ++c) if (w[c] > 0.0) mdb += dbias[c];
            mdb /= nR;
            for (int hh = 0; hh < g; ++hh) {
                const double* wh = what + (long long)hh * Tc;
                double s1 = 0.0, s2 = 0.0;
                for (int c = 0; c < nvis; ++c) {
                    if (!(wh[c] > 0.0)) continue;
                    const double s = pow(wh[c], 2.0 - cf->alpha);
                    const double dwh = cf->inv_sigma * (dbias[c] - mdb) / w[c] / g;
                    s1 += s;
                    s2 += s * dwh;
                }
                const float* q = Q_AT(Q, i, hh);
                double* gq = Q_AT(dQ, i, hh);
                for (int c = 0; c < nvis; ++c) {
                    if (!(wh[c] > 0.0)) continue;
                    const double s = pow(wh[c], 2.0 - cf->alpha);
                    const double dwh = cf->inv_sigma * (dbias[c] - mdb) / w[c] / g;
                    const double dz = cf->gamma * (s * dwh - s * s2 / s1);
                    for (int e = 0; e < d; ++e) {
                        gq[e] += dz * kbar[(long long)c * d + e] * scale;
                        dkbar[(long long)c * d + e] += dz * (double)q[e] * scale;
                    }
                }
            }
        }
    }

    /* Stage 0 backward (Eq. 4) */
    for (int c = 0; c < T; ++c) {
        const double* kb = kbar + (long long)c * d;
        const double* gkb = dkbar + (long long)c * d;
        double amax = -INFINITY, den = 0.0, kbg = 0.0;
        for (int e = 0; e < d; ++e) kbg += kb[e] * gkb[e];
        for (int t = 0; t < B; ++t) {
            const float* k = KV_AT(K, c * B + t);
            double dot = 0.0;
            for (int e = 0; e < d; ++e) dot += (double)qbar[r * d + e] * (double)k[e];
            zl[t] = dot * scale;
            if (zl[t] > amax) amax = zl[t];
        }
        for (int t = 0; t < B; ++t) { pl[t] = exp(zl[t] - amax); den += pl[t]; }
        for (int t = 0; t < B; ++t) {
            const float* k = KV_AT(K, c * B + t);
            double* gk = KV_AT(dK, c * B + t);
            const double pi = pl[t] / den;
            double kg = 0.0;
            for (int e = 0; e < d; ++e) kg += (double)k[e] * gkb[e];
            const double da = pi * (kg - kbg);
            for (int e = 0; e < d; ++e) {
                gk[e] += pi * gkb[e] + da * (double)qbar[r * d + e] * scale;
                dqbar_part[e] += da * (double)k[e] * scale;
            }
        }
    }
#undef KV_AT
#undef Q_AT
    free(kbar); free(dkbar); free(what); free(w); free(bias); free(dbias); free(x);
    free(zl); free(pl); free(idx);
}

void orc_backward(const orc_cfg* cf, const float* Q, const float* K, const float* V, const float* qbar,
                  const float* dO, double* dQ, double* dK, double* dV, double* dqbar, int nthreads)
{
    const int d = cf->d, hkv = cf->h_kv;
    const long long pairs = (long long)cf->batch * hkv;
    double* part = (double*)calloc((size_t)pairs * d, sizeof(double));
#ifdef _OPENMP
    #pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
#endif
    for (long long u = 0; u < pairs; ++u)
        bwd_pair(cf, Q, K, V, qbar, dO, dQ, dK, dV, part + u * d, (int)(u / hkv), (int)(u % hkv));
    for (int r = 0; r < hkv; ++r)
        for (int e = 0; e < d; ++e) dqbar[(long long)r * d + e] = 0.0;
    for (long long u = 0; u < pairs; ++u)
        for (int e = 0; e < d; ++e) dqbar[(u % hkv) * d + e] += part[u * d + e];
    free(part);
    (void)nthreads;
}
