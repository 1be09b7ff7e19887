/*
 * CPU oracle for the decay-masked linear-attention (SSD) forward operator.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * reference that the CUDA path is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * Everything is computed in double precision from the float32 input values
 * (inputs that the GPU sees as bf16 are passed here already rounded, so both
 * sides read the same numbers).
 *
 * Sources (2Mamba2Furious, Mongaras & Larson, 2026; the thelatestinai.com
 * summary page):
 *   - Algorithm 2 "Mamba-2 Setup" and Algorithm 3 "Mamba-2 Forward Pass":
 *       A = -exp(A_log), dt = softplus(dt_P + dt_bias), A^CS = cumsum(A*dt),
 *       D_res = V * D  (D is one value per channel, H*d_h of them).
 *   - Algorithm 4 (Mamba-2S): A^M_ij = exp(A^CS_i - A^CS_j), M_ij = [i >= j].
 *   - Algorithm 1 / Algorithm 5 (2Mamba): y = ((phi(Q)phi(K)^T)^p (.) A^M (.) M) V,
 *       N = row sums of the same masked matrix, y_n = y / N.
 *   - Algorithm 6 (2Mamba inference): H_up_t = a_t H_up_{t-1} + phi(k_t)^T v_t,
 *       H_dn_t = a_t H_dn_{t-1} + phi(k_t), phi(x) = x (x) x for order 2.
 *
 *   - Algorithm 4 (Mamba-2S): A = -softplus(h W_A) given per token (the
 *       "log_decay" input here), A^CS = cumsum(A), and the value
 *       discretisation V_dt = V (.) dt with dt = softplus(h W_dt) (the
 *       "value_dt" switch, with dt = softplus(dt_P + dt_bias)).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - the cumulative sum is inclusive and starts at zero for every (b, h);
 *   - the contraction uses raw V unless value_dt is set (then V_dt);
 *   - the normaliser sums the masked score matrix only (it does not see dt);
 *   - the D residual is added after normalisation, to raw V;
 *   - the normaliser divides by the exact row sum, with no epsilon;
 *   - the Algorithm 6 output line is cut off on the page; the plain reading
 *     y_t = phi(q_t)^T H_up_t (divided by phi(q_t) . H_dn_t when normalising)
 *     is used.
 *
 * Layouts: q, k, v, out are [B, H, N, d] row-major; dt_p and log_decay are
 * [B, H, N]; A_log and dt_bias are [H]; D is [H*d] or NULL.  Pointers that an
 * option does not use may be NULL: A_log when log_decay is given; dt_p and
 * dt_bias when log_decay is given and value_dt is off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(x) = log(1 + e^x), written in the overflow-free form
 * max(x, 0) + log1p(exp(-|x|)).  Algorithm 3, dt line. */
double oracle_softplus(double x)
{
    double ax = fabs(x);
    return (x > 0.0 ? x : 0.0) + log1p(exp(-ax));
}

/* Per-token log-decay a_t and its inclusive cumulative sum
 * A^CS_t = sum_{tau <= t} a_tau for one (b, h) row of length N.
 * Algorithm 3: A = -exp(A_log), dt = softplus(dt_P + dt_bias),
 * a_t = A * dt_t.  Algorithm 4: a_t is given directly (ld_row != NULL). */
static void log_decay_row(const float *dt_p_row, double A_log_h, double dt_bias_h,
                          const float *ld_row, int N, double *acs_row)
{
    double run = 0.0;
    for (int t = 0; t < N; ++t) {
        if (ld_row) {
            run += (double)ld_row[t];
        } else {
            double dt = oracle_softplus((double)dt_p_row[t] + dt_bias_h);
            run += -exp(A_log_h) * dt;
        }
        acs_row[t] = run;
    }
}

/* A^CS for every (b, h): out is [B, H, N].  log_decay ([B, H, N], may be
 * NULL) replaces A * dt when given; A_log, dt_p and dt_bias are then unused. */
void oracle_log_decay(const float *dt_p, const float *A_log, const float *dt_bias,
                      const float *log_decay, int B, int H, int N, double *acs)
{
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t off = ((size_t)b * H + h) * (size_t)N;
            log_decay_row(log_decay ? NULL : dt_p + off, log_decay ? 0.0 : A_log[h],
                          log_decay ? 0.0 : dt_bias[h], log_decay ? log_decay + off : NULL, N,
                          acs + off);
        }
}

/* Value factor of token t: dt_t = softplus(dt_P + dt_bias) when value_dt
 * (Algorithm 4, V_dt = V (.) dt), else 1. */
static double value_factor(const float *dt_p, const float *dt_bias, int value_dt, size_t tok, int h)
{
    return value_dt ? oracle_softplus((double)dt_p[tok] + (double)dt_bias[h]) : 1.0;
}

/* Mask entry A^M_ij * M_ij (Algorithm 4): exp(A^CS_i - A^CS_j) when i >= j,
 * zero otherwise. */
double oracle_mask(const double *acs_row, int i, int j)
{
    if (i < j) return 0.0;
    return exp(acs_row[i] - acs_row[j]);
}

/* Feature map phi: identity for order 1, the tensor square x (x) x for
 * order 2 (Algorithm 6, (q_t)^{(x)2} = q_t (x) q_t), entry (a, b) stored at
 * a*d + b.  Returns the feature length d^order. */
int oracle_feature(const double *x, int d, int order, double *out)
{
    if (order == 1) {
        for (int a = 0; a < d; ++a) out[a] = x[a];
        return d;
    }
    for (int a = 0; a < d; ++a)
        for (int b = 0; b < d; ++b) out[a * d + b] = x[a] * x[b];
    return d * d;
}

/* Quadratic (masked-matrix) form, Algorithm 1 / Algorithm 5, evaluated for a
 * chosen set of rows.  For every (b, h) and every listed row i:
 *     s_ij = q_i . k_j,   w_ij = s_ij^order * A^M_ij * M_ij,
 *     y_i  = sum_j w_ij f_j v_j,   N_i = sum_j w_ij,
 * with f_j = dt_j under value_dt and 1 otherwise,
 *     y_i /= N_i when normalise != 0,   y_ic += D[h*d + c] * v_ic when D.
 * With an initial state (h0 [B, H, D_phi, d], z0 [B, H, D_phi], either may be
 * NULL for zero) the state carried into token 0 decays by exp(A^CS_i) up to
 * token i (Algorithm 6 unrolled): y_i += exp(A^CS_i) phi(q_i)^T h0 and
 * N_i += exp(A^CS_i) phi(q_i) . z0.
 * rows: n_rows row indices (each in [0, N)), or NULL for all N rows.
 * out: [B, H, n_rows, d] (n_rows = N when rows is NULL).
 * norm_out (may be NULL): [B, H, n_rows], the row sums N_i.
 * Returns 0, or -1 on a bad argument. */
int oracle_ssd_quadratic(const float *q, const float *k, const float *v,
                         const float *dt_p, const float *A_log, const float *dt_bias,
                         const float *D, const float *log_decay, int value_dt,
                         const double *h0, const double *z0,
                         int B, int H, int N, int d, int order, int normalise,
                         const int *rows, int n_rows,
                         double *out, double *norm_out)
{
    if (order != 1 && order != 2) return -1;
    if (B < 0 || H < 0 || N < 0 || d <= 0 || d > 64) return -1;
    if (rows == NULL) n_rows = N;
    for (int r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;

    int BH = B * H;
    double *acs = (double *)malloc(sizeof(double) * (size_t)BH * (size_t)(N > 0 ? N : 1));
    if (!acs) return -1;
    oracle_log_decay(dt_p, A_log, dt_bias, log_decay, B, H, N, acs);

    long long total = (long long)BH * n_rows;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long task = 0; task < total; ++task) {
        int bh = (int)(task / n_rows);
        int r = (int)(task % n_rows);
        int h = bh % H;
        int i = rows ? rows[r] : r;
        size_t base = (size_t)bh * N;
        const double *acs_row = acs + base;
        const float *qi = q + (base + i) * d;
        double *yi = out + ((size_t)bh * n_rows + r) * d;
        for (int c = 0; c < d; ++c) yi[c] = 0.0;
        double ni = 0.0;
        for (int j = 0; j <= i; ++j) {
            const float *kj = k + (base + j) * d;
            const float *vj = v + (base + j) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += (double)qi[c] * (double)kj[c];
            double score = (order == 1) ? s : s * s;
            double w = score * oracle_mask(acs_row, i, j);
            double wv = w * value_factor(dt_p, dt_bias, value_dt, base + j, h);
            for (int c = 0; c < d; ++c) yi[c] += wv * (double)vj[c];
            ni += w;
        }
        if (h0 || z0) {
            int Dphi = (order == 1) ? d : d * d;
            double e = exp(acs_row[i]);
            double xq[64], fq[64 * 64];
            for (int c = 0; c < d; ++c) xq[c] = qi[c];
            oracle_feature(xq, d, order, fq);
            for (int m = 0; m < Dphi; ++m) {
                if (h0) {
                    const double *row = h0 + ((size_t)bh * Dphi + m) * d;
                    for (int c = 0; c < d; ++c) yi[c] += e * fq[m] * row[c];
                }
                if (z0) ni += e * fq[m] * z0[(size_t)bh * Dphi + m];
            }
        }
        if (normalise)
            for (int c = 0; c < d; ++c) yi[c] /= ni;
        if (D) {
            const float *vi = v + (base + i) * d;
            for (int c = 0; c < d; ++c) yi[c] += (double)D[h * d + c] * (double)vi[c];
        }
        if (norm_out) norm_out[(size_t)bh * n_rows + r] = ni;
    }
    free(acs);
    return 0;
}

/* Token-by-token recurrent form, Algorithm 6, with the multiplicative decay
 * a_t = exp(A_h * dt_t) of Algorithm 3 (or exp(log_decay_t), Algorithm 4):
 *     H_up_t = a_t H_up_{t-1} + phi(k_t) (f_t v_t)^T     (D_phi x d),
 *     f_t = dt_t under value_dt, else 1
 *     H_dn_t = a_t H_dn_{t-1} + phi(k_t)           (D_phi)
 *     y_t = phi(q_t)^T H_up_t,  N_t = phi(q_t) . H_dn_t,
 * then y_t /= N_t when normalising and y_tc += D[h*d+c] v_tc when D.
 * The states start at h0 [B, H, D_phi, d] and z0 [B, H, D_phi] (zero when
 * NULL).  out is [B, H, N, d]; norm_out may be NULL.
 * state_out (may be NULL) receives the final H_up as [B, H, D_phi, d] and
 * zstate_out (may be NULL) the final H_dn as [B, H, D_phi].
 * Returns 0, or -1 on a bad argument / allocation failure. */
int oracle_ssd_recurrent(const float *q, const float *k, const float *v,
                         const float *dt_p, const float *A_log, const float *dt_bias,
                         const float *D, const float *log_decay, int value_dt,
                         const double *h0, const double *z0,
                         int B, int H, int N, int d, int order, int normalise,
                         double *out, double *norm_out,
                         double *state_out, double *zstate_out)
{
    if (order != 1 && order != 2) return -1;
    if (B < 0 || H < 0 || N < 0 || d <= 0) return -1;
    int Dphi = (order == 1) ? d : d * d;
    int BH = B * H;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        int h = bh % H;
        double *Hup = (double *)calloc((size_t)Dphi * d, sizeof(double));
        double *Hdn = (double *)calloc((size_t)Dphi, sizeof(double));
        double *fq = (double *)malloc(sizeof(double) * Dphi);
        double *fk = (double *)malloc(sizeof(double) * Dphi);
        double *xq = (double *)malloc(sizeof(double) * d);
        double *xk = (double *)malloc(sizeof(double) * d);
        if (!Hup || !Hdn || !fq || !fk || !xq || !xk) {
#pragma omp atomic write
            failed = 1;
            free(Hup); free(Hdn); free(fq); free(fk); free(xq); free(xk);
            continue;
        }
        if (h0) memcpy(Hup, h0 + (size_t)bh * Dphi * d, sizeof(double) * (size_t)Dphi * d);
        if (z0) memcpy(Hdn, z0 + (size_t)bh * Dphi, sizeof(double) * (size_t)Dphi);
        size_t base = (size_t)bh * N;
        for (int t = 0; t < N; ++t) {
            double a;
            if (log_decay) {
                a = exp((double)log_decay[base + t]);
            } else {
                double dt = oracle_softplus((double)dt_p[base + t] + (double)dt_bias[h]);
                a = exp(-exp((double)A_log[h]) * dt);
            }
            double f = value_factor(dt_p, dt_bias, value_dt, base + t, h);
            const float *qt = q + (base + t) * d;
            const float *kt = k + (base + t) * d;
            const float *vt = v + (base + t) * d;
            for (int c = 0; c < d; ++c) { xq[c] = qt[c]; xk[c] = kt[c]; }
            oracle_feature(xq, d, order, fq);
            oracle_feature(xk, d, order, fk);
            for (int m = 0; m < Dphi; ++m) {
                double *row = Hup + (size_t)m * d;
                for (int c = 0; c < d; ++c) row[c] = a * row[c] + fk[m] * f * (double)vt[c];
                Hdn[m] = a * Hdn[m] + fk[m];
            }
            double *yt = out + (base + t) * d;
            for (int c = 0; c < d; ++c) yt[c] = 0.0;
            double nt = 0.0;
            for (int m = 0; m < Dphi; ++m) {
                const double *row = Hup + (size_t)m * d;
                for (int c = 0; c < d; ++c) yt[c] += fq[m] * row[c];
                nt += fq[m] * Hdn[m];
            }
            if (normalise)
                for (int c = 0; c < d; ++c) yt[c] /= nt;
            if (D)
                for (int c = 0; c < d; ++c) yt[c] += (double)D[h * d + c] * (double)vt[c];
            if (norm_out) norm_out[base + t] = nt;
        }
        if (state_out) memcpy(state_out + (size_t)bh * Dphi * d, Hup, sizeof(double) * (size_t)Dphi * d);
        if (zstate_out) memcpy(zstate_out + (size_t)bh * Dphi, Hdn, sizeof(double) * (size_t)Dphi);
        free(Hup); free(Hdn); free(fq); free(fk); free(xq); free(xk);
    }
    return failed ? -1 : 0;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* SiLU(x) = x / (1 + e^-x)  (Algorithm 3, the sigma after the convolution). */
double oracle_silu(double x)
{
    return x / (1.0 + exp(-x));
}

/* Causal depthwise 1-D convolution over the token axis, optionally followed by
 * SiLU: the prologue Q, K, V = sigma(conv_1d(h W_QKV)) of Algorithm 3, and the
 * window-2 convolution q^c_t = conv_1d(q_t, q_{t-1}) of the Algorithm 6 page.
 * For every (b, h), token t and channel c (channel index h*d + c of the
 * weights):
 *     u = bias[h*d + c] + sum_{j < width} w[(h*d + c)*width + j] * x[t - j, c]
 * with x[t < 0] = 0 (each (b, h) sequence starts from zero), out = SiLU(u) when
 * silu != 0, else u.  x, out: [B, H, N, d]; w: [H*d, width]; bias: [H*d] or
 * NULL.  Returns 0, or -1 on a bad argument. */
int oracle_conv1d(const float *x, const float *w, const float *bias, int B, int H, int N, int d,
                  int width, int silu, double *out)
{
    if (B < 0 || H < 0 || N < 0 || d <= 0 || width < 1) return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            size_t base = ((size_t)b * H + h) * (size_t)N;
            for (int t = 0; t < N; ++t)
                for (int c = 0; c < d; ++c) {
                    int ch = h * d + c;
                    double u = bias ? (double)bias[ch] : 0.0;
                    for (int j = 0; j < width && j <= t; ++j)
                        u += (double)w[(size_t)ch * width + j] * (double)x[(base + t - j) * d + c];
                    out[(base + t) * d + c] = silu ? oracle_silu(u) : u;
                }
        }
    return 0;
}
