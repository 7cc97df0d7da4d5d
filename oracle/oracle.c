/*
 * oracle.c -- plain fp64 CPU oracle for the MatMamba block at a Matryoshka
 * width m_i.  TEST INFRASTRUCTURE ONLY: nothing in the product path links,
 * loads or calls this file.  It is used by tests/, by the smoke check and by
 * the CPU-baseline leg of bench.py.
 *
 * Sources (page title, part of the page):
 *  - "MatMamba: A Matryoshka State Space Model", block-definition paragraph:
 *    the Mamba2 block is an input projection W_in = (W_z, W_x, W_B, W_C, W_dt),
 *    a causal 1-D convolution of kernel 4 whose weights are conv_x ^ conv_B ^
 *    conv_C applied per channel, a chunk + selective scan with learnable A and
 *    D, the nonlinearity sigma = SiLU, Norm = RMSNorm, and an output
 *    projection W_out; input and output are (b, l, d).
 *  - same page, nested sub-block paragraph: at width m_i, d_i = e*m_i,
 *    h_i = d_i/d_head, d_i mod d_head = 0; (d_inner, .) parameters are cut to
 *    their first d_i rows and (n_heads) parameters to their first h_i entries.
 *  - same page, stacking paragraph: a model f_i is L blocks M_i stacked.
 *  - "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *    (summary page), Architecture and Sampling Rule: the SSM branch is gated
 *    multiplicatively by the parallel branch, and the hidden state is updated
 *    with input-dependent discretised parameters (the step dt).
 *
 * The pages drop the block's equations.  The readings taken here (the plainest
 * ones the rest of the text supports) are:
 *   z, x, B, C, r = view rows of W_in applied to u_t
 *   v = x ^ B ^ C;  c_t = SiLU(conv_b + sum_j conv_w[j] * v_{t-3+j})  (causal,
 *                   zero history unless a conv state is given)
 *   dt_t = softplus(r_t + dt_bias)
 *   H_t = exp(dt_t*A) * H_{t-1} + dt_t * B_t x_t^T   (per head, N x P)
 *   y_t = C_t^T H_t + D * x_t
 *   q = y (.) SiLU(z);  n = q / sqrt(mean(q^2) + eps) (.) norm_w
 *   out_t = W_out[:, 0:d] n_t
 * The scan is evaluated in its sequential (recurrent) form: the chunked form
 * used by the GPU kernels is an exact refactorisation of it.
 *
 * Every function here is parity-pinned by tests/test_oracle_pins.py against
 * closed forms, brute-force matrix forms, library routines and invariants.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int d_model;
    int d_inner;
    int d_head;
    int d_state;
    int ngroups;
    int d_conv;
    double norm_eps;
} orc_dims;

static double silu(double a) { return a / (1.0 + exp(-a)); }

/* softplus(v) = log(1 + e^v), written in the two algebraically equal forms so
 * that neither branch overflows. */
static double softplus(double v) { return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v)); }

/* Width rule of the nested sub-block paragraph: d_i = d_inner*m/d_model must
 * be an integer multiple of d_head, 0 < m <= d_model.  Returns 0 and fills
 * d_i, h_i, or -1 for an invalid width. */
int orc_width(const orc_dims* g, int m, int* d_out, int* h_out)
{
    if (m <= 0 || m > g->d_model) return -1;
    long num = (long)g->d_inner * (long)m;
    if (num % g->d_model) return -1;
    int d = (int)(num / g->d_model);
    if (d % g->d_head) return -1;
    *d_out = d;
    *h_out = d / g->d_head;
    return 0;
}

/* Sequential selective-scan recurrence for contiguous tensors.
 *   x (batch, L, h, P), dt (batch, L, h), A (h), B, C (batch, L, G, N),
 *   D (h) or NULL, init_state (batch, h, P, N) or NULL,
 *   y (batch, L, h, P), final_state (batch, h, P, N) or NULL.
 * Head i reads group i / heads_per_group.  The state element [b,i,p,n] is
 * H_i[n, p] of the recurrence. */
int orc_ssd_scan(int batch, int L, int h, int P, int N, int G, int heads_per_group,
                 const double* x, const double* dt, const double* A,
                 const double* Bm, const double* Cm, const double* D,
                 const double* init_state, double* y, double* final_state)
{
    if (batch < 0 || L < 0 || h <= 0 || P <= 0 || N <= 0 || G <= 0 || heads_per_group <= 0) return -1;
    if ((h - 1) / heads_per_group >= G) return -1;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < batch; ++b) {
        for (int i = 0; i < h; ++i) {
            double* H = (double*)malloc(sizeof(double) * (size_t)P * N);
            for (int e = 0; e < P * N; ++e)
                H[e] = init_state ? init_state[(((size_t)b * h + i) * P) * N + e] : 0.0;
            int g = i / heads_per_group;
            for (int t = 0; t < L; ++t) {
                size_t tok = (size_t)b * L + t;
                double dti = dt[tok * h + i];
                double a = exp(dti * A[i]);
                const double* Bt = Bm + (tok * G + g) * N;
                const double* Ct = Cm + (tok * G + g) * N;
                for (int p = 0; p < P; ++p) {
                    double xp = x[(tok * h + i) * P + p];
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double v = a * H[p * N + n] + dti * Bt[n] * xp;
                        H[p * N + n] = v;
                        acc += Ct[n] * v;
                    }
                    y[(tok * h + i) * P + p] = acc + (D ? D[i] * xp : 0.0);
                }
            }
            if (final_state)
                for (int e = 0; e < P * N; ++e)
                    final_state[(((size_t)b * h + i) * P) * N + e] = H[e];
            free(H);
        }
    }
    return 0;
}

/* Row-wise RMSNorm over the last dimension: out = v / sqrt(mean(v^2)+eps) * w.
 * Used for the pre-norm of the stacked model. */
int orc_rmsnorm_rows(int rows, int cols, const double* v, const double* w, double eps, double* out)
{
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const double* vr = v + (size_t)r * cols;
        double ss = 0.0;
        for (int c = 0; c < cols; ++c) ss += vr[c] * vr[c];
        double inv = 1.0 / sqrt(ss / cols + eps);
        for (int c = 0; c < cols; ++c) out[(size_t)r * cols + c] = vr[c] * inv * w[c];
    }
    return 0;
}

/*
 * Block forward at width m (the sub-block M_i of the nested sub-block
 * paragraph), fp64, for every batch row.
 *
 * Full-width parameters (E = d_inner, GN = ngroups*d_state, H = E/d_head):
 *   W_in (2E + 2GN + H, d_model) rows z | x | B | C | dt,
 *   conv_w (E + 2GN, d_conv) rows x | B | C, conv_b (E + 2GN),
 *   dt_bias, A, D (H), norm_w (E), W_out (d_model, E).
 * u (batch, L, d_model); out (batch, L, d_model).
 * Optional state: ssm (batch, H, P, N) and conv (batch, E + 2GN, d_conv - 1),
 * oldest tap first.  Only heads [0, h_i) and conv rows [0, d_i) u [E, E+2GN)
 * are read or written; other entries of the *_out buffers are not touched.
 * Optional trace buffers (NULL to skip), per token: z (d_i), xbc after
 * conv + SiLU (d_i + 2GN), dt (h_i), y scan output including D*x (d_i),
 * nrm gated + normalised activations (d_i).
 */
int orc_block_fwd(const orc_dims* g,
                  const double* W_in, const double* conv_w, const double* conv_b,
                  const double* dt_bias, const double* A, const double* D,
                  const double* norm_w, const double* W_out,
                  int batch, int L, int m, const double* u,
                  const double* ssm_state_in, const double* conv_state_in,
                  double* out, double* ssm_state_out, double* conv_state_out,
                  double* tr_z, double* tr_xbc, double* tr_dt, double* tr_y, double* tr_nrm)
{
    int d, h;
    if (orc_width(g, m, &d, &h)) return -1;
    const int Dm = g->d_model, E = g->d_inner, P = g->d_head, N = g->d_state, G = g->ngroups;
    const int K = g->d_conv, GN = G * N, H = E / P;
    const int nconv = d + 2 * GN;           /* active conv channels: x | B | C */
    const int hpg = H / G;                  /* heads per group over the full width */
    if (E % P || H % G || K < 1) return -1;

    for (int b = 0; b < batch; ++b) {
        const double* ub = u + (size_t)b * L * Dm;
        double* zb = (double*)malloc(sizeof(double) * (size_t)L * d);
        double* vb = (double*)malloc(sizeof(double) * (size_t)L * nconv);   /* pre-conv x|B|C */
        double* rb = (double*)malloc(sizeof(double) * (size_t)L * h);       /* raw dt */
        double* cb = (double*)malloc(sizeof(double) * (size_t)L * nconv);   /* post conv+SiLU */
        double* db = (double*)malloc(sizeof(double) * (size_t)L * h);       /* dt */
        double* yb = (double*)malloc(sizeof(double) * (size_t)L * d);
        double* nb = (double*)malloc(sizeof(double) * (size_t)L * d);

        /* 1. input projection through the width view of W_in */
#pragma omp parallel for schedule(static)
        for (int t = 0; t < L; ++t) {
            const double* ut = ub + (size_t)t * Dm;
            for (int c = 0; c < d; ++c) {                    /* z rows [0, d) */
                const double* w = W_in + (size_t)c * Dm;
                double s = 0.0;
                for (int k = 0; k < Dm; ++k) s += w[k] * ut[k];
                zb[(size_t)t * d + c] = s;
            }
            for (int c = 0; c < nconv; ++c) {                /* x rows [E, E+d), B|C rows [2E, 2E+2GN) */
                int row = c < d ? E + c : 2 * E + (c - d);
                const double* w = W_in + (size_t)row * Dm;
                double s = 0.0;
                for (int k = 0; k < Dm; ++k) s += w[k] * ut[k];
                vb[(size_t)t * nconv + c] = s;
            }
            for (int i = 0; i < h; ++i) {                    /* dt rows [2E+2GN, 2E+2GN+h) */
                const double* w = W_in + (size_t)(2 * E + 2 * GN + i) * Dm;
                double s = 0.0;
                for (int k = 0; k < Dm; ++k) s += w[k] * ut[k];
                rb[(size_t)t * h + i] = s;
            }
        }

        /* 2. causal depthwise convolution + SiLU on x ^ B ^ C */
#pragma omp parallel for schedule(static)
        for (int c = 0; c < nconv; ++c) {
            int row = c < d ? c : E + (c - d);               /* conv row of this channel */
            for (int t = 0; t < L; ++t) {
                double s = conv_b[row];
                for (int j = 0; j < K; ++j) {
                    int tau = t - (K - 1) + j;
                    double v;
                    if (tau >= 0) v = vb[(size_t)tau * nconv + c];
                    else if (conv_state_in) v = conv_state_in[((size_t)b * (E + 2 * GN) + row) * (K - 1) + (K - 1 + tau)];
                    else v = 0.0;
                    s += conv_w[(size_t)row * K + j] * v;
                }
                cb[(size_t)t * nconv + c] = silu(s);
            }
            if (conv_state_out && K > 1) {
                for (int k = 0; k < K - 1; ++k) {
                    int tau = L - (K - 1) + k;
                    double v;
                    if (tau >= 0) v = vb[(size_t)tau * nconv + c];
                    else if (conv_state_in) v = conv_state_in[((size_t)b * (E + 2 * GN) + row) * (K - 1) + (K - 1 + tau)];
                    else v = 0.0;
                    conv_state_out[((size_t)b * (E + 2 * GN) + row) * (K - 1) + k] = v;
                }
            }
        }

        /* 3. dt = softplus(raw + dt_bias) */
        for (int t = 0; t < L; ++t)
            for (int i = 0; i < h; ++i)
                db[(size_t)t * h + i] = softplus(rb[(size_t)t * h + i] + dt_bias[i]);

        /* 4. selective scan over heads [0, h) with the D skip term */
#pragma omp parallel for schedule(dynamic)
        for (int i = 0; i < h; ++i) {
            int grp = i / hpg;
            double* Hs = (double*)malloc(sizeof(double) * (size_t)P * N);
            for (int e = 0; e < P * N; ++e)
                Hs[e] = ssm_state_in ? ssm_state_in[(((size_t)b * H + i) * P) * N + e] : 0.0;
            for (int t = 0; t < L; ++t) {
                const double* ct = cb + (size_t)t * nconv;
                const double* Bt = ct + d + grp * N;
                const double* Ct = ct + d + GN + grp * N;
                double dti = db[(size_t)t * h + i];
                double a = exp(dti * A[i]);
                for (int p = 0; p < P; ++p) {
                    double xp = ct[i * P + p];
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        double v = a * Hs[p * N + n] + dti * Bt[n] * xp;
                        Hs[p * N + n] = v;
                        acc += Ct[n] * v;
                    }
                    yb[(size_t)t * d + i * P + p] = acc + D[i] * xp;
                }
            }
            if (ssm_state_out)
                for (int e = 0; e < P * N; ++e)
                    ssm_state_out[(((size_t)b * H + i) * P) * N + e] = Hs[e];
            free(Hs);
        }

        /* 5. gate by SiLU(z), then RMSNorm over the d active channels */
#pragma omp parallel for schedule(static)
        for (int t = 0; t < L; ++t) {
            double ss = 0.0;
            for (int c = 0; c < d; ++c) {
                double q = yb[(size_t)t * d + c] * silu(zb[(size_t)t * d + c]);
                nb[(size_t)t * d + c] = q;
                ss += q * q;
            }
            double inv = 1.0 / sqrt(ss / d + g->norm_eps);
            for (int c = 0; c < d; ++c) nb[(size_t)t * d + c] *= inv * norm_w[c];
        }

        /* 6. output projection through the K-prefix W_out[:, 0:d] */
#pragma omp parallel for schedule(static)
        for (int t = 0; t < L; ++t) {
            const double* nt = nb + (size_t)t * d;
            double* ot = out + ((size_t)b * L + t) * Dm;
            for (int j = 0; j < Dm; ++j) {
                const double* w = W_out + (size_t)j * E;
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += w[c] * nt[c];
                ot[j] = s;
            }
        }

        if (tr_z) memcpy(tr_z + (size_t)b * L * d, zb, sizeof(double) * (size_t)L * d);
        if (tr_xbc) memcpy(tr_xbc + (size_t)b * L * nconv, cb, sizeof(double) * (size_t)L * nconv);
        if (tr_dt) memcpy(tr_dt + (size_t)b * L * h, db, sizeof(double) * (size_t)L * h);
        if (tr_y) memcpy(tr_y + (size_t)b * L * d, yb, sizeof(double) * (size_t)L * d);
        if (tr_nrm) memcpy(tr_nrm + (size_t)b * L * d, nb, sizeof(double) * (size_t)L * d);
        free(zb); free(vb); free(rb); free(cb); free(db); free(yb); free(nb);
    }
    return 0;
}

/* Number of OpenMP threads the oracle runs with (reported beside CPU timings). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
