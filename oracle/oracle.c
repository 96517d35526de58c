/*
 * CPU oracle for the ParaRNN Newton solve of diagonal GRU / LSTM recurrences.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library: the two agree only because both follow the same mathematics.
 *
 * Plain, slow, obviously correct: fp64 state, libm exp/tanh, one loop per
 * formula, OpenMP only over independent channels.  No blocking, fusion or
 * reordering beyond what the definitions state.
 *
 * Source page cited throughout (cafecomtech.com, 2026-04-23):
 *   "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
 *    pra 7B parâmetros"
 * Sections used:
 *   "O compromisso que SSMs fizeram"  - the nonlinear recurrence
 *        h_l = sigma_l(h_{l-1}, x_l) applied one step at a time, and the
 *        linear SSM h_l = A_l h_{l-1} + B_l x_l.
 *   "A sacada: método de Newton"      - the whole sequence is one system of
 *        equations with every hidden state unknown; Newton linearises it with
 *        the Jacobians, which take the place of A_l, so each iteration is a
 *        linear SSM.
 *   "Engenharia pra escalar"          - diagonal matrices in the cell, hence a
 *        diagonal Jacobian (ParaGRU) or a 2x2 block-diagonal one per channel
 *        over (c, h) (ParaLSTM).
 * The pages do not print the cell equations.  The cells below are the
 * diagonal GRU and LSTM of the ParaGRU / ParaLSTM workloads:
 *   GRU : z = s(u_z + a_z h), r = s(u_r + a_r h), c = tanh(u_c + a_c r h),
 *         h' = (1 - z) h + z c
 *   LSTM: i,f,o = s(u + a h), g = tanh(u_g + a_g h), c' = f c + i g,
 *         h' = o tanh(c')                           (gate order i, f, o, g)
 *
 * Layouts (row-major, D fastest): u [B][L][G][D], a [G][D], h0/c0 [B][D],
 * states [B][L][D] holding h_1..h_L (h_0 is an input, not an unknown).
 *
 * Parity pins: every function here is checked in the CPU test suite against
 * torch.nn.GRU / torch.nn.LSTM in float64, torch autograd, dense linear
 * solves of the full Newton system, and central finite differences.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_NOT_CONVERGED 1
#define ORACLE_NONFINITE (-5)
#define ORACLE_NOMEM (-2)

static double logistic(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------------ cells */

/* One diagonal-GRU step for one channel, and its derivative with respect to
 * the previous state (the diagonal Jacobian entry of "Engenharia pra
 * escalar").  Derivative by the product and chain rules:
 *   d/dh[(1-z)h + z c] = (1-z) + z'(c - h) + z c'
 *   z' = z(1-z) a_z,  r' = r(1-r) a_r,  c' = (1 - c^2) a_c (r + h r').      */
void oracle_gru_cell(double h, const double u[3], const double a[3],
                     double *f_out, double *A_out)
{
    double z = logistic(u[0] + a[0] * h);
    double r = logistic(u[1] + a[1] * h);
    double c = tanh(u[2] + a[2] * r * h);
    *f_out = (1.0 - z) * h + z * c;
    if (A_out) {
        double dz = z * (1.0 - z) * a[0];
        double dr = r * (1.0 - r) * a[1];
        double dc = (1.0 - c * c) * a[2] * (r + h * dr);
        *A_out = (1.0 - z) + dz * (c - h) + z * dc;
    }
}

/* One diagonal-LSTM step for one channel and its 2x2 Jacobian over (c, h)
 * ("Engenharia pra escalar": block-diagonal 2x2 per channel).
 * J is row-major: J[0] = dc'/dc, J[1] = dc'/dh, J[2] = dh'/dc, J[3] = dh'/dh. */
void oracle_lstm_cell(double c, double h, const double u[4], const double a[4],
                      double *c_out, double *h_out, double J[4])
{
    double i = logistic(u[0] + a[0] * h);
    double f = logistic(u[1] + a[1] * h);
    double o = logistic(u[2] + a[2] * h);
    double g = tanh(u[3] + a[3] * h);
    double cn = f * c + i * g;
    double t = tanh(cn);
    *c_out = cn;
    *h_out = o * t;
    if (J) {
        double di = i * (1.0 - i) * a[0];
        double df = f * (1.0 - f) * a[1];
        double dO = o * (1.0 - o) * a[2];
        double dg = (1.0 - g * g) * a[3];
        double dcn_dh = df * c + di * g + i * dg;
        J[0] = f;
        J[1] = dcn_dh;
        J[2] = o * (1.0 - t * t) * f;
        J[3] = dO * t + o * (1.0 - t * t) * dcn_dh;
    }
}

static void gather_u(const double *u, int64_t L, int64_t G, int64_t D,
                     int64_t b, int64_t l, int64_t d, double *out)
{
    for (int64_t g = 0; g < G; ++g)
        out[g] = u[((b * L + l) * G + g) * D + d];
}

static void gather_a(const double *a, int64_t G, int64_t D, int64_t d, double *out)
{
    for (int64_t g = 0; g < G; ++g)
        out[g] = a[g * D + d];
}

/* --------------------------------------------------- sequential application */

/* "O compromisso que SSMs fizeram": h_l = sigma(h_{l-1}, x_l), one step at a
 * time.  This is the exact solution of the Newton system (unique: its
 * Jacobian is unit lower bidiagonal), so it is the reference for states. */
void oracle_gru_seq(int64_t B, int64_t L, int64_t D, const double *u,
                    const double *a, const double *h0, double *h)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t d = 0; d < D; ++d) {
            double ad[3], ul[3], f;
            gather_a(a, 3, D, d, ad);
            double hp = h0 ? h0[b * D + d] : 0.0;
            for (int64_t l = 0; l < L; ++l) {
                gather_u(u, L, 3, D, b, l, d, ul);
                oracle_gru_cell(hp, ul, ad, &f, NULL);
                h[(b * L + l) * D + d] = f;
                hp = f;
            }
        }
}

void oracle_lstm_seq(int64_t B, int64_t L, int64_t D, const double *u,
                     const double *a, const double *c0, const double *h0,
                     double *c, double *h)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t d = 0; d < D; ++d) {
            double ad[4], ul[4], cn, hn;
            gather_a(a, 4, D, d, ad);
            double cp = c0 ? c0[b * D + d] : 0.0;
            double hp = h0 ? h0[b * D + d] : 0.0;
            for (int64_t l = 0; l < L; ++l) {
                gather_u(u, L, 4, D, b, l, d, ul);
                oracle_lstm_cell(cp, hp, ul, ad, &cn, &hn, NULL);
                c[(b * L + l) * D + d] = cn;
                h[(b * L + l) * D + d] = hn;
                cp = cn;
                hp = hn;
            }
        }
}

/* ------------------------------------------------------------ Newton solve */

/* Max-abs residual accumulator that keeps non-finite values visible:
 * NaN if any residual is NaN, else +inf if any is infinite. */
typedef struct { double m; int nan; int inf; } resmax_t;

static void resmax_add(resmax_t *r, double v)
{
    if (isnan(v)) r->nan = 1;
    else if (isinf(v)) r->inf = 1;
    else if (fabs(v) > r->m) r->m = fabs(v);
}

static double resmax_value(const resmax_t *r)
{
    if (r->nan) return NAN;
    if (r->inf) return INFINITY;
    return r->m;
}

/* "A sacada: método de Newton": all states H = (h_1..h_L) are unknowns of
 * F_l(H) = h_l - f(h_{l-1}, u_l) = 0.  Newton step k:
 *   r_k = max |F(H^k)|; stop if r_k <= tol or k == max_iters;
 *   A_l = df/dh_{l-1} at H^k (the Jacobians play the role of A_l);
 *   delta_0 = 0, delta_l = A_l delta_{l-1} - F_l   (the linear SSM, solved
 *   here by a plain serial loop; the parallel scan is the GPU's business);
 *   H^{k+1} = H^k + delta.
 * Initial guess H^0 = 0 (the pages give none).  Returns the status; iters is
 * the number of updates applied to the returned H, residual = r of that H.
 * res_hist (optional, max_iters+1 entries) receives r_0..r_iters.          */
int oracle_gru_newton(int64_t B, int64_t L, int64_t D, const double *u,
                      const double *a, const double *h0, double tol,
                      int max_iters, double *H, int *iters_out,
                      double *residual_out, double *res_hist)
{
    size_t n = (size_t)(B * L * D);
    double *F = (double *)malloc(n * sizeof(double));
    double *A = (double *)malloc(n * sizeof(double));
    if (!F || !A) { free(F); free(A); return ORACLE_NOMEM; }
    memset(H, 0, n * sizeof(double));
    int k = 0;
    double r;
    int status;
    for (;;) {
        resmax_t rm = {0.0, 0, 0};
        for (int64_t b = 0; b < B; ++b)
            for (int64_t l = 0; l < L; ++l)
                for (int64_t d = 0; d < D; ++d) {
                    double ad[3], ul[3], f, Al;
                    gather_a(a, 3, D, d, ad);
                    gather_u(u, L, 3, D, b, l, d, ul);
                    double hp = (l == 0) ? (h0 ? h0[b * D + d] : 0.0)
                                         : H[(b * L + l - 1) * D + d];
                    oracle_gru_cell(hp, ul, ad, &f, &Al);
                    size_t idx = (size_t)((b * L + l) * D + d);
                    F[idx] = H[idx] - f;
                    A[idx] = Al;
                    resmax_add(&rm, F[idx]);
                }
        r = resmax_value(&rm);
        if (res_hist) res_hist[k] = r;
        if (!isfinite(r)) { status = ORACLE_NONFINITE; break; }
        if (r <= tol) { status = ORACLE_OK; break; }
        if (k == max_iters) { status = ORACLE_NOT_CONVERGED; break; }
        for (int64_t b = 0; b < B; ++b)
            for (int64_t d = 0; d < D; ++d) {
                double delta = 0.0;
                for (int64_t l = 0; l < L; ++l) {
                    size_t idx = (size_t)((b * L + l) * D + d);
                    delta = A[idx] * delta - F[idx];
                    H[idx] += delta;
                }
            }
        ++k;
    }
    *iters_out = k;
    *residual_out = r;
    free(F);
    free(A);
    return status;
}

/* Same algorithm for the 2x2 block system of the LSTM over (c, h):
 * F_l = (c_l, h_l) - f(c_{l-1}, h_{l-1}, u_l); delta_l = J_l delta_{l-1} - F_l.
 * The residual is the max over both components. */
int oracle_lstm_newton(int64_t B, int64_t L, int64_t D, const double *u,
                       const double *a, const double *c0, const double *h0,
                       double tol, int max_iters, double *C, double *H,
                       int *iters_out, double *residual_out, double *res_hist)
{
    size_t n = (size_t)(B * L * D);
    double *Fc = (double *)malloc(n * sizeof(double));
    double *Fh = (double *)malloc(n * sizeof(double));
    double *J = (double *)malloc(4 * n * sizeof(double));
    if (!Fc || !Fh || !J) { free(Fc); free(Fh); free(J); return ORACLE_NOMEM; }
    memset(C, 0, n * sizeof(double));
    memset(H, 0, n * sizeof(double));
    int k = 0;
    double r;
    int status;
    for (;;) {
        resmax_t rm = {0.0, 0, 0};
        for (int64_t b = 0; b < B; ++b)
            for (int64_t l = 0; l < L; ++l)
                for (int64_t d = 0; d < D; ++d) {
                    double ad[4], ul[4], cn, hn;
                    gather_a(a, 4, D, d, ad);
                    gather_u(u, L, 4, D, b, l, d, ul);
                    double cp, hp;
                    if (l == 0) {
                        cp = c0 ? c0[b * D + d] : 0.0;
                        hp = h0 ? h0[b * D + d] : 0.0;
                    } else {
                        cp = C[(b * L + l - 1) * D + d];
                        hp = H[(b * L + l - 1) * D + d];
                    }
                    size_t idx = (size_t)((b * L + l) * D + d);
                    oracle_lstm_cell(cp, hp, ul, ad, &cn, &hn, &J[4 * idx]);
                    Fc[idx] = C[idx] - cn;
                    Fh[idx] = H[idx] - hn;
                    resmax_add(&rm, Fc[idx]);
                    resmax_add(&rm, Fh[idx]);
                }
        r = resmax_value(&rm);
        if (res_hist) res_hist[k] = r;
        if (!isfinite(r)) { status = ORACLE_NONFINITE; break; }
        if (r <= tol) { status = ORACLE_OK; break; }
        if (k == max_iters) { status = ORACLE_NOT_CONVERGED; break; }
        for (int64_t b = 0; b < B; ++b)
            for (int64_t d = 0; d < D; ++d) {
                double dc = 0.0, dh = 0.0;
                for (int64_t l = 0; l < L; ++l) {
                    size_t idx = (size_t)((b * L + l) * D + d);
                    const double *Jl = &J[4 * idx];
                    double ndc = Jl[0] * dc + Jl[1] * dh - Fc[idx];
                    double ndh = Jl[2] * dc + Jl[3] * dh - Fh[idx];
                    dc = ndc;
                    dh = ndh;
                    C[idx] += dc;
                    H[idx] += dh;
                }
            }
        ++k;
    }
    *iters_out = k;
    *residual_out = r;
    free(Fc);
    free(Fh);
    free(J);
    return status;
}

/* ------------------------------------------------------------------- BPTT */

/* Gradients of Loss = sum_{b,l,d} gh[b,l,d] * h[b,l,d] by plain
 * backpropagation through time of the sequential recurrence.  The pages do
 * not describe training gradients; this is the textbook chain rule applied
 * to the GRU step, written without the Jacobian A_l so that it is an
 * independent check of any adjoint-scan formulation.
 * du [B][L][3][D] (gradients w.r.t. the gate pre-activations), da [3][D]
 * (summed over b and l), dh0 [B][D] (may be NULL).                          */
void oracle_gru_bptt(int64_t B, int64_t L, int64_t D, const double *u,
                     const double *a, const double *h0, const double *gh,
                     double *du, double *da, double *dh0)
{
#pragma omp parallel for schedule(static)
    for (int64_t d = 0; d < D; ++d) {
        double ad[3], ul[3], f;
        double sz = 0.0, sr = 0.0, sc = 0.0;
        double *hs = (double *)malloc((size_t)(L + 1) * sizeof(double));
        gather_a(a, 3, D, d, ad);
        for (int64_t b = 0; b < B; ++b) {
            hs[0] = h0 ? h0[b * D + d] : 0.0;
            for (int64_t l = 0; l < L; ++l) {
                gather_u(u, L, 3, D, b, l, d, ul);
                oracle_gru_cell(hs[l], ul, ad, &f, NULL);
                hs[l + 1] = f;
            }
            double lam = 0.0; /* dLoss/dh_l accumulated from later steps */
            for (int64_t l = L - 1; l >= 0; --l) {
                lam += gh[(b * L + l) * D + d];
                gather_u(u, L, 3, D, b, l, d, ul);
                double h = hs[l];
                double z = logistic(ul[0] + ad[0] * h);
                double r = logistic(ul[1] + ad[1] * h);
                double c = tanh(ul[2] + ad[2] * r * h);
                double g_z = lam * (c - h) * z * (1.0 - z);
                double g_c = lam * z * (1.0 - c * c);
                double g_r = g_c * ad[2] * h * r * (1.0 - r);
                double *dul = &du[((b * L + l) * 3) * D + d];
                dul[0 * D] = g_z;
                dul[1 * D] = g_r;
                dul[2 * D] = g_c;
                sz += g_z * h;
                sr += g_r * h;
                sc += g_c * r * h;
                lam = lam * (1.0 - z) + g_z * ad[0] + g_r * ad[1] + g_c * ad[2] * r;
            }
            if (dh0) dh0[b * D + d] = lam;
        }
        da[0 * D + d] = sz;
        da[1 * D + d] = sr;
        da[2 * D + d] = sc;
        free(hs);
    }
}

/* Gradients of Loss = sum gh*h + sum gc*c (gc may be NULL = 0) for the
 * diagonal LSTM, by plain backpropagation through time.  du [B][L][4][D],
 * da [4][D], dc0/dh0 [B][D] (either may be NULL).                           */
void oracle_lstm_bptt(int64_t B, int64_t L, int64_t D, const double *u,
                      const double *a, const double *c0, const double *h0,
                      const double *gh, const double *gc, double *du,
                      double *da, double *dc0, double *dh0)
{
#pragma omp parallel for schedule(static)
    for (int64_t d = 0; d < D; ++d) {
        double ad[4], ul[4], cn, hn;
        double si = 0.0, sf = 0.0, so = 0.0, sg = 0.0;
        double *cs = (double *)malloc((size_t)(L + 1) * sizeof(double));
        double *hs = (double *)malloc((size_t)(L + 1) * sizeof(double));
        gather_a(a, 4, D, d, ad);
        for (int64_t b = 0; b < B; ++b) {
            cs[0] = c0 ? c0[b * D + d] : 0.0;
            hs[0] = h0 ? h0[b * D + d] : 0.0;
            for (int64_t l = 0; l < L; ++l) {
                gather_u(u, L, 4, D, b, l, d, ul);
                oracle_lstm_cell(cs[l], hs[l], ul, ad, &cn, &hn, NULL);
                cs[l + 1] = cn;
                hs[l + 1] = hn;
            }
            double lc = 0.0, lh = 0.0;
            for (int64_t l = L - 1; l >= 0; --l) {
                size_t sidx = (size_t)((b * L + l) * D + d);
                lh += gh[sidx];
                if (gc) lc += gc[sidx];
                gather_u(u, L, 4, D, b, l, d, ul);
                double cp = cs[l], hp = hs[l];
                double i = logistic(ul[0] + ad[0] * hp);
                double f = logistic(ul[1] + ad[1] * hp);
                double o = logistic(ul[2] + ad[2] * hp);
                double g = tanh(ul[3] + ad[3] * hp);
                double t = tanh(f * cp + i * g);
                double gcn = lc + lh * o * (1.0 - t * t); /* total dLoss/dc_l */
                double g_o = lh * t * o * (1.0 - o);
                double g_i = gcn * g * i * (1.0 - i);
                double g_f = gcn * cp * f * (1.0 - f);
                double g_g = gcn * i * (1.0 - g * g);
                double *dul = &du[((b * L + l) * 4) * D + d];
                dul[0 * D] = g_i;
                dul[1 * D] = g_f;
                dul[2 * D] = g_o;
                dul[3 * D] = g_g;
                si += g_i * hp;
                sf += g_f * hp;
                so += g_o * hp;
                sg += g_g * hp;
                lc = gcn * f;
                lh = g_i * ad[0] + g_f * ad[1] + g_o * ad[2] + g_g * ad[3];
            }
            if (dc0) dc0[b * D + d] = lc;
            if (dh0) dh0[b * D + d] = lh;
        }
        da[0 * D + d] = si;
        da[1 * D + d] = sf;
        da[2 * D + d] = so;
        da[3 * D + d] = sg;
        free(cs);
        free(hs);
    }
}

/* ---------------------------------------------------------------- threads */

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
