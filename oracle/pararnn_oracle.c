/*
 * pararnn_oracle.c -- plain, slow, obviously-correct fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links,
 * loads or calls this file; only the tests, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * What it computes (all in double precision, one (b,d) channel at a time):
 *
 *   1. The sequential recurrence h_t = f(h_{t-1}, u_t), t = 1..T.  This is the
 *      plain definition of "applying the RNN to the sequence" and, because the
 *      residual r_t = s_t - f(s_{t-1}) vanishes on it term by term, it is the
 *      unique root of the residual system
 *      [Параллельность RNN?, §1.1 "Постановка как задача нахождения корня"].
 *   2. Back-propagation through time over that trajectory (reverse loop over t
 *      with the transposed per-step Jacobians).
 *   3. A reference DEER/Newton solve that follows the page's steps in order:
 *      evaluate the residual and the sub-diagonal Jacobian blocks at the
 *      current iterate, solve J * ds = -r by forward substitution
 *      ds_1 = -r_1, ds_t = A_t ds_{t-1} - r_t, then s <- s + ds
 *      [Параллельность RNN?, §1.2 "Итерации Ньютона" and §1.3, forward
 *      substitution equations].  It is used for iteration counts and for the
 *      invariants the page fixes (prefix exactness, one-step convergence of an
 *      affine map); the states oracle is (1).
 *   4. The same three for a general cell with a dense D x D Jacobian (the GRU
 *      with full recurrent matrices), at the end of the file.
 *
 * Cells.  Both cells have diagonal recurrent weights, so every channel is an
 * independent scalar (ParaGRU) or 2-state (ParaLSTM) recurrence and the
 * Jacobian of the step is diagonal, resp. 2x2 block-diagonal
 * [Apple научила классические RNN масштабироваться..., "Что именно сделали
 * технически", item 3].  The page gives no cell equations; this file uses the
 * standard GRU/LSTM gate equations with every recurrent matrix replaced by an
 * elementwise weight a_g and the bias added inside each activation:
 *
 *   ParaGRU   z = sig(a_z h + u_z + b_z)      r = sig(a_r h + u_r + b_r)
 *             c = tanh(a_c (r h) + u_c + b_c) h' = (1 - z) h + z c
 *   ParaLSTM  i = sig(a_i h + u_i + b_i)  f = sig(a_f h + u_f + b_f)
 *             g = tanh(a_g h + u_g + b_g) o = sig(a_o h + u_o + b_o)
 *             c' = f c + i g                  h' = o tanh(c')
 *
 * Layouts (row-major, D fastest), identical to the library's:
 *   u    [B][T][G][D]   G = 3 (z,r,c) or 4 (i,f,g,o)
 *   a,b  [G][D]
 *   h0,c0[B][D]
 *   h,c  [B][T][D]      (state after step t, t = 1..T stored at index t-1)
 *
 * Build:  gcc -O2 -fopenmp -shared -fPIC -o _liboracle.so pararnn_oracle.c -lm
 * (no -ffast-math: every operation is an IEEE double operation in source order).
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* threads                                                                   */
/* ------------------------------------------------------------------------- */
void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

#define IDX_U(b, t, g, d) ((((size_t)(b) * T + (t)) * G + (g)) * D + (d))
#define IDX_S(b, t, d) (((size_t)(b) * T + (t)) * D + (d))

/* ========================================================================= */
/* ParaGRU                                                                   */
/* ========================================================================= */

/* One ParaGRU step for a single channel, with all its first derivatives.
 *   f      = h'
 *   A      = df/dh                          (the sub-diagonal Jacobian block)
 *   dfdu[g]= df/du_g  (g = z, r, c)         (== df/db_g)
 *   dfda[g]= df/da_g
 * Derivatives are written out from the chain rule of the equations above. */
typedef struct {
  double z, r, c, f, A, dfdu[3], dfda[3];
} gru_step_t;

static void gru_step(double h, double uz, double ur, double uc, double az,
                     double ar, double ac, double bz, double br, double bc,
                     gru_step_t* s) {
  double z = sigm(az * h + uz + bz);
  double r = sigm(ar * h + ur + br);
  double c = tanh(ac * (r * h) + uc + bc);
  s->z = z;
  s->r = r;
  s->c = c;
  s->f = (1.0 - z) * h + z * c;
  double dz = z * (1.0 - z);   /* dz/d(pre_z) */
  double dr = r * (1.0 - r);   /* dr/d(pre_r) */
  double dc = 1.0 - c * c;     /* dc/d(pre_c) */
  /* df/dpre_z = (c - h) dz ; df/dpre_c = z dc ; df/dpre_r = z dc * ac h * dr */
  double gz = (c - h) * dz;
  double gc = z * dc;
  double gr = gc * ac * h * dr;
  s->dfdu[0] = gz;
  s->dfdu[1] = gr;
  s->dfdu[2] = gc;
  s->dfda[0] = gz * h;        /* d pre_z / d a_z = h     */
  s->dfda[1] = gr * h;        /* d pre_r / d a_r = h     */
  s->dfda[2] = gc * r * h;    /* d pre_c / d a_c = r h   */
  /* df/dh = (1 - z) + gz*az + gc*(ac*r + ac*h*dr*ar) */
  s->A = (1.0 - z) + gz * az + gc * (ac * r + ac * h * dr * ar);
}

/* Vectorised single step over n independent channels (for derivative pins).
 * h[n], u[n][3], a[n][3], bias[n][3] (bias may be NULL) -> f[n], A[n],
 * dfdu[n][3], dfda[n][3] (any output may be NULL). */
void oracle_gru_step(int n, const double* h, const double* u, const double* a,
                     const double* bias, double* f, double* A, double* dfdu,
                     double* dfda) {
  for (int i = 0; i < n; ++i) {
    gru_step_t s;
    double b0 = bias ? bias[3 * i] : 0, b1 = bias ? bias[3 * i + 1] : 0,
           b2 = bias ? bias[3 * i + 2] : 0;
    gru_step(h[i], u[3 * i], u[3 * i + 1], u[3 * i + 2], a[3 * i], a[3 * i + 1],
             a[3 * i + 2], b0, b1, b2, &s);
    if (f) f[i] = s.f;
    if (A) A[i] = s.A;
    for (int g = 0; g < 3; ++g) {
      if (dfdu) dfdu[3 * i + g] = s.dfdu[g];
      if (dfda) dfda[3 * i + g] = s.dfda[g];
    }
  }
}

static void gru_step_at(const double* u, const double* a, const double* bias,
                        int T, int D, int b, int t, int d, double h,
                        gru_step_t* s) {
  const int G = 3;
  double bz = bias ? bias[0 * D + d] : 0, br = bias ? bias[1 * D + d] : 0,
         bc = bias ? bias[2 * D + d] : 0;
  gru_step(h, u[IDX_U(b, t, 0, d)], u[IDX_U(b, t, 1, d)], u[IDX_U(b, t, 2, d)],
           a[0 * D + d], a[1 * D + d], a[2 * D + d], bz, br, bc, s);
}

/* Sequential evaluation: h_t = f(h_{t-1}, u_t) for t = 1..T. */
void oracle_gru_seq(const double* u, const double* a, const double* bias,
                    const double* h0, double* h, int B, int T, int D) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int d = 0; d < D; ++d) {
      double hp = h0 ? h0[(size_t)b * D + d] : 0.0;
      for (int t = 0; t < T; ++t) {
        gru_step_t s;
        gru_step_at(u, a, bias, T, D, b, t, d, hp, &s);
        h[IDX_S(b, t, d)] = s.f;
        hp = s.f;
      }
    }
}

/* Residual r_t = h_t - f(h_{t-1}, u_t) of a candidate trajectory h. */
void oracle_gru_residual(const double* u, const double* a, const double* bias,
                         const double* h0, const double* h, double* res, int B,
                         int T, int D) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int d = 0; d < D; ++d) {
      double hp = h0 ? h0[(size_t)b * D + d] : 0.0;
      for (int t = 0; t < T; ++t) {
        gru_step_t s;
        gru_step_at(u, a, bias, T, D, b, t, d, hp, &s);
        res[IDX_S(b, t, d)] = h[IDX_S(b, t, d)] - s.f;
        hp = h[IDX_S(b, t, d)];
      }
    }
}

/* BPTT over a trajectory h (normally the sequential one).
 *   lambda_T = g_T ; lambda_t = g_t + A_{t+1} lambda_{t+1}
 *   du_t = dfdu_t * lambda_t ; da = sum_{b,t} dfda_t * lambda_t ;
 *   dbias = sum_{b,t} du_t ; dh0 = A_1 lambda_1
 * du [B][T][3][D], da [3][D], dbias [3][D] (may be NULL), dh0 [B][D] (NULL ok).
 * Parallel over d; each d owns its da/dbias entries (no races, fixed order). */
void oracle_gru_bptt(const double* u, const double* a, const double* bias,
                     const double* h0, const double* h, const double* dLdh,
                     double* du, double* da, double* dbias, double* dh0, int B,
                     int T, int D) {
  const int G = 3;
#pragma omp parallel for schedule(static)
  for (int d = 0; d < D; ++d) {
    double sa[3] = {0, 0, 0}, sb[3] = {0, 0, 0};
    for (int b = 0; b < B; ++b) {
      double lam_next = 0.0; /* lambda_{t+1} */
      double A_next = 0.0;   /* A_{t+1}      */
      for (int t = T - 1; t >= 0; --t) {
        double hp = t > 0 ? h[IDX_S(b, t - 1, d)]
                          : (h0 ? h0[(size_t)b * D + d] : 0.0);
        gru_step_t s;
        gru_step_at(u, a, bias, T, D, b, t, d, hp, &s);
        double lam = dLdh[IDX_S(b, t, d)] + A_next * lam_next;
        for (int g = 0; g < 3; ++g) {
          double dug = s.dfdu[g] * lam;
          du[IDX_U(b, t, g, d)] = dug;
          sa[g] += s.dfda[g] * lam;
          sb[g] += dug;
        }
        lam_next = lam;
        A_next = s.A;
      }
      if (dh0) dh0[(size_t)b * D + d] = A_next * lam_next;
    }
    for (int g = 0; g < 3; ++g) {
      da[g * D + d] = sa[g];
      if (dbias) dbias[g * D + d] = sb[g];
    }
  }
}

/* Reference DEER/Newton for ParaGRU.
 * h (in/out) [B][T][D]: initial guess in, final iterate out.
 * Loop: evaluate r at the iterate; record max|r| in trace[k]; stop if
 * max|r| < tol or k == max_iters; else forward-substitute ds and update.
 * iters_out = number of updates applied.  trace has max_iters+1 entries.
 * chan_k [B][D] (may be NULL): per channel, the first iterate index k from
 * which that channel's max_t |r_t| stays < tol (k = last failing index + 1).
 * The whole [B,T,D] system is one Newton system; stopping is global. */
void oracle_gru_newton(const double* u, const double* a, const double* bias,
                       const double* h0, double* h, int B, int T, int D,
                       double tol, int max_iters, double* trace, int* iters_out,
                       int* chan_k) {
  size_t n = (size_t)B * T * D;
  double* res = (double*)malloc(n * sizeof(double));
  double* A = (double*)malloc(n * sizeof(double));
  int* last_bad = (int*)malloc((size_t)B * D * sizeof(int));
  for (size_t i = 0; i < (size_t)B * D; ++i) last_bad[i] = -1;
  int k = 0;
  for (;; ++k) {
    double m = 0.0;
    int nonfinite = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(max : m) reduction(| : nonfinite)
    for (int b = 0; b < B; ++b)
      for (int d = 0; d < D; ++d) {
        double hp = h0 ? h0[(size_t)b * D + d] : 0.0, mc = 0.0;
        for (int t = 0; t < T; ++t) {
          gru_step_t s;
          gru_step_at(u, a, bias, T, D, b, t, d, hp, &s);
          double rt = h[IDX_S(b, t, d)] - s.f;
          res[IDX_S(b, t, d)] = rt;
          A[IDX_S(b, t, d)] = s.A; /* df/dh evaluated at h_{t-1} */
          if (!isfinite(rt)) nonfinite = 1;
          if (fabs(rt) > mc) mc = fabs(rt);
          hp = h[IDX_S(b, t, d)];
        }
        if (!(mc < tol)) last_bad[(size_t)b * D + d] = k;
        if (mc > m) m = mc;
      }
    if (nonfinite) m = INFINITY;
    if (trace) trace[k] = m;
    if (m < tol || k >= max_iters) break;
    /* forward substitution: ds_1 = -r_1 ; ds_t = A_t ds_{t-1} - r_t */
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int d = 0; d < D; ++d) {
        double ds = 0.0;
        for (int t = 0; t < T; ++t) {
          size_t i = IDX_S(b, t, d);
          ds = (t == 0 ? 0.0 : A[i] * ds) - res[i];
          h[i] += ds;
        }
      }
  }
  if (iters_out) *iters_out = k;
  if (chan_k)
    for (size_t i = 0; i < (size_t)B * D; ++i) chan_k[i] = last_bad[i] + 1;
  free(res);
  free(A);
  free(last_bad);
}

/* Forward substitution of a scalar linear recurrence, the page's solver for
 * J ds = -r with ds_0 = x0:  x_t = A_t x_{t-1} + b_t, t = 1..n.
 * Used by the scan pins (compared against the closed form and tree orders). */
void oracle_linrec(int n, const double* A, const double* b, double x0,
                   double* x) {
  double p = x0;
  for (int t = 0; t < n; ++t) {
    p = A[t] * p + b[t];
    x[t] = p;
  }
}

/* ========================================================================= */
/* ParaLSTM                                                                  */
/* ========================================================================= */

/* One ParaLSTM step for one channel with state s = (c, h).
 *   fc, fh      = c', h'
 *   A[2][2]     = d(c',h')/d(c,h)           (the 2x2 Jacobian block)
 *   dfdu[2][4]  = d(c',h')/du_g, g = i,f,g,o   (== d/db_g)
 *   dfda[2][4]  = d(c',h')/da_g                                        */
typedef struct {
  double fc, fh, A[2][2], dfdu[2][4], dfda[2][4];
} lstm_step_t;

static void lstm_step(double c, double h, const double u[4], const double a[4],
                      const double bb[4], lstm_step_t* s) {
  double i = sigm(a[0] * h + u[0] + bb[0]);
  double f = sigm(a[1] * h + u[1] + bb[1]);
  double g = tanh(a[2] * h + u[2] + bb[2]);
  double o = sigm(a[3] * h + u[3] + bb[3]);
  double cn = f * c + i * g;
  double tc = tanh(cn);
  double hn = o * tc;
  s->fc = cn;
  s->fh = hn;
  /* derivatives of the gates w.r.t. their pre-activations */
  double di = i * (1.0 - i), df = f * (1.0 - f), dg = 1.0 - g * g,
         dox = o * (1.0 - o);
  double dtc = 1.0 - tc * tc; /* d tanh(c') / d c' */
  /* d c' / d pre_{i,f,g,o} */
  double gcp[4] = {g * di, c * df, i * dg, 0.0};
  /* d h' / d pre = o * dtc * dc'/dpre  (+ tanh(c') * do/dpre for o) */
  double ghp[4] = {o * dtc * gcp[0], o * dtc * gcp[1], o * dtc * gcp[2],
                   tc * dox};
  for (int q = 0; q < 4; ++q) {
    s->dfdu[0][q] = gcp[q];
    s->dfdu[1][q] = ghp[q];
    s->dfda[0][q] = gcp[q] * h; /* d pre_q / d a_q = h */
    s->dfda[1][q] = ghp[q] * h;
  }
  /* d/dc: only c' = f c + ... depends on c directly */
  double dcn_dc = f;
  /* d/dh: through every pre-activation, d pre_q/dh = a_q */
  double dcn_dh = gcp[0] * a[0] + gcp[1] * a[1] + gcp[2] * a[2];
  s->A[0][0] = dcn_dc;
  s->A[0][1] = dcn_dh;
  s->A[1][0] = o * dtc * dcn_dc;
  s->A[1][1] = ghp[3] * a[3] + o * dtc * dcn_dh;
}

static void lstm_step_at(const double* u, const double* a, const double* bias,
                         int T, int D, int b, int t, int d, double c, double h,
                         lstm_step_t* s) {
  const int G = 4;
  double uu[4], aa[4], bb[4];
  for (int q = 0; q < 4; ++q) {
    uu[q] = u[IDX_U(b, t, q, d)];
    aa[q] = a[q * D + d];
    bb[q] = bias ? bias[q * D + d] : 0.0;
  }
  lstm_step(c, h, uu, aa, bb, s);
}

/* Vectorised single step (for derivative pins).  c[n], h[n], u[n][4],
 * a[n][4], bias[n][4] (NULL ok) -> fc[n], fh[n], A[n][2][2], dfdu[n][2][4],
 * dfda[n][2][4]. */
void oracle_lstm_step(int n, const double* c, const double* h, const double* u,
                      const double* a, const double* bias, double* fc,
                      double* fh, double* A, double* dfdu, double* dfda) {
  static const double zero4[4] = {0, 0, 0, 0};
  for (int k = 0; k < n; ++k) {
    lstm_step_t s;
    lstm_step(c[k], h[k], u + 4 * k, a + 4 * k, bias ? bias + 4 * k : zero4,
              &s);
    if (fc) fc[k] = s.fc;
    if (fh) fh[k] = s.fh;
    for (int p = 0; p < 2; ++p) {
      for (int q = 0; q < 2; ++q)
        if (A) A[4 * k + 2 * p + q] = s.A[p][q];
      for (int q = 0; q < 4; ++q) {
        if (dfdu) dfdu[8 * k + 4 * p + q] = s.dfdu[p][q];
        if (dfda) dfda[8 * k + 4 * p + q] = s.dfda[p][q];
      }
    }
  }
}

void oracle_lstm_seq(const double* u, const double* a, const double* bias,
                     const double* c0, const double* h0, double* c, double* h,
                     int B, int T, int D) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int d = 0; d < D; ++d) {
      double cp = c0 ? c0[(size_t)b * D + d] : 0.0;
      double hp = h0 ? h0[(size_t)b * D + d] : 0.0;
      for (int t = 0; t < T; ++t) {
        lstm_step_t s;
        lstm_step_at(u, a, bias, T, D, b, t, d, cp, hp, &s);
        c[IDX_S(b, t, d)] = s.fc;
        h[IDX_S(b, t, d)] = s.fh;
        cp = s.fc;
        hp = s.fh;
      }
    }
}

void oracle_lstm_residual(const double* u, const double* a, const double* bias,
                          const double* c0, const double* h0, const double* c,
                          const double* h, double* rc, double* rh, int B, int T,
                          int D) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int d = 0; d < D; ++d) {
      double cp = c0 ? c0[(size_t)b * D + d] : 0.0;
      double hp = h0 ? h0[(size_t)b * D + d] : 0.0;
      for (int t = 0; t < T; ++t) {
        lstm_step_t s;
        size_t i = IDX_S(b, t, d);
        lstm_step_at(u, a, bias, T, D, b, t, d, cp, hp, &s);
        rc[i] = c[i] - s.fc;
        rh[i] = h[i] - s.fh;
        cp = c[i];
        hp = h[i];
      }
    }
}

/* BPTT for ParaLSTM.  The loss depends on h only (dL/dc_t = 0 explicitly);
 * lambda_t = (lc, lh) = (0, g_t) + A_{t+1}^T lambda_{t+1}.
 * du [B][T][4][D]; da, dbias [4][D]; dc0, dh0 [B][D] (NULL ok). */
void oracle_lstm_bptt(const double* u, const double* a, const double* bias,
                      const double* c0, const double* h0, const double* c,
                      const double* h, const double* dLdh, double* du,
                      double* da, double* dbias, double* dc0, double* dh0,
                      int B, int T, int D) {
  const int G = 4;
#pragma omp parallel for schedule(static)
  for (int d = 0; d < D; ++d) {
    double sa[4] = {0, 0, 0, 0}, sb[4] = {0, 0, 0, 0};
    for (int b = 0; b < B; ++b) {
      double lc_n = 0.0, lh_n = 0.0;                /* lambda_{t+1}  */
      double An[2][2] = {{0.0, 0.0}, {0.0, 0.0}};  /* A_{t+1}       */
      for (int t = T - 1; t >= 0; --t) {
        double cp, hp;
        if (t > 0) {
          cp = c[IDX_S(b, t - 1, d)];
          hp = h[IDX_S(b, t - 1, d)];
        } else {
          cp = c0 ? c0[(size_t)b * D + d] : 0.0;
          hp = h0 ? h0[(size_t)b * D + d] : 0.0;
        }
        lstm_step_t s;
        lstm_step_at(u, a, bias, T, D, b, t, d, cp, hp, &s);
        /* lambda_t = g_t + A_{t+1}^T lambda_{t+1} */
        double lc = 0.0 + An[0][0] * lc_n + An[1][0] * lh_n;
        double lh = dLdh[IDX_S(b, t, d)] + An[0][1] * lc_n + An[1][1] * lh_n;
        for (int q = 0; q < 4; ++q) {
          double duq = s.dfdu[0][q] * lc + s.dfdu[1][q] * lh;
          du[IDX_U(b, t, q, d)] = duq;
          sa[q] += s.dfda[0][q] * lc + s.dfda[1][q] * lh;
          sb[q] += duq;
        }
        lc_n = lc;
        lh_n = lh;
        memcpy(An, s.A, sizeof(An));
      }
      /* d L / d (c0, h0) = A_1^T lambda_1 */
      if (dc0) dc0[(size_t)b * D + d] = An[0][0] * lc_n + An[1][0] * lh_n;
      if (dh0) dh0[(size_t)b * D + d] = An[0][1] * lc_n + An[1][1] * lh_n;
    }
    for (int q = 0; q < 4; ++q) {
      da[q * D + d] = sa[q];
      if (dbias) dbias[q * D + d] = sb[q];
    }
  }
}

/* Reference DEER/Newton for ParaLSTM on the stacked state s_t = (c_t, h_t);
 * same loop and outputs as oracle_gru_newton, the residual norm being the max
 * over both components. */
void oracle_lstm_newton(const double* u, const double* a, const double* bias,
                        const double* c0, const double* h0, double* c,
                        double* h, int B, int T, int D, double tol,
                        int max_iters, double* trace, int* iters_out,
                        int* chan_k) {
  size_t n = (size_t)B * T * D;
  double* rc = (double*)malloc(n * sizeof(double));
  double* rh = (double*)malloc(n * sizeof(double));
  double* J = (double*)malloc(4 * n * sizeof(double));
  int* last_bad = (int*)malloc((size_t)B * D * sizeof(int));
  for (size_t i = 0; i < (size_t)B * D; ++i) last_bad[i] = -1;
  int k = 0;
  for (;; ++k) {
    double m = 0.0;
    int nonfinite = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(max : m) reduction(| : nonfinite)
    for (int b = 0; b < B; ++b)
      for (int d = 0; d < D; ++d) {
        double cp = c0 ? c0[(size_t)b * D + d] : 0.0;
        double hp = h0 ? h0[(size_t)b * D + d] : 0.0, mc = 0.0;
        for (int t = 0; t < T; ++t) {
          size_t i = IDX_S(b, t, d);
          lstm_step_t s;
          lstm_step_at(u, a, bias, T, D, b, t, d, cp, hp, &s);
          rc[i] = c[i] - s.fc;
          rh[i] = h[i] - s.fh;
          J[4 * i + 0] = s.A[0][0];
          J[4 * i + 1] = s.A[0][1];
          J[4 * i + 2] = s.A[1][0];
          J[4 * i + 3] = s.A[1][1];
          if (!isfinite(rc[i]) || !isfinite(rh[i])) nonfinite = 1;
          if (fabs(rc[i]) > mc) mc = fabs(rc[i]);
          if (fabs(rh[i]) > mc) mc = fabs(rh[i]);
          cp = c[i];
          hp = h[i];
        }
        if (!(mc < tol)) last_bad[(size_t)b * D + d] = k;
        if (mc > m) m = mc;
      }
    if (nonfinite) m = INFINITY;
    if (trace) trace[k] = m;
    if (m < tol || k >= max_iters) break;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int d = 0; d < D; ++d) {
        double dc = 0.0, dh = 0.0;
        for (int t = 0; t < T; ++t) {
          size_t i = IDX_S(b, t, d);
          double nc = -rc[i], nh = -rh[i];
          if (t > 0) {
            nc += J[4 * i + 0] * dc + J[4 * i + 1] * dh;
            nh += J[4 * i + 2] * dc + J[4 * i + 3] * dh;
          }
          dc = nc;
          dh = nh;
          c[i] += dc;
          h[i] += dh;
        }
      }
  }
  if (iters_out) *iters_out = k;
  if (chan_k)
    for (size_t i = 0; i < (size_t)B * D; ++i) chan_k[i] = last_bad[i] + 1;
  free(rc);
  free(rh);
  free(J);
  free(last_bad);
}

/* ------------------------------------------------------------------------- */
/* A general cell: the GRU with full recurrent matrices (dense Jacobian)     */
/* ------------------------------------------------------------------------- */
/*
 * The Newton step of the pages holds for any Markov cell: the Jacobian of the
 * residual is block-bidiagonal, identity blocks on the diagonal and
 * -df/ds(s_{t-1}) below it, a full D x D matrix for a general cell
 * [Параллельность RNN?, §1.3, the block-bidiagonal J and "Сколько нам реально
 * нужно памяти"].  The general cell here is the standard GRU with full
 * recurrent matrices W [3][D][D] (row i of W_g feeds h into gate g of unit i),
 * the reset gate applied to the recurrent term of the candidate, as in
 * PyTorch's GRU cell:
 *
 *   z = sig(W_z h + u_z + b_z)        r = sig(W_r h + u_r + b_r)
 *   q = W_c h                         c = tanh(u_c + b_c + r q)
 *   h' = (1 - z) h + z c              (products of vectors elementwise)
 *
 * With W_g = diag(a_g), r q = a_c (r h) and this is the ParaGRU cell above.
 * Its Jacobian, by the chain rule on each line:
 *
 *   dh'/dh = diag(1 - z) + diag((c - h) z (1 - z)) W_z
 *            + diag(z (1 - c^2)) [diag(r) W_c + diag(q r (1 - r)) W_r]
 *
 * Layouts: u [B][T][3][D] as for ParaGRU, W [3][D][D] row-major, bias [3][D],
 * h0 [B][D], h [B][T][D], J [D][D] row-major (J[i][j] = dh'_i / dh_j).
 */
#define DW(g, i, j) W[((size_t)(g) * D + (i)) * D + (j)]

/* One step for one batch row: h [D], u [3][D] (gate stride D) -> hn [D] and,
 * if J is not NULL, the Jacobian [D][D].  work holds 4 D doubles. */
static void dense_gru_cell(int D, const double* W, const double* bias, const double* h,
                           const double* u, double* hn, double* J, double* work) {
  double* z = work;
  double* r = work + D;
  double* q = work + 2 * D;
  double* c = work + 3 * D;
  for (int i = 0; i < D; ++i) {
    double pz = u[i] + (bias ? bias[i] : 0.0), pr = u[D + i] + (bias ? bias[D + i] : 0.0);
    double qi = 0.0;
    for (int j = 0; j < D; ++j) {
      pz += DW(0, i, j) * h[j];
      pr += DW(1, i, j) * h[j];
      qi += DW(2, i, j) * h[j];
    }
    z[i] = sigm(pz);
    r[i] = sigm(pr);
    q[i] = qi;
  }
  for (int i = 0; i < D; ++i) {
    c[i] = tanh(u[2 * D + i] + (bias ? bias[2 * D + i] : 0.0) + r[i] * q[i]);
    hn[i] = (1.0 - z[i]) * h[i] + z[i] * c[i];
  }
  if (!J) return;
  for (int i = 0; i < D; ++i) {
    const double gz = (c[i] - h[i]) * z[i] * (1.0 - z[i]);
    const double gc = z[i] * (1.0 - c[i] * c[i]);
    const double gr = q[i] * r[i] * (1.0 - r[i]);
    for (int j = 0; j < D; ++j)
      J[(size_t)i * D + j] = (i == j ? 1.0 - z[i] : 0.0) + gz * DW(0, i, j) +
                             gc * (r[i] * DW(2, i, j) + gr * DW(1, i, j));
  }
}

/* Single step over a batch: h [n][D], u [n][3][D] -> hn [n][D], J [n][D][D]
 * (J may be NULL). */
void oracle_dense_gru_step(int n, int D, const double* h, const double* u, const double* W,
                           const double* bias, double* hn, double* J) {
#pragma omp parallel for schedule(static)
  for (int b = 0; b < n; ++b) {
    double* work = (double*)malloc(4 * (size_t)D * sizeof(double));
    dense_gru_cell(D, W, bias, h + (size_t)b * D, u + (size_t)b * 3 * D, hn + (size_t)b * D,
                   J ? J + (size_t)b * D * D : NULL, work);
    free(work);
  }
}

/* The sequential recurrence h_t = f(h_{t-1}, u_t) with the general cell. */
void oracle_dense_gru_seq(const double* u, const double* W, const double* bias,
                          const double* h0, double* h, int B, int T, int D) {
#pragma omp parallel for schedule(static)
  for (int b = 0; b < B; ++b) {
    double* work = (double*)malloc(5 * (size_t)D * sizeof(double));
    double* hp = work + 4 * D;
    for (int d = 0; d < D; ++d) hp[d] = h0 ? h0[(size_t)b * D + d] : 0.0;
    for (int t = 0; t < T; ++t) {
      double* ht = h + ((size_t)b * T + t) * D;
      dense_gru_cell(D, W, bias, hp, u + ((size_t)b * T + t) * 3 * D, ht, NULL, work);
      memcpy(hp, ht, (size_t)D * sizeof(double));
    }
    free(work);
  }
}

/* Reference DEER/Newton with dense Jacobian blocks, in the pages' order:
 * evaluate r_t = h_t - f(h_{t-1}) and J_t = df/dh(h_{t-1}) at the iterate,
 * record max|r| in trace[k], stop if it is below tol or k == max_iters, else
 * forward-substitute ds_t = J_t ds_{t-1} - r_t (ds_0 = 0: h0 is given) and
 * update h += ds.  h (in/out) [B][T][D] holds the initial guess and the final
 * iterate; iters_out = updates applied; trace has max_iters + 1 entries.  The
 * whole [B, T, D] system is one Newton system (global stopping). */
void oracle_dense_gru_newton(const double* u, const double* W, const double* bias,
                             const double* h0, double* h, int B, int T, int D, double tol,
                             int max_iters, double* trace, int* iters_out) {
  const size_t n = (size_t)B * T * D;
  double* res = (double*)malloc(n * sizeof(double));
  double* J = (double*)malloc(n * (size_t)D * sizeof(double));
  int k = 0;
  for (;; ++k) {
    double m = 0.0;
    int nonfinite = 0;
#pragma omp parallel for schedule(static) reduction(max : m) reduction(| : nonfinite)
    for (int b = 0; b < B; ++b) {
      double* work = (double*)malloc(5 * (size_t)D * sizeof(double));
      double* f = work + 4 * D;
      for (int t = 0; t < T; ++t) {
        const double* hp = t > 0 ? h + ((size_t)b * T + t - 1) * D : NULL;
        double* zero = NULL;
        if (!hp) { /* the state before step 1 is h0 (zeros when absent) */
          zero = (double*)calloc((size_t)D, sizeof(double));
          if (h0) memcpy(zero, h0 + (size_t)b * D, (size_t)D * sizeof(double));
          hp = zero;
        }
        const size_t o = ((size_t)b * T + t) * D;
        dense_gru_cell(D, W, bias, hp, u + o * 3, f, J + o * D, work);
        for (int d = 0; d < D; ++d) {
          const double rt = h[o + d] - f[d];
          res[o + d] = rt;
          if (!isfinite(rt)) nonfinite = 1;
          if (fabs(rt) > m) m = fabs(rt);
        }
        free(zero);
      }
      free(work);
    }
    if (nonfinite) m = INFINITY;
    if (trace) trace[k] = m;
    if (m < tol || k >= max_iters) break;
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b) {
      double* ds = (double*)calloc((size_t)D, sizeof(double));
      double* nx = (double*)malloc((size_t)D * sizeof(double));
      for (int t = 0; t < T; ++t) {
        const size_t o = ((size_t)b * T + t) * D;
        for (int i = 0; i < D; ++i) {
          double v = -res[o + i];
          if (t > 0)
            for (int j = 0; j < D; ++j) v += J[(o + i) * D + j] * ds[j];
          nx[i] = v;
        }
        for (int i = 0; i < D; ++i) {
          ds[i] = nx[i];
          h[o + i] += nx[i];
        }
      }
      free(ds);
      free(nx);
    }
  }
  if (iters_out) *iters_out = k;
  free(res);
  free(J);
}
#undef DW
