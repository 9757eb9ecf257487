/*
 * m3_oracle.c -- fp64 CPU oracle of the Mamba-3 SSM layer core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header or table with the CUDA path.
 *
 * What it computes (one independent recurrence per (batch, head); g is the
 * B/C/theta group of head h, g = h / (H/G)):
 *
 *   Bb_{t,r} = B[b,t,g,r,:] + bias_B[h,r,:]        Cb_{t,r} = C[b,t,g,r,:] + bias_C[h,r,:]
 *   X_{t,r}  = W_x[h,r,:] * x[b,t,h,:]              (MIMO input branches)
 *   u_t      = sum_r Bb_{t,r} X_{t,r}^T             (N x P, rank <= R update)
 *   alpha_t  = exp(dt_t A_t), beta'_t = (1 - lam_t) dt_t, gamma_t = lam_t dt_t
 *   phi_{t,k}= dt_t theta[b,t,g,k]                  (rotation of complex pair k; theta[b,t,g,k]
 *                                                    itself in the direct-angle variant)
 *   h_t      = alpha_t Rot(phi_t) (h_{t-1} + beta'_t u_{t-1}) + gamma_t u_t
 *   Y_{t,r}  = Cb_{t,r}^T h_t ;  y[b,t,h,:] = sum_r W_o[h,r,:] * Y_{t,r} + D_h x[b,t,h,:]
 *
 * Sources (Mamba-3 paper note, docsaid.org, "Mamba-3: Improved Sequence Modeling
 * using State Space Principles"):
 *   - section "その1 表現力の高い離散化": the exponential-trapezoidal recurrence
 *     h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1} + gamma_t B_t x_t with
 *     alpha = e^{dt A}, beta = (1-lam) dt e^{dt A}, gamma = lam dt.  Written above
 *     as alpha Rot (h + beta' u_{t-1}) because beta = beta' * e^{dt A}.
 *   - section "その2 複素数の状態": the complex SSM equals a real SSM of doubled
 *     size whose transition is the decay times a block diagonal of 2x2 rotations
 *     [[c, -s], [s, c]] (the rotation used in that section's parity example).
 *     The pairs are adjacent state rows (2k, 2k+1); the angle of step t is
 *     dt_t * theta_t, i.e. theta is the imaginary part of A in e^{dt A}.
 *   - section "その3 MIMO": R input branches of x and B, rank <= R state update,
 *     R readouts with their own C; state size unchanged.
 *   - IBM page "Mamba モデルとは", state-space equations: the D x skip term.
 *   - Cartesia blog "Mamba-3", section アーキテクチャ: the B/C bias is added
 *     after the B/C normalisation (the normalisation happens before the core).
 *
 * Readings where the pages leave a step open (each listed in the design notes):
 *   - the previous-input term at the first token comes from the carried state
 *     (carry_B, carry_x); a fresh, all-zero carry means no such term;
 *   - beta's e^{dt A} includes the rotation (A is complex);
 *   - the R branches are formed by per-rank, per-channel scales W_x (in) and
 *     W_o (out); NULL W_x / W_o mean all ones, NULL bias means zero, NULL D
 *     means no skip term.
 *
 * Layouts (row-major, last index fastest):
 *   x, y      (b, L, H, P)      dt, A, lam (b, L, H)
 *   B, C      (b, L, G, R, N)   theta      (b, L, G, N/2)
 *   bias_B/C  (H, R, N)         W_x, W_o   (H, R, P)     D (H)
 *   h         (b, H, N, P)      carry_B    (b, H, R, N)  carry_x (b, H, P)
 * h, carry_B and carry_x are read as the initial state and overwritten with
 * the final state (the carry holds the last token's raw B and x).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int64_t b, L;
  int32_t H, P, N, R, G;
  int32_t angle_direct; /* variant: phi_{t,k} = theta[b,t,g,k] (no dt factor) */
} m3o_dims;

/* One (batch, head) recurrence over all L tokens.  Returns 0, or -1 on OOM. */
static int scan_one(const m3o_dims* d, int64_t bi, int32_t hi,
                    const double* x, const double* dt, const double* A, const double* lam,
                    const double* B, const double* C, const double* theta,
                    const double* bias_B, const double* bias_C,
                    const double* W_x, const double* W_o, const double* D,
                    double* h, double* carry_B, double* carry_x, double* y) {
  const int64_t L = d->L;
  const int32_t H = d->H, P = d->P, N = d->N, R = d->R, G = d->G;
  const int32_t K = N / 2;
  const int32_t g = hi / (H / G);
  double* hs = h + ((bi * H + hi) * (int64_t)N) * P;          /* state, updated in place */
  double* cB = carry_B + ((bi * H + hi) * (int64_t)R) * N;     /* previous raw B (R x N) */
  double* cx = carry_x + (bi * H + hi) * (int64_t)P;           /* previous raw x (P) */

  double* u = (double*)malloc(sizeof(double) * (size_t)N * P);
  double* up = (double*)malloc(sizeof(double) * (size_t)N * P);
  double* Bb = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* Bbp = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* Cb = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* X = (double*)malloc(sizeof(double) * (size_t)R * P);
  double* Xp = (double*)malloc(sizeof(double) * (size_t)R * P);
  double* Y = (double*)malloc(sizeof(double) * (size_t)R * P);
  if (!u || !up || !Bb || !Bbp || !Cb || !X || !Xp || !Y) {
    free(u); free(up); free(Bb); free(Bbp); free(Cb); free(X); free(Xp); free(Y);
    return -1;
  }

  for (int64_t t = 0; t < L; ++t) {
    const int64_t tok = bi * L + t;
    const double delta = dt[tok * H + hi];
    const double a = A[tok * H + hi];
    const double lm = lam[tok * H + hi];
    const double alpha = exp(delta * a);
    const double bprime = (1.0 - lm) * delta;
    const double gamma = lm * delta;
    const double* xt = x + (tok * H + hi) * (int64_t)P;
    const double* Bt = B + ((tok * G + g) * (int64_t)R) * N;
    const double* Ct = C + ((tok * G + g) * (int64_t)R) * N;
    const double* th = theta + (tok * G + g) * (int64_t)K;

    /* biased B and C of this token and of the previous one; MIMO input branches */
    for (int32_t r = 0; r < R; ++r) {
      for (int32_t n = 0; n < N; ++n) {
        const double bb = bias_B ? bias_B[((int64_t)hi * R + r) * N + n] : 0.0;
        const double bc = bias_C ? bias_C[((int64_t)hi * R + r) * N + n] : 0.0;
        Bb[r * N + n] = Bt[r * N + n] + bb;
        Bbp[r * N + n] = cB[r * N + n] + bb;
        Cb[r * N + n] = Ct[r * N + n] + bc;
      }
      for (int32_t p = 0; p < P; ++p) {
        const double wx = W_x ? W_x[((int64_t)hi * R + r) * P + p] : 1.0;
        X[r * P + p] = wx * xt[p];
        Xp[r * P + p] = wx * cx[p];
      }
    }
    /* u_t and u_{t-1}: sums of R outer products */
    for (int32_t n = 0; n < N; ++n) {
      for (int32_t p = 0; p < P; ++p) {
        double s = 0.0, sp = 0.0;
        for (int32_t r = 0; r < R; ++r) {
          s += Bb[r * N + n] * X[r * P + p];
          sp += Bbp[r * N + n] * Xp[r * P + p];
        }
        u[(int64_t)n * P + p] = s;
        up[(int64_t)n * P + p] = sp;
      }
    }
    /* h_t = alpha Rot(phi) (h_{t-1} + beta' u_{t-1}) + gamma u_t, pair by pair */
    for (int32_t k = 0; k < K; ++k) {
      const double phi = d->angle_direct ? th[k] : delta * th[k];
      const double c = cos(phi), s = sin(phi);
      double* h0 = hs + (int64_t)(2 * k) * P;
      double* h1 = hs + (int64_t)(2 * k + 1) * P;
      const double* u0 = u + (int64_t)(2 * k) * P;
      const double* u1 = u + (int64_t)(2 * k + 1) * P;
      const double* q0 = up + (int64_t)(2 * k) * P;
      const double* q1 = up + (int64_t)(2 * k + 1) * P;
      for (int32_t p = 0; p < P; ++p) {
        const double v0 = h0[p] + bprime * q0[p];
        const double v1 = h1[p] + bprime * q1[p];
        h0[p] = alpha * (c * v0 - s * v1) + gamma * u0[p];
        h1[p] = alpha * (s * v0 + c * v1) + gamma * u1[p];
      }
    }
    /* readout: Y_r = Cb_r^T h, y = sum_r W_o_r * Y_r + D x */
    for (int32_t r = 0; r < R; ++r)
      for (int32_t p = 0; p < P; ++p) Y[r * P + p] = 0.0;
    for (int32_t n = 0; n < N; ++n) {
      const double* hn = hs + (int64_t)n * P;
      for (int32_t r = 0; r < R; ++r) {
        const double cn = Cb[r * N + n];
        for (int32_t p = 0; p < P; ++p) Y[r * P + p] += cn * hn[p];
      }
    }
    double* yt = y + (tok * H + hi) * (int64_t)P;
    const double dh = D ? D[hi] : 0.0;
    for (int32_t p = 0; p < P; ++p) {
      double s = 0.0;
      for (int32_t r = 0; r < R; ++r) {
        const double wo = W_o ? W_o[((int64_t)hi * R + r) * P + p] : 1.0;
        s += wo * Y[r * P + p];
      }
      yt[p] = s + dh * xt[p];
    }
    /* this token becomes the previous one */
    memcpy(cB, Bt, sizeof(double) * (size_t)R * N);
    memcpy(cx, xt, sizeof(double) * (size_t)P);
  }
  free(u); free(up); free(Bb); free(Bbp); free(Cb); free(X); free(Xp); free(Y);
  return 0;
}

/*
 * m3o_scan: run the recurrence for the (batch, head) pairs listed in sel
 * (entries bi*H + hi), or for all pairs when sel is NULL.  Pairs are independent
 * and are spread over OpenMP threads (nthreads <= 0: the OpenMP default).
 * y rows of pairs not selected are left untouched.
 * Returns 0 on success, -1 on bad dimensions, -2 on allocation failure.
 */
int m3o_scan(const m3o_dims* d,
             const double* x, const double* dt, const double* A, const double* lam,
             const double* B, const double* C, const double* theta,
             const double* bias_B, const double* bias_C,
             const double* W_x, const double* W_o, const double* D,
             double* h, double* carry_B, double* carry_x, double* y,
             const int64_t* sel, int64_t nsel, int nthreads) {
  if (!d || d->b < 0 || d->L < 0 || d->H <= 0 || d->P <= 0 || d->N <= 0 || d->R <= 0 ||
      d->G <= 0 || (d->N % 2) != 0 || (d->H % d->G) != 0)
    return -1;
  const int64_t npairs = sel ? nsel : d->b * d->H;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
  for (int64_t i = 0; i < npairs; ++i) {
    const int64_t id = sel ? sel[i] : i;
    if (id < 0 || id >= d->b * d->H) { err |= 1; continue; }
    if (scan_one(d, id / d->H, (int32_t)(id % d->H), x, dt, A, lam, B, C, theta,
                 bias_B, bias_C, W_x, W_o, D, h, carry_B, carry_x, y) != 0)
      err |= 2;
  }
  if (err & 1) return -1;
  if (err & 2) return -2;
  return 0;
}

int m3o_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
