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

/*
 * Reverse-mode gradient of the same recurrence (the backward pass of the layer core).
 *
 * For one (batch, head) it runs the forward recurrence of scan_one once, keeping every state
 * h_t, then walks t = L-1 .. 0 and applies the chain rule to each line of the forward step,
 * in reverse order:
 *   y_t     = sum_r W_o_r * (Cb_{t,r}^T h_t) + D x_t
 *   h_t     = alpha_t Rot(phi_t) z_t + gamma_t u_t,      z_t = h_{t-1} + beta'_t u_{t-1}
 *   u_t     = sum_r Bb_{t,r} X_{t,r}^T,  X_{t,r} = W_x_r * x_t,  Bb = B + bias_B, Cb = C + bias_C
 *   alpha_t = exp(dt_t A_t), beta'_t = (1 - lam_t) dt_t, gamma_t = lam_t dt_t,
 *   phi_{t,k} = dt_t theta_{t,k} (theta_{t,k} in the direct-angle variant).
 * u_{t-1} enters two steps (gamma at t-1, beta' at t), so its gradient collects both before it
 * is propagated into B_{t-1} and x_{t-1}; at t = 0 the previous input is the carry.
 * Cotangents: dy (b, L, H, P) and dh_final (b, H, N, P) (NULL: zero).  Gradients are ADDED to
 * the outputs (the caller zeroes them): dx (b,L,H,P), ddt / dA / dlam (b,L,H), dB / dC
 * (b,L,G,R,N) and dtheta (b,L,G,N/2) summed over the heads of a group, dbias_B / dbias_C
 * (H,R,N), dW_x / dW_o (H,R,P) and dD (H) summed over batch and tokens, and the initial
 * state's dh0 (b,H,N,P), dcarry_B (b,H,R,N), dcarry_x (b,H,P).  Pairs run one after another
 * (the per-group and per-head sums are shared).  Returns 0, -1 on bad dimensions, -2 on OOM.
 */
typedef struct {
  double *dx, *ddt, *dA, *dlam, *dB, *dC, *dtheta, *dbias_B, *dbias_C, *dW_x, *dW_o, *dD, *dh0, *dcarry_B,
      *dcarry_x;
} m3o_grads;

static int bwd_one(const m3o_dims* d, int64_t bi, int32_t hi, const double* x, const double* dt,
                   const double* A, const double* lam, const double* B, const double* C,
                   const double* theta, const double* bias_B, const double* bias_C, const double* W_x,
                   const double* W_o, const double* D, const double* h_init, const double* cB_init,
                   const double* cx_init, const double* dy, const double* dh_final, const m3o_grads* gr) {
  const int64_t L = d->L;
  const int32_t H = d->H, P = d->P, N = d->N, R = d->R, G = d->G, K = N / 2;
  const int32_t g = hi / (H / G);
  const int64_t pair = bi * H + hi;
  const size_t NP = (size_t)N * P;
  double* hs = (double*)malloc(sizeof(double) * (size_t)(L + 1) * NP);
  double* u = (double*)malloc(sizeof(double) * NP);
  double* up = (double*)malloc(sizeof(double) * NP);
  double* gN = (double*)malloc(sizeof(double) * NP);    /* dL/dh_t */
  double* duN = (double*)malloc(sizeof(double) * NP);   /* beta'_{t+1} dz_{t+1}: u_t's share from step t+1 */
  double* du = (double*)malloc(sizeof(double) * NP);
  double* dz = (double*)malloc(sizeof(double) * NP);
  double* Bb = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* Bbp = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* Cb = (double*)malloc(sizeof(double) * (size_t)R * N);
  double* X = (double*)malloc(sizeof(double) * (size_t)R * P);
  double* Xp = (double*)malloc(sizeof(double) * (size_t)R * P);
  double* dYr = (double*)malloc(sizeof(double) * (size_t)P);
  double* dphi = (double*)malloc(sizeof(double) * (size_t)K);
  int rc = 0;
  if (!hs || !u || !up || !gN || !duN || !du || !dz || !Bb || !Bbp || !Cb || !X || !Xp || !dYr || !dphi) {
    rc = -2;
    goto done;
  }

  /* operands of token t (t = -1: the carry) */
#define BIASB(r, n) (bias_B ? bias_B[((int64_t)hi * R + (r)) * N + (n)] : 0.0)
#define BIASC(r, n) (bias_C ? bias_C[((int64_t)hi * R + (r)) * N + (n)] : 0.0)
#define WX(r, p) (W_x ? W_x[((int64_t)hi * R + (r)) * P + (p)] : 1.0)
#define WO(r, p) (W_o ? W_o[((int64_t)hi * R + (r)) * P + (p)] : 1.0)
#define TOK(t) (bi * L + (t))
  const double* cB0 = cB_init + pair * (int64_t)R * N;
  const double* cx0 = cx_init + pair * (int64_t)P;

  /* forward, keeping h_{t} in hs[t + 1] (hs[0] = h_{-1}) */
  memcpy(hs, h_init + pair * (int64_t)NP, sizeof(double) * NP);
  for (int64_t t = 0; t < L; ++t) {
    const int64_t tok = TOK(t);
    const double delta = dt[tok * H + hi], a = A[tok * H + hi], lm = lam[tok * H + hi];
    const double alpha = exp(delta * a), bprime = (1.0 - lm) * delta, gamma = lm * delta;
    const double* xt = x + (tok * H + hi) * (int64_t)P;
    const double* Bt = B + ((tok * G + g) * (int64_t)R) * N;
    const double* xq = t > 0 ? x + ((tok - 1) * H + hi) * (int64_t)P : cx0;
    const double* Bq = t > 0 ? B + (((tok - 1) * G + g) * (int64_t)R) * N : cB0;
    const double* th = theta + (tok * G + g) * (int64_t)K;
    for (int32_t n = 0; n < N; ++n)
      for (int32_t p = 0; p < P; ++p) {
        double s = 0.0, sp = 0.0;
        for (int32_t r = 0; r < R; ++r) {
          s += (Bt[r * N + n] + BIASB(r, n)) * WX(r, p) * xt[p];
          sp += (Bq[r * N + n] + BIASB(r, n)) * WX(r, p) * xq[p];
        }
        u[(size_t)n * P + p] = s;
        up[(size_t)n * P + p] = sp;
      }
    const double* hp = hs + (size_t)t * NP;
    double* hn = hs + (size_t)(t + 1) * NP;
    for (int32_t k = 0; k < K; ++k) {
      const double phi = d->angle_direct ? th[k] : delta * th[k];
      const double c = cos(phi), s = sin(phi);
      for (int32_t p = 0; p < P; ++p) {
        const double z0 = hp[(size_t)(2 * k) * P + p] + bprime * up[(size_t)(2 * k) * P + p];
        const double z1 = hp[(size_t)(2 * k + 1) * P + p] + bprime * up[(size_t)(2 * k + 1) * P + p];
        hn[(size_t)(2 * k) * P + p] = alpha * (c * z0 - s * z1) + gamma * u[(size_t)(2 * k) * P + p];
        hn[(size_t)(2 * k + 1) * P + p] = alpha * (s * z0 + c * z1) + gamma * u[(size_t)(2 * k + 1) * P + p];
      }
    }
  }

  /* reverse */
  for (size_t i = 0; i < NP; ++i) {
    gN[i] = dh_final ? dh_final[pair * (int64_t)NP + i] : 0.0;
    duN[i] = 0.0;
  }
  for (int64_t t = L - 1; t >= 0; --t) {
    const int64_t tok = TOK(t);
    const double delta = dt[tok * H + hi], a = A[tok * H + hi], lm = lam[tok * H + hi];
    const double alpha = exp(delta * a), bprime = (1.0 - lm) * delta, gamma = lm * delta;
    const double* xt = x + (tok * H + hi) * (int64_t)P;
    const double* Bt = B + ((tok * G + g) * (int64_t)R) * N;
    const double* Ct = C + ((tok * G + g) * (int64_t)R) * N;
    const double* xq = t > 0 ? x + ((tok - 1) * H + hi) * (int64_t)P : cx0;
    const double* Bq = t > 0 ? B + (((tok - 1) * G + g) * (int64_t)R) * N : cB0;
    const double* th = theta + (tok * G + g) * (int64_t)K;
    const double* dyt = dy ? dy + (tok * H + hi) * (int64_t)P : NULL;
    const double* ht = hs + (size_t)(t + 1) * NP;
    const double* hp = hs + (size_t)t * NP;
    for (int32_t r = 0; r < R; ++r) {
      for (int32_t n = 0; n < N; ++n) {
        Bb[r * N + n] = Bt[r * N + n] + BIASB(r, n);
        Bbp[r * N + n] = Bq[r * N + n] + BIASB(r, n);
        Cb[r * N + n] = Ct[r * N + n] + BIASC(r, n);
      }
      for (int32_t p = 0; p < P; ++p) {
        X[r * P + p] = WX(r, p) * xt[p];
        Xp[r * P + p] = WX(r, p) * xq[p];
      }
    }
    for (int32_t n = 0; n < N; ++n)
      for (int32_t p = 0; p < P; ++p) {
        double s = 0.0, sp = 0.0;
        for (int32_t r = 0; r < R; ++r) {
          s += Bb[r * N + n] * X[r * P + p];
          sp += Bbp[r * N + n] * Xp[r * P + p];
        }
        u[(size_t)n * P + p] = s;
        up[(size_t)n * P + p] = sp;
      }
    /* readout y_t = sum_r W_o_r * (Cb_r^T h_t) + D x_t */
    if (dyt) {
      for (int32_t r = 0; r < R; ++r) {
        for (int32_t p = 0; p < P; ++p) {
          dYr[p] = WO(r, p) * dyt[p];
          double Y = 0.0;
          for (int32_t n = 0; n < N; ++n) Y += Cb[r * N + n] * ht[(size_t)n * P + p];
          if (W_o) gr->dW_o[((int64_t)hi * R + r) * P + p] += dyt[p] * Y;
        }
        for (int32_t n = 0; n < N; ++n) {
          double dcb = 0.0;
          for (int32_t p = 0; p < P; ++p) {
            dcb += ht[(size_t)n * P + p] * dYr[p];
            gN[(size_t)n * P + p] += Cb[r * N + n] * dYr[p];
          }
          gr->dC[((tok * G + g) * (int64_t)R + r) * N + n] += dcb;
          if (bias_C) gr->dbias_C[((int64_t)hi * R + r) * N + n] += dcb;
        }
      }
      if (D) {
        double sd = 0.0;
        for (int32_t p = 0; p < P; ++p) {
          sd += dyt[p] * xt[p];
          gr->dx[(tok * H + hi) * (int64_t)P + p] += D[hi] * dyt[p];
        }
        gr->dD[hi] += sd;
      }
    }
    /* step h_t = alpha Rot(phi) z + gamma u_t, z = h_{t-1} + beta' u_{t-1} */
    double dalpha = 0.0, dgamma = 0.0, dbp = 0.0;
    for (int32_t k = 0; k < K; ++k) {
      const double phi = d->angle_direct ? th[k] : delta * th[k];
      const double c = cos(phi), s = sin(phi);
      double dph = 0.0;
      for (int32_t p = 0; p < P; ++p) {
        const size_t i0 = (size_t)(2 * k) * P + p, i1 = (size_t)(2 * k + 1) * P + p;
        const double z0 = hp[i0] + bprime * up[i0], z1 = hp[i1] + bprime * up[i1];
        const double m0 = c * z0 - s * z1, m1 = s * z0 + c * z1;
        dalpha += gN[i0] * m0 + gN[i1] * m1;
        dgamma += gN[i0] * u[i0] + gN[i1] * u[i1];
        du[i0] = gamma * gN[i0] + duN[i0];
        du[i1] = gamma * gN[i1] + duN[i1];
        const double dm0 = alpha * gN[i0], dm1 = alpha * gN[i1];
        dz[i0] = c * dm0 + s * dm1;   /* Rot^T dm */
        dz[i1] = -s * dm0 + c * dm1;
        dph += dm0 * (-s * z0 - c * z1) + dm1 * (c * z0 - s * z1);
        dbp += dz[i0] * up[i0] + dz[i1] * up[i1];
      }
      dphi[k] = dph;
    }
    for (size_t i = 0; i < NP; ++i) {
      duN[i] = bprime * dz[i]; /* u_{t-1}'s share from this step */
      gN[i] = dz[i];           /* dL/dh_{t-1} */
    }
    /* u_t = sum_r Bb_r X_r^T */
    for (int32_t r = 0; r < R; ++r) {
      for (int32_t n = 0; n < N; ++n) {
        double db = 0.0;
        for (int32_t p = 0; p < P; ++p) db += du[(size_t)n * P + p] * X[r * P + p];
        gr->dB[((tok * G + g) * (int64_t)R + r) * N + n] += db;
        if (bias_B) gr->dbias_B[((int64_t)hi * R + r) * N + n] += db;
      }
      for (int32_t p = 0; p < P; ++p) {
        double dX = 0.0;
        for (int32_t n = 0; n < N; ++n) dX += du[(size_t)n * P + p] * Bb[r * N + n];
        if (W_x) gr->dW_x[((int64_t)hi * R + r) * P + p] += dX * xt[p];
        gr->dx[(tok * H + hi) * (int64_t)P + p] += WX(r, p) * dX;
      }
    }
    /* scalars of the step */
    double dth_dt = 0.0;
    for (int32_t k = 0; k < K; ++k) {
      if (!d->angle_direct) dth_dt += dphi[k] * th[k];
      gr->dtheta[(tok * G + g) * (int64_t)K + k] += dphi[k] * (d->angle_direct ? 1.0 : delta);
    }
    gr->ddt[tok * H + hi] += dalpha * alpha * a + dgamma * lm + dbp * (1.0 - lm) + dth_dt;
    gr->dA[tok * H + hi] += dalpha * alpha * delta;
    gr->dlam[tok * H + hi] += (dgamma - dbp) * delta;
  }
  /* the initial state: h_{-1} and the carry, through u_{-1} = sum_r (carry_B_r + bias_B_r)(W_x_r * carry_x)^T */
  for (size_t i = 0; i < NP; ++i) gr->dh0[pair * (int64_t)NP + i] += gN[i];
  for (int32_t r = 0; r < R; ++r) {
    for (int32_t n = 0; n < N; ++n) {
      double db = 0.0;
      for (int32_t p = 0; p < P; ++p) db += duN[(size_t)n * P + p] * WX(r, p) * cx0[p];
      gr->dcarry_B[(pair * R + r) * (int64_t)N + n] += db;
      if (bias_B) gr->dbias_B[((int64_t)hi * R + r) * N + n] += db;
    }
    for (int32_t p = 0; p < P; ++p) {
      double dX = 0.0;
      for (int32_t n = 0; n < N; ++n) dX += duN[(size_t)n * P + p] * (cB0[r * N + n] + BIASB(r, n));
      if (W_x) gr->dW_x[((int64_t)hi * R + r) * P + p] += dX * cx0[p];
      gr->dcarry_x[pair * (int64_t)P + p] += WX(r, p) * dX;
    }
  }
#undef BIASB
#undef BIASC
#undef WX
#undef WO
#undef TOK
done:
  free(hs); free(u); free(up); free(gN); free(duN); free(du); free(dz);
  free(Bb); free(Bbp); free(Cb); free(X); free(Xp); free(dYr); free(dphi);
  return rc;
}

int m3o_scan_bwd(const m3o_dims* d, const double* x, const double* dt, const double* A, const double* lam,
                 const double* B, const double* C, const double* theta, const double* bias_B,
                 const double* bias_C, const double* W_x, const double* W_o, const double* D,
                 const double* h0, const double* carry_B0, const double* carry_x0, const double* dy,
                 const double* dh_final, const m3o_grads* gr) {
  if (!d || d->b < 0 || d->L < 0 || d->H <= 0 || d->P <= 0 || d->N <= 0 || d->R <= 0 ||
      d->G <= 0 || (d->N % 2) != 0 || (d->H % d->G) != 0 || !gr)
    return -1;
  for (int64_t i = 0; i < d->b * d->H; ++i) {
    const int rc = bwd_one(d, i / d->H, (int32_t)(i % d->H), x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x,
                           W_o, D, h0, carry_B0, carry_x0, dy, dh_final, gr);
    if (rc != 0) return rc;
  }
  return 0;
}

int m3o_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
