/*
 * Gated delta-rule oracle: plain, slow, float64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (one independent recurrence per batch b and head h):
 *
 *   b_t = sqrt(beta_k_t) (.) k_t                     erase key ("k tilde")
 *   a_t = s_t (.) b_t   (s_t = 1 unless given)       write-side key
 *   w_t = beta_v_t (.) v_t  if beta_v is given,  else  sqrt(beta_k_t) (.) v_t
 *   D_t = Diag(alpha_t)                              (alpha = 1 if absent)
 *   S_t = (I - a_t b_t^T) D_t S_{t-1} + a_t w_t^T    S in R^{dk x dv}
 *   o_t = S_t^T q_t
 *
 * Passages followed:
 *   - DeltaNet page (robocikowo.com, "DeltaNet"), numbered steps 3-6: read the
 *     current mapping with the key, form the error against v scaled by beta,
 *     write the rank-1 correction, read the output with the query from the
 *     UPDATED state.  That page stores the state as dv x dk; this file keeps
 *     the transpose, dk x dv, so the read is S^T k and the output S^T q.
 *   - FG2-GDN page (gist.science), section 2 "Kerninnovation": the update
 *     equation S_t = (I - k~ k~^T) Diag(alpha_t) S_{t-1} + k~ v~^T with
 *     k~ = sqrt(beta) (.) k and v~ = sqrt(beta) (.) v; decay is applied first
 *     and the erase acts on the decayed state.
 *   - Same page, section 2 "Erweiterung: FG2-GDN+": separate erase strength
 *     beta^k and write strength beta^v; the write vector is beta^v (.) v.
 *   - Same page, section 1: scalar forget factor (GDN) or channel-wise
 *     alpha_t in R^{dk} (KDA), applied on the key dimension.
 *   - OSDN summary (turingwire.com), "Method": the diagonal preconditioner is
 *     a per-feature scaling of the write-side key, i.e. a_t = s_t (.) b_t.
 *
 * Two evaluations are provided:
 *   dro_sequential  - the recurrence above, one token at a time.  This is the
 *                     definition and the parity reference.
 *   dro_chunkwise   - the same result through the chunkwise WY/UT
 *                     (Householder-product) factorisation, in float64, used
 *                     to check that factorisation and to expose its
 *                     per-chunk intermediates.  It must agree with
 *                     dro_sequential to rounding.
 *
 * Layouts (row-major, all float64):
 *   q, k, s_scale : [B, T, H, dk]      v : [B, T, H, dv]      o : [B, T, H, dv]
 *   alpha, beta_k : [B, T, H] (scalar mode) or [B, T, H, dk] (channel mode)
 *   beta_v        : [B, T, H] (scalar mode) or [B, T, H, dv] (channel mode)
 *   S0, ST        : [B, H, dk, dv]
 * Mode codes: 0 = absent, 1 = scalar per (b, t, h), 2 = channel vector.
 * Return value: 0 on success, negative on an invalid argument.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define DRO_ABSENT 0
#define DRO_SCALAR 1
#define DRO_CHANNEL 2

typedef struct {
  int B, T, H, dk, dv;
  const double *q, *k, *v;
  const double *alpha;  int alpha_mode;
  const double *beta_k; int beta_k_mode;
  const double *beta_v; int beta_v_mode;
  const double *s_scale;
  const double *S0;
  double *o, *ST;
} dro_args;

/* value of a per-token gate at (token-head index th, channel i) */
static double gate(const double *g, int mode, size_t th, int width, int i) {
  if (mode == DRO_ABSENT) return 1.0;
  if (mode == DRO_SCALAR) return g[th];
  return g[th * (size_t)width + (size_t)i];
}

static int check_args(const dro_args *a) {
  if (a->B < 0 || a->T < 0 || a->H < 0 || a->dk <= 0 || a->dv <= 0) return -1;
  if (!a->q || !a->k || !a->v || !a->o || !a->beta_k) return -2;
  if (a->alpha_mode < 0 || a->alpha_mode > 2) return -3;
  if (a->alpha_mode != DRO_ABSENT && !a->alpha) return -3;
  if (a->beta_k_mode != DRO_SCALAR && a->beta_k_mode != DRO_CHANNEL) return -4;
  if (a->beta_v_mode < 0 || a->beta_v_mode > 2) return -5;
  if (a->beta_v_mode != DRO_ABSENT && !a->beta_v) return -5;
  /* sqrt(beta) (.) v with beta in R^{dk} only type-checks when dk == dv */
  if (a->beta_v_mode == DRO_ABSENT && a->beta_k_mode == DRO_CHANNEL && a->dk != a->dv) return -6;
  return 0;
}

/* scaled keys and write vector of one token (the input scaling) */
static void token_vectors(const dro_args *a, size_t th, double *bv, double *av, double *wv) {
  const int dk = a->dk, dv = a->dv;
  for (int i = 0; i < dk; ++i) {
    const double bk = sqrt(gate(a->beta_k, a->beta_k_mode, th, dk, i)) * a->k[th * dk + i];
    bv[i] = bk;
    av[i] = a->s_scale ? a->s_scale[th * dk + i] * bk : bk;
  }
  for (int j = 0; j < dv; ++j) {
    const double vj = a->v[th * dv + j];
    if (a->beta_v_mode != DRO_ABSENT)
      wv[j] = gate(a->beta_v, a->beta_v_mode, th, dv, j) * vj;
    else
      wv[j] = sqrt(gate(a->beta_k, a->beta_k_mode, th, dk, j)) * vj;
  }
}

/* ---------------------------------------------------------------------- */
/* The recurrence, token by token.                                         */
/* ---------------------------------------------------------------------- */
static void sequential_head(const dro_args *a, int b, int h) {
  const int T = a->T, H = a->H, dk = a->dk, dv = a->dv;
  double *S = (double *)malloc(sizeof(double) * dk * dv);
  double *bv = (double *)malloc(sizeof(double) * dk);
  double *av = (double *)malloc(sizeof(double) * dk);
  double *wv = (double *)malloc(sizeof(double) * dv);
  double *u = (double *)malloc(sizeof(double) * dv);
  const size_t sh = ((size_t)b * H + h) * dk * dv;
  if (a->S0) memcpy(S, a->S0 + sh, sizeof(double) * dk * dv);
  else memset(S, 0, sizeof(double) * dk * dv);

  for (int t = 0; t < T; ++t) {
    const size_t th = ((size_t)b * T + t) * H + h;
    token_vectors(a, th, bv, av, wv);
    /* decay first: S <- Diag(alpha_t) S */
    for (int i = 0; i < dk; ++i) {
      const double al = gate(a->alpha, a->alpha_mode, th, dk, i);
      for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;
    }
    /* read with the erase key and form the error: u = w - (D S)^T b */
    for (int j = 0; j < dv; ++j) {
      double r = 0.0;
      for (int i = 0; i < dk; ++i) r += S[i * dv + j] * bv[i];
      u[j] = wv[j] - r;
    }
    /* rank-1 write: S <- D S + a u^T  ==  (I - a b^T) D S + a w^T */
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) S[i * dv + j] += av[i] * u[j];
    /* output from the updated state: o_t = S_t^T q_t */
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * a->q[th * dk + i];
      a->o[th * dv + j] = acc;
    }
  }
  if (a->ST) memcpy(a->ST + sh, S, sizeof(double) * dk * dv);
  free(S); free(bv); free(av); free(wv); free(u);
}

/* ---------------------------------------------------------------------- */
/* The chunkwise WY/UT evaluation (DeltaNet page, step 7 and the remark on */
/* Householder-product representations; FG2-GDN page, section 2, the note  */
/* that the symmetric sqrt(beta) scaling keeps the rank-1 Householder      */
/* structure that the chunkwise WY form needs).                            */
/*                                                                         */
/* For a chunk of L tokens starting from state S (local index r = 0..L-1): */
/*   g_r   = sum_{j<=r} log alpha_j          (per key channel)             */
/*   Bh_r  = exp(g_r) (.) b_r    Ac_r = a_r (.) exp(-g_r)                  */
/*   Qh_r  = exp(g_r) (.) q_r    Kd_r = a_r (.) exp(g_{L-1} - g_r)         */
/*   A     = strictly lower part of Bh Ac^T,   T = (I + A)^{-1}            */
/*   W     = T Bh,   U0 = T Wr   (Wr = rows w_r)                           */
/*   U     = U0 - W S                        (row r of U is u_r)           */
/*   P     = lower part, diagonal included, of Qh Ac^T                     */
/*   O     = Qh S + P U                       (row r is o_r)               */
/*   S    <- Diag(exp(g_{L-1})) S + Kd^T U                                 */
/* ---------------------------------------------------------------------- */
static void chunkwise_head(const dro_args *a, int b, int h, int C) {
  const int T = a->T, H = a->H, dk = a->dk, dv = a->dv;
  double *S = (double *)malloc(sizeof(double) * dk * dv);
  double *g = (double *)malloc(sizeof(double) * C * dk);
  double *Bh = (double *)malloc(sizeof(double) * C * dk);
  double *Ac = (double *)malloc(sizeof(double) * C * dk);
  double *Qh = (double *)malloc(sizeof(double) * C * dk);
  double *Kd = (double *)malloc(sizeof(double) * C * dk);
  double *Wr = (double *)malloc(sizeof(double) * C * dv);
  double *A = (double *)malloc(sizeof(double) * C * C);
  double *Ti = (double *)malloc(sizeof(double) * C * C);
  double *P = (double *)malloc(sizeof(double) * C * C);
  double *W = (double *)malloc(sizeof(double) * C * dk);
  double *U = (double *)malloc(sizeof(double) * C * dv);
  double *Sn = (double *)malloc(sizeof(double) * dk * dv);
  double *bv = (double *)malloc(sizeof(double) * dk);
  double *av = (double *)malloc(sizeof(double) * dk);
  const size_t sh = ((size_t)b * H + h) * dk * dv;
  if (a->S0) memcpy(S, a->S0 + sh, sizeof(double) * dk * dv);
  else memset(S, 0, sizeof(double) * dk * dv);

  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = (T - t0 < C) ? (T - t0) : C;
    /* cumulative log-gate within the chunk */
    for (int r = 0; r < L; ++r) {
      const size_t th = ((size_t)b * T + t0 + r) * H + h;
      for (int i = 0; i < dk; ++i) {
        double lg = log(gate(a->alpha, a->alpha_mode, th, dk, i));
        g[r * dk + i] = (r == 0 ? 0.0 : g[(r - 1) * dk + i]) + lg;
      }
    }
    /* scaled operands */
    for (int r = 0; r < L; ++r) {
      const size_t th = ((size_t)b * T + t0 + r) * H + h;
      token_vectors(a, th, bv, av, Wr + (size_t)r * dv);
      for (int i = 0; i < dk; ++i) {
        double gr = g[r * dk + i], gl = g[(L - 1) * dk + i];
        Bh[r * dk + i] = exp(gr) * bv[i];
        Ac[r * dk + i] = av[i] * exp(-gr);
        Qh[r * dk + i] = exp(gr) * a->q[th * dk + i];
        Kd[r * dk + i] = av[i] * exp(gl - gr);
      }
    }
    /* A (strictly lower) and P (lower, diagonal included) */
    for (int r = 0; r < L; ++r)
      for (int i = 0; i < L; ++i) {
        double sa = 0.0, sp = 0.0;
        for (int c = 0; c < dk; ++c) {
          sa += Bh[r * dk + c] * Ac[i * dk + c];
          sp += Qh[r * dk + c] * Ac[i * dk + c];
        }
        A[r * C + i] = (i < r) ? sa : 0.0;
        P[r * C + i] = (i <= r) ? sp : 0.0;
      }
    /* T = (I + A)^{-1} by forward substitution, one column at a time */
    for (int j = 0; j < L; ++j)
      for (int r = 0; r < L; ++r) {
        if (r < j) { Ti[r * C + j] = 0.0; continue; }
        double x = (r == j) ? 1.0 : 0.0;
        for (int m = j; m < r; ++m) x -= A[r * C + m] * Ti[m * C + j];
        Ti[r * C + j] = x;
      }
    /* W = T Bh,  U = T Wr - W S */
    for (int r = 0; r < L; ++r) {
      for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int m = 0; m < L; ++m) acc += Ti[r * C + m] * Bh[m * dk + c];
        W[r * dk + c] = acc;
      }
      for (int j = 0; j < dv; ++j) {
        double u0 = 0.0, ws = 0.0;
        for (int m = 0; m < L; ++m) u0 += Ti[r * C + m] * Wr[m * dv + j];
        for (int c = 0; c < dk; ++c) ws += W[r * dk + c] * S[c * dv + j];
        U[r * dv + j] = u0 - ws;
      }
    }
    /* O = Qh S + P U */
    for (int r = 0; r < L; ++r) {
      const size_t th = ((size_t)b * T + t0 + r) * H + h;
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += Qh[r * dk + c] * S[c * dv + j];
        for (int m = 0; m < L; ++m) acc += P[r * C + m] * U[m * dv + j];
        a->o[th * dv + j] = acc;
      }
    }
    /* S <- Diag(exp(g_{L-1})) S + Kd^T U */
    for (int c = 0; c < dk; ++c)
      for (int j = 0; j < dv; ++j) {
        double acc = exp(g[(L - 1) * dk + c]) * S[c * dv + j];
        for (int m = 0; m < L; ++m) acc += Kd[m * dk + c] * U[m * dv + j];
        Sn[c * dv + j] = acc;
      }
    memcpy(S, Sn, sizeof(double) * dk * dv);
  }
  if (a->ST) memcpy(a->ST + sh, S, sizeof(double) * dk * dv);
  free(S); free(g); free(Bh); free(Ac); free(Qh); free(Kd); free(Wr);
  free(A); free(Ti); free(P); free(W); free(U); free(Sn); free(bv); free(av);
}

static int run_all(const dro_args *a, int chunk, int nthreads) {
  int rc = check_args(a);
  if (rc) return rc;
  const long nbh = (long)a->B * a->H;
#ifdef _OPENMP
  if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
  for (long bh = 0; bh < nbh; ++bh) {
    int b = (int)(bh / a->H), h = (int)(bh % a->H);
    if (chunk <= 0) sequential_head(a, b, h);
    else chunkwise_head(a, b, h, chunk);
  }
  (void)nthreads;
  return 0;
}

int dro_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int dro_sequential(int B, int T, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *alpha, int alpha_mode,
                   const double *beta_k, int beta_k_mode,
                   const double *beta_v, int beta_v_mode,
                   const double *s_scale, const double *S0,
                   double *o, double *ST, int nthreads) {
  dro_args a = {B, T, H, dk, dv, q, k, v, alpha, alpha_mode, beta_k, beta_k_mode,
                beta_v, beta_v_mode, s_scale, S0, o, ST};
  return run_all(&a, 0, nthreads);
}

int dro_chunkwise(int B, int T, int H, int dk, int dv, int chunk,
                  const double *q, const double *k, const double *v,
                  const double *alpha, int alpha_mode,
                  const double *beta_k, int beta_k_mode,
                  const double *beta_v, int beta_v_mode,
                  const double *s_scale, const double *S0,
                  double *o, double *ST, int nthreads) {
  if (chunk <= 0) return -7;
  dro_args a = {B, T, H, dk, dv, q, k, v, alpha, alpha_mode, beta_k, beta_k_mode,
                beta_v, beta_v_mode, s_scale, S0, o, ST};
  return run_all(&a, chunk, nthreads);
}
