/*
 * Plain fp64 CPU oracle for the Mamba-2 mixer core (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header or constant with the CUDA
 * library in mamba_ssd_scan_mixer_b200/; it is written to be read against the
 * sources, not to be fast.
 *
 * What it computes, and where each step comes from:
 *  - causal depthwise conv1d of width d_conv over the x|B|C channels, with
 *    bias, followed by SiLU: "Zamba2 hybrid architecture in Transformers"
 *    (qwbw.cn), section 三 (Mamba2 Mixer), step 2; bias per section 五
 *    (use_conv_bias=True).  Tap k of channel c multiplies the input k-(d_conv-1)
 *    steps before the current token (cross-correlation with left padding), and
 *    the d_conv-1 inputs before the first token come from the carried conv
 *    state (zeros for a fresh sequence).
 *  - dt = softplus(dt_raw + dt_bias), and the selective SSM recurrence
 *    h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,  y_t = C_t h_t + D_h x_t:
 *    the Mamba-2 (state-space duality) layer named on the state-spaces/mamba
 *    repository page (opendeer.net), "About the project".  Section 三 of the
 *    qwbw.cn page gives its two evaluation orders: the chunked scan for
 *    prefill and the single-token state update for decode.
 *  - gated group RMSNorm y * silu(z), eps 1e-5, groups of d_inner/ngroups
 *    channels, with the norm_before_gate switch: qwbw.cn page, section 三
 *    step 4 and section 五 (rms_norm_eps).
 *  - the conv and SSM states carried between calls: qwbw.cn page, section 三
 *    (the cache holds the conv and recurrent state of every Mamba layer).
 *
 * Three evaluation orders of the scan are provided so that each can be
 * checked against the others: token-by-token (the definition), the
 * materialised quadratic semiseparable form (brute force), and the chunked
 * form for any chunk length.
 *
 * Layouts (all row-major, double):
 *   xBC  [L, conv_dim]   channels: x (H*P, head-major) | B (G*N) | C (G*N)
 *   x    [L, H, P] view of xBC, B/C [L, G, N] views, head h uses group
 *        h / (H/G)
 *   dt   [L, H]
 *   state h[H, P, N]  (d_state contiguous)
 *   conv state [conv_dim, d_conv], oldest input first.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* elementwise functions                                              */
/* ------------------------------------------------------------------ */

double m2o_silu(double s) { return s / (1.0 + exp(-s)); }

/* softplus(s) = log(1 + e^s), evaluated without overflow; no threshold. */
double m2o_softplus(double s) { return fmax(s, 0.0) + log1p(exp(-fabs(s))); }

/* ------------------------------------------------------------------ */
/* a tiny parallel-for over independent items (batch rows, heads)     */
/* ------------------------------------------------------------------ */

typedef void (*m2o_item_fn)(void *ctx, int64_t item);

typedef struct {
  m2o_item_fn fn;
  void *ctx;
  int64_t begin, end;
} m2o_range;

static void *m2o_range_worker(void *arg) {
  m2o_range *r = (m2o_range *)arg;
  for (int64_t i = r->begin; i < r->end; ++i) r->fn(r->ctx, i);
  return NULL;
}

static void m2o_parallel_for(int64_t n, int nthreads, m2o_item_fn fn, void *ctx) {
  if (nthreads <= 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(ctx, i);
    return;
  }
  if (nthreads > n) nthreads = (int)n;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  m2o_range *rg = (m2o_range *)malloc(sizeof(m2o_range) * (size_t)nthreads);
  int started = 0;
  for (int i = 0; i < nthreads; ++i) {
    rg[i].fn = fn;
    rg[i].ctx = ctx;
    rg[i].begin = n * i / nthreads;
    rg[i].end = n * (i + 1) / nthreads;
    if (pthread_create(&th[i], NULL, m2o_range_worker, &rg[i]) == 0) {
      started = i + 1;
    } else {
      m2o_range_worker(&rg[i]); /* could not start a thread: run it here */
      th[i] = (pthread_t)0;
    }
  }
  for (int i = 0; i < started; ++i)
    if (th[i]) pthread_join(th[i], NULL);
  free(th);
  free(rg);
}

/* ------------------------------------------------------------------ */
/* conv1d + SiLU over one sequence                                    */
/* ------------------------------------------------------------------ */

/* Input value v[tau, c]: tau >= 0 is token tau of xBC; tau in [-K, -1] is
 * entry K+tau of the carried conv state (0 when there is none). */
static double conv_input(const double *xBC, int64_t conv_dim, const double *state_in,
                         int64_t K, int64_t tau, int64_t c) {
  if (tau >= 0) return xBC[tau * conv_dim + c];
  if (state_in == NULL) return 0.0;
  return state_in[c * K + (K + tau)];
}

void m2o_conv_silu(int64_t L, int64_t conv_dim, int64_t K, const double *xBC,
                   const double *state_in, const double *w, const double *b, double *u,
                   double *state_out) {
  for (int64_t t = 0; t < L; ++t)
    for (int64_t c = 0; c < conv_dim; ++c) {
      double acc = b[c];
      for (int64_t k = 0; k < K; ++k)
        acc += w[c * K + k] * conv_input(xBC, conv_dim, state_in, K, t - (K - 1) + k, c);
      u[t * conv_dim + c] = m2o_silu(acc);
    }
  if (state_out != NULL) {
    /* the last K raw inputs, oldest first; built aside so that state_out may
     * be the same buffer as state_in */
    double *new_state = (double *)malloc(sizeof(double) * (size_t)(conv_dim * K));
    for (int64_t c = 0; c < conv_dim; ++c)
      for (int64_t k = 0; k < K; ++k)
        new_state[c * K + k] = conv_input(xBC, conv_dim, state_in, K, L - K + k, c);
    memcpy(state_out, new_state, sizeof(double) * (size_t)(conv_dim * K));
    free(new_state);
  }
}

/* ------------------------------------------------------------------ */
/* the scan: three evaluation orders                                  */
/* ------------------------------------------------------------------ */

/* Common argument block for one sequence.  x, B, C are strided views:
 * x[t, h, p] = x[t*ldx + h*P + p], B[t, g, n] = B[t*ldbc + g*N + n], same
 * for C; y[t, h, p] = y[t*ldy + h*P + p]; dt[t, h] = dt[t*H + h]. */
typedef struct {
  int64_t L, H, P, N, G;
  const double *x;
  int64_t ldx;
  const double *B;
  const double *C;
  int64_t ldbc;
  const double *dt;
  const double *A;
  const double *D;
  const double *h0; /* [H, P, N] or NULL (zeros) */
  double *y;
  int64_t ldy;
  double *hL; /* [H, P, N] or NULL */
  int64_t chunk;
} m2o_scan_args;

static int64_t group_of(const m2o_scan_args *a, int64_t h) { return h / (a->H / a->G); }

/* Token-by-token recurrence for head h: the definition. */
static void scan_sequential_head(void *ctx, int64_t h) {
  const m2o_scan_args *a = (const m2o_scan_args *)ctx;
  const int64_t P = a->P, N = a->N, g = group_of(a, h);
  double *s = (double *)calloc((size_t)(P * N), sizeof(double));
  if (a->h0 != NULL) memcpy(s, a->h0 + h * P * N, sizeof(double) * (size_t)(P * N));
  for (int64_t t = 0; t < a->L; ++t) {
    const double dt = a->dt[t * a->H + h];
    const double decay = exp(dt * a->A[h]);
    const double *xt = a->x + t * a->ldx + h * P;
    const double *Bt = a->B + t * a->ldbc + g * N;
    const double *Ct = a->C + t * a->ldbc + g * N;
    for (int64_t p = 0; p < P; ++p) {
      double yp = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double *spn = &s[p * N + n];
        *spn = decay * (*spn) + dt * xt[p] * Bt[n];
        yp += (*spn) * Ct[n];
      }
      a->y[t * a->ldy + h * P + p] = yp + a->D[h] * xt[p];
    }
  }
  if (a->hL != NULL) memcpy(a->hL + h * P * N, s, sizeof(double) * (size_t)(P * N));
  free(s);
}

/* Sum of dt_r * A_h for r in [r0, r1] (inclusive), written out as a plain sum. */
static double seg_sum(const m2o_scan_args *a, int64_t h, int64_t r0, int64_t r1) {
  double acc = 0.0;
  for (int64_t r = r0; r <= r1; ++r) acc += a->dt[r * a->H + h] * a->A[h];
  return acc;
}

/* Materialised semiseparable matrix for head h:
 *   M[t, s] = (C_t . B_s) * exp(sum_{r=s+1..t} dt_r A) * dt_s   for s <= t,
 *   y = M x + exp(sum_{r=0..t} dt_r A) (C_t . h0[p, :]) + D x,
 *   hL = exp(sum_{r=0..L-1} dt_r A) h0 + sum_s exp(sum_{r=s+1..L-1} dt_r A) dt_s x_s B_s^T.
 * O(L^3) per head: for tiny sequences only. */
static void scan_quadratic_head(void *ctx, int64_t h) {
  const m2o_scan_args *a = (const m2o_scan_args *)ctx;
  const int64_t L = a->L, P = a->P, N = a->N, g = group_of(a, h);
  double *M = (double *)calloc((size_t)(L * L), sizeof(double));
  for (int64_t t = 0; t < L; ++t) {
    const double *Ct = a->C + t * a->ldbc + g * N;
    for (int64_t s = 0; s <= t; ++s) {
      const double *Bs = a->B + s * a->ldbc + g * N;
      double cb = 0.0;
      for (int64_t n = 0; n < N; ++n) cb += Ct[n] * Bs[n];
      M[t * L + s] = cb * exp(seg_sum(a, h, s + 1, t)) * a->dt[s * a->H + h];
    }
  }
  for (int64_t t = 0; t < L; ++t) {
    const double *Ct = a->C + t * a->ldbc + g * N;
    const double carry = exp(seg_sum(a, h, 0, t));
    for (int64_t p = 0; p < P; ++p) {
      double yp = 0.0;
      for (int64_t s = 0; s <= t; ++s) yp += M[t * L + s] * a->x[s * a->ldx + h * P + p];
      if (a->h0 != NULL) {
        double ch = 0.0;
        for (int64_t n = 0; n < N; ++n) ch += Ct[n] * a->h0[(h * P + p) * N + n];
        yp += carry * ch;
      }
      a->y[t * a->ldy + h * P + p] = yp + a->D[h] * a->x[t * a->ldx + h * P + p];
    }
  }
  if (a->hL != NULL) {
    const double carry = exp(seg_sum(a, h, 0, L - 1));
    for (int64_t p = 0; p < P; ++p)
      for (int64_t n = 0; n < N; ++n) {
        double acc = (a->h0 != NULL) ? carry * a->h0[(h * P + p) * N + n] : 0.0;
        for (int64_t s = 0; s < L; ++s)
          acc += exp(seg_sum(a, h, s + 1, L - 1)) * a->dt[s * a->H + h] *
                 a->x[s * a->ldx + h * P + p] * a->B[s * a->ldbc + g * N + n];
        a->hL[(h * P + p) * N + n] = acc;
      }
  }
  free(M);
}

/* Chunked (state-space duality) form for head h, chunk length Q >= 1:
 * inside chunk [c0, c1) with cum[t] = sum_{r=c0..t} dt_r A,
 *   y[t] = sum_{s=c0..t} (C_t . B_s) exp(cum[t]-cum[s]) dt_s x_s     (diagonal block)
 *        + exp(cum[t]) C_t H_c^T                                     (carried state)
 *        + D x_t
 *   S_c   = sum_{s} exp(cum[c1-1]-cum[s]) dt_s x_s B_s^T             (chunk state)
 *   H_{c+1} = exp(cum[c1-1]) H_c + S_c                               (state passing)
 * The last chunk may be shorter than Q. */
static void scan_chunked_head(void *ctx, int64_t h) {
  const m2o_scan_args *a = (const m2o_scan_args *)ctx;
  const int64_t L = a->L, P = a->P, N = a->N, Q = a->chunk, g = group_of(a, h);
  double *Hc = (double *)calloc((size_t)(P * N), sizeof(double));
  double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));
  double *cum = (double *)malloc(sizeof(double) * (size_t)Q);
  if (a->h0 != NULL) memcpy(Hc, a->h0 + h * P * N, sizeof(double) * (size_t)(P * N));
  for (int64_t c0 = 0; c0 < L; c0 += Q) {
    const int64_t c1 = (c0 + Q < L) ? c0 + Q : L;
    double run = 0.0;
    for (int64_t t = c0; t < c1; ++t) {
      run += a->dt[t * a->H + h] * a->A[h];
      cum[t - c0] = run;
    }
    for (int64_t t = c0; t < c1; ++t) {
      const double *Ct = a->C + t * a->ldbc + g * N;
      for (int64_t p = 0; p < P; ++p) {
        double yp = 0.0;
        for (int64_t s = c0; s <= t; ++s) {
          const double *Bs = a->B + s * a->ldbc + g * N;
          double cb = 0.0;
          for (int64_t n = 0; n < N; ++n) cb += Ct[n] * Bs[n];
          yp += cb * exp(cum[t - c0] - cum[s - c0]) * a->dt[s * a->H + h] *
                a->x[s * a->ldx + h * P + p];
        }
        double ch = 0.0;
        for (int64_t n = 0; n < N; ++n) ch += Ct[n] * Hc[p * N + n];
        yp += exp(cum[t - c0]) * ch;
        a->y[t * a->ldy + h * P + p] = yp + a->D[h] * a->x[t * a->ldx + h * P + p];
      }
    }
    for (int64_t p = 0; p < P; ++p)
      for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t s = c0; s < c1; ++s)
          acc += exp(cum[c1 - 1 - c0] - cum[s - c0]) * a->dt[s * a->H + h] *
                 a->x[s * a->ldx + h * P + p] * a->B[s * a->ldbc + g * N + n];
        S[p * N + n] = acc;
      }
    const double chunk_decay = exp(cum[c1 - 1 - c0]);
    for (int64_t i = 0; i < P * N; ++i) Hc[i] = chunk_decay * Hc[i] + S[i];
  }
  if (a->hL != NULL) memcpy(a->hL + h * P * N, Hc, sizeof(double) * (size_t)(P * N));
  free(Hc);
  free(S);
  free(cum);
}

/* form: 0 = sequential, 1 = quadratic, 2 = chunked (chunk = Q). */
int m2o_scan(int form, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
             const double *x, int64_t ldx, const double *B, const double *C, int64_t ldbc,
             const double *dt, const double *A, const double *D, const double *h0, double *y,
             int64_t ldy, double *hL, int64_t chunk, int nthreads) {
  if (L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0) return -1;
  if (form == 2 && chunk < 1) return -1;
  m2o_scan_args a = {L, H, P, N, G, x, ldx, B, C, ldbc, dt, A, D, h0, y, ldy, hL, chunk};
  if (L == 0) {
    if (hL != NULL) {
      if (h0 != NULL) memcpy(hL, h0, sizeof(double) * (size_t)(H * P * N));
      else memset(hL, 0, sizeof(double) * (size_t)(H * P * N));
    }
    return 0;
  }
  m2o_item_fn fn = form == 0 ? scan_sequential_head
                 : form == 1 ? scan_quadratic_head
                 : form == 2 ? scan_chunked_head
                             : NULL;
  if (fn == NULL) return -1;
  m2o_parallel_for(H, nthreads, fn, &a);
  return 0;
}

/* ------------------------------------------------------------------ */
/* gated group RMSNorm                                                */
/* ------------------------------------------------------------------ */

/* For each token and each of the G_norm groups of d_inner/G_norm contiguous
 * channels:
 *   norm_before_gate = 0:  g = y * silu(z);  out = g / sqrt(mean(g^2) + eps) * w
 *   norm_before_gate = 1:  out = y / sqrt(mean(y^2) + eps) * w * silu(z)        */
void m2o_gated_rmsnorm(int64_t L, int64_t d_inner, int64_t G_norm, const double *y, int64_t ldy,
                       const double *z, int64_t ldz, const double *w, double eps,
                       int norm_before_gate, double *out, int64_t ldo) {
  const int64_t gs = d_inner / G_norm;
  double *v = (double *)malloc(sizeof(double) * (size_t)gs);
  for (int64_t t = 0; t < L; ++t)
    for (int64_t k = 0; k < G_norm; ++k) {
      double ss = 0.0;
      for (int64_t i = 0; i < gs; ++i) {
        const int64_t c = k * gs + i;
        v[i] = norm_before_gate ? y[t * ldy + c] : y[t * ldy + c] * m2o_silu(z[t * ldz + c]);
        ss += v[i] * v[i];
      }
      const double inv = 1.0 / sqrt(ss / (double)gs + eps);
      for (int64_t i = 0; i < gs; ++i) {
        const int64_t c = k * gs + i;
        double o = v[i] * inv * w[c];
        if (norm_before_gate) o *= m2o_silu(z[t * ldz + c]);
        out[t * ldo + c] = o;
      }
    }
  free(v);
}

/* ------------------------------------------------------------------ */
/* whole mixer core: prefill over a batch, and the decode step        */
/* ------------------------------------------------------------------ */

typedef struct {
  int64_t batch, L, H, P, N, G, K;
  const double *xBC, *z, *dt_raw;                      /* [b,L,conv_dim], [b,L,H*P], [b,L,H] */
  const double *conv_w, *conv_b, *dt_bias, *A, *D, *norm_w;
  const double *conv_state_in, *ssm_state_in;          /* nullable */
  double *y, *conv_state_out, *ssm_state_out;          /* state outs nullable */
  double eps;
  int norm_before_gate, form;
  int64_t chunk;
  int scan_threads;
} m2o_mixer_args;

static void mixer_prefill_row(void *ctx, int64_t bi) {
  const m2o_mixer_args *m = (const m2o_mixer_args *)ctx;
  const int64_t L = m->L, H = m->H, P = m->P, N = m->N, G = m->G, K = m->K;
  const int64_t d_inner = H * P, conv_dim = d_inner + 2 * G * N;
  double *u = (double *)malloc(sizeof(double) * (size_t)(L * conv_dim + 1));
  double *dt = (double *)malloc(sizeof(double) * (size_t)(L * H + 1));
  double *ypre = (double *)malloc(sizeof(double) * (size_t)(L * d_inner + 1));
  /* step 1: conv + SiLU; the conv state out is the last K raw inputs */
  m2o_conv_silu(L, conv_dim, K, m->xBC + bi * L * conv_dim,
                m->conv_state_in ? m->conv_state_in + bi * conv_dim * K : NULL, m->conv_w,
                m->conv_b, u, m->conv_state_out ? m->conv_state_out + bi * conv_dim * K : NULL);
  /* step 2: dt */
  for (int64_t t = 0; t < L; ++t)
    for (int64_t h = 0; h < H; ++h)
      dt[t * H + h] = m2o_softplus(m->dt_raw[(bi * L + t) * H + h] + m->dt_bias[h]);
  /* step 3: scan (+ D skip) */
  m2o_scan(m->form, L, H, P, N, G, u, conv_dim, u + d_inner, u + d_inner + G * N, conv_dim, dt,
           m->A, m->D, m->ssm_state_in ? m->ssm_state_in + bi * H * P * N : NULL, ypre, d_inner,
           m->ssm_state_out ? m->ssm_state_out + bi * H * P * N : NULL, m->chunk, m->scan_threads);
  /* step 4: gated RMSNorm, ngroups norm groups */
  m2o_gated_rmsnorm(L, d_inner, G, ypre, d_inner, m->z + bi * L * d_inner, d_inner, m->norm_w,
                    m->eps, m->norm_before_gate, m->y + bi * L * d_inner, d_inner);
  free(u);
  free(dt);
  free(ypre);
}

int m2o_mixer_prefill(int64_t batch, int64_t L, int64_t H, int64_t P, int64_t N, int64_t G,
                      int64_t K, const double *xBC, const double *z, const double *dt_raw,
                      const double *conv_w, const double *conv_b, const double *dt_bias,
                      const double *A, const double *D, const double *norm_w,
                      const double *conv_state_in, const double *ssm_state_in, double *y,
                      double *conv_state_out, double *ssm_state_out, double eps,
                      int norm_before_gate, int form, int64_t chunk, int nthreads) {
  if (batch < 0 || L < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || K < 1 || H % G != 0)
    return -1;
  if (form < 0 || form > 2 || (form == 2 && chunk < 1)) return -1;
  m2o_mixer_args m = {batch, L, H, P, N, G, K, xBC, z, dt_raw, conv_w, conv_b, dt_bias, A, D,
                      norm_w, conv_state_in, ssm_state_in, y, conv_state_out, ssm_state_out, eps,
                      norm_before_gate, form, chunk, 1};
  if (nthreads < 1) nthreads = 1;
  if (batch >= nthreads) {
    m2o_parallel_for(batch, nthreads, mixer_prefill_row, &m);
  } else {
    m.scan_threads = nthreads; /* few rows: spread each row's heads instead */
    for (int64_t bi = 0; bi < batch; ++bi) mixer_prefill_row(&m, bi);
  }
  return 0;
}

/* One decode step for batch row bi, written from the single-token update:
 * shift the conv state left by one and append the new xBC column; conv output
 * is the dot product of the K-wide window with the taps; then one step of the
 * recurrence from the carried SSM state.  States are updated in place. */
static void mixer_step_row(void *ctx, int64_t bi) {
  const m2o_mixer_args *m = (const m2o_mixer_args *)ctx;
  const int64_t H = m->H, P = m->P, N = m->N, G = m->G, K = m->K;
  const int64_t d_inner = H * P, conv_dim = d_inner + 2 * G * N;
  double *cs = m->conv_state_out + bi * conv_dim * K;
  double *hs = m->ssm_state_out + bi * H * P * N;
  double *u = (double *)malloc(sizeof(double) * (size_t)conv_dim);
  double *ypre = (double *)malloc(sizeof(double) * (size_t)d_inner);
  for (int64_t c = 0; c < conv_dim; ++c) {
    for (int64_t k = 0; k + 1 < K; ++k) cs[c * K + k] = cs[c * K + k + 1];
    cs[c * K + K - 1] = m->xBC[bi * conv_dim + c];
    double acc = m->conv_b[c];
    for (int64_t k = 0; k < K; ++k) acc += m->conv_w[c * K + k] * cs[c * K + k];
    u[c] = m2o_silu(acc);
  }
  for (int64_t h = 0; h < H; ++h) {
    const int64_t g = h / (H / G);
    const double dt = m2o_softplus(m->dt_raw[bi * H + h] + m->dt_bias[h]);
    const double decay = exp(dt * m->A[h]);
    const double *Bv = u + d_inner + g * N;
    const double *Cv = u + d_inner + G * N + g * N;
    for (int64_t p = 0; p < P; ++p) {
      const double xp = u[h * P + p];
      double yp = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        double *s = &hs[(h * P + p) * N + n];
        *s = decay * (*s) + dt * xp * Bv[n];
        yp += (*s) * Cv[n];
      }
      ypre[h * P + p] = yp + m->D[h] * xp;
    }
  }
  m2o_gated_rmsnorm(1, d_inner, G, ypre, d_inner, m->z + bi * d_inner, d_inner, m->norm_w, m->eps,
                    m->norm_before_gate, m->y + bi * d_inner, d_inner);
  free(u);
  free(ypre);
}

/* States are updated in place: conv_state [b, conv_dim, K], ssm_state [b, H, P, N]. */
int m2o_mixer_step(int64_t batch, int64_t H, int64_t P, int64_t N, int64_t G, int64_t K,
                   const double *xBC, const double *z, const double *dt_raw,
                   const double *conv_w, const double *conv_b, const double *dt_bias,
                   const double *A, const double *D, const double *norm_w, double *conv_state,
                   double *ssm_state, double *y, double eps, int norm_before_gate,
                   int nthreads) {
  if (batch < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || K < 1 || H % G != 0) return -1;
  if (conv_state == NULL || ssm_state == NULL) return -1;
  m2o_mixer_args m = {batch, 1, H, P, N, G, K, xBC, z, dt_raw, conv_w, conv_b, dt_bias, A, D,
                      norm_w, NULL, NULL, y, conv_state, ssm_state, eps, norm_before_gate, 0, 0,
                      1};
  m2o_parallel_for(batch, nthreads < 1 ? 1 : nthreads, mixer_step_row, &m);
  return 0;
}
