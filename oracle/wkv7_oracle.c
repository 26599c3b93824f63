/*
 * WKV-7 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct fp64 implementation of the WKV-7 recurrence
 * (the generalised delta rule of RWKV-7 "Goose"), its hand-derived backward
 * pass and its single-token decode step.  Only the test suite, the smoke
 * check and the benchmark's CPU-baseline leg load this file; the CUDA library
 * never does, and the two share no code.
 *
 * The method (rwkv-metal page, "The Metal WKV-7 kernel": one state per head,
 * updated token by token; RWKV-MLX page, "Key Design Decisions" 1-2).  Per
 * (batch b, head h) the state S is an N x N matrix, row i = value channel,
 * column j = key channel.  For each token t:
 *
 *     sa[i]   = sum_j S[i][j] * a[j]                  (S before the update)
 *     S[i][j] = S[i][j]*w[j] + sa[i]*b[j] + v[i]*k[j]
 *     y[i]    = sum_j S[i][j] * r[j]                  (S after the update)
 *
 * i.e. S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T and y_t = S_t r_t.
 * A reset flag at token t replaces the incoming state by zero before the
 * token is applied (packed sequences, HF model card page: the state is zeroed
 * where each packed document begins).
 *
 * Layout: r,w,k,v,a,b,y,dy and the gradients are [B,T,H,N] row-major;
 * states are [B,H,N,N] row-major (S[i][j] at i*N+j); reset is [B,T] bytes.
 * Units (b,h) are independent and are spread over POSIX threads.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
  int64_t B, T, H, N;
  const double *r, *w, *k, *v, *a, *b, *s0, *dy, *dsT;
  const uint8_t* reset;
  double *y, *s_out;
  double *dr, *dw, *dk, *dv, *da, *db, *ds0;
  int64_t next_unit;
  pthread_mutex_t lock;
  int failed;
} job_t;

static int64_t take_unit(job_t* J) {
  pthread_mutex_lock(&J->lock);
  int64_t u = J->next_unit++;
  pthread_mutex_unlock(&J->lock);
  return u;
}

/* offset of x[b][t][h][0] in a [B,T,H,N] tensor */
static int64_t tok(const job_t* J, int64_t b, int64_t t, int64_t h) {
  return ((b * J->T + t) * J->H + h) * J->N;
}

/* --------------------------------------------------------------- forward */
/* One (b,h) unit, token order, exactly the three lines of the method. */
static void forward_unit(job_t* J, int64_t b, int64_t h, double* S, double* sa) {
  const int64_t N = J->N;
  const int64_t unit = b * J->H + h;
  if (J->s0)
    memcpy(S, J->s0 + unit * N * N, sizeof(double) * N * N);
  else
    memset(S, 0, sizeof(double) * N * N);
  for (int64_t t = 0; t < J->T; ++t) {
    const int64_t o = tok(J, b, t, h);
    const double *w = J->w + o, *k = J->k + o, *v = J->v + o;
    const double *a = J->a + o, *bb = J->b + o, *r = J->r + o;
    if (J->reset && J->reset[b * J->T + t]) memset(S, 0, sizeof(double) * N * N);
    for (int64_t i = 0; i < N; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < N; ++j) acc += S[i * N + j] * a[j];
      sa[i] = acc;
    }
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j)
        S[i * N + j] = S[i * N + j] * w[j] + sa[i] * bb[j] + v[i] * k[j];
    for (int64_t i = 0; i < N; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < N; ++j) acc += S[i * N + j] * r[j];
      J->y[o + i] = acc;
    }
  }
  if (J->s_out) memcpy(J->s_out + unit * N * N, S, sizeof(double) * N * N);
}

static void* forward_worker(void* arg) {
  job_t* J = (job_t*)arg;
  const int64_t N = J->N;
  double* S = (double*)malloc(sizeof(double) * N * N);
  double* sa = (double*)malloc(sizeof(double) * N);
  if (!S || !sa) { J->failed = 1; free(S); free(sa); return NULL; }
  for (int64_t u; (u = take_unit(J)) < J->B * J->H;) forward_unit(J, u / J->H, u % J->H, S, sa);
  free(S);
  free(sa);
  return NULL;
}

/* --------------------------------------------------------------- backward */
/*
 * Reverse-mode derivative of the forward above (derived by hand; the pages
 * print none).  With G_t = diag(w_t) + a_t b_t^T the forward is
 * S_t = P_t G_t + v_t k_t^T, y_t = S_t r_t, where P_t is the state entering
 * token t (zero if reset[t], else S_{t-1}).  Carrying D = dL/dS_t backwards:
 *
 *     D    += dy_t r_t^T                 (y_t reads S_t)
 *     dr_t  = S_t^T dy_t
 *     dv_t  = D k_t,   dk_t = D^T v_t
 *     dsa   = D b_t,   db_t = D^T sa_t   (sa_t = P_t a_t)
 *     dw_t  = diag(D^T P_t)              i.e. dw_t[j] = sum_i D[i][j] P_t[i][j]
 *     da_t  = P_t^T dsa
 *     D     = D diag(w_t) + dsa a_t^T     (= D G_t^T, the gradient w.r.t. P_t)
 *     if reset[t]:  D = 0                 (P_t is a constant zero)
 *
 * and dS0 is D after t = 0.  Every P_t is kept (no checkpoints, no inversion).
 */
static void backward_unit(job_t* J, int64_t b, int64_t h, double* P, double* D, double* sa,
                          double* dsa) {
  const int64_t N = J->N, NN = N * N, T = J->T;
  const int64_t unit = b * J->H + h;
  /* forward, keeping P_t (state entering token t) for every t, and S_T in P[T] */
  double* S = P + T * NN;
  if (J->s0)
    memcpy(S, J->s0 + unit * NN, sizeof(double) * NN);
  else
    memset(S, 0, sizeof(double) * NN);
  for (int64_t t = 0; t < T; ++t) {
    const int64_t o = tok(J, b, t, h);
    double* Pt = P + t * NN;
    if (J->reset && J->reset[b * T + t])
      memset(Pt, 0, sizeof(double) * NN);
    else
      memcpy(Pt, S, sizeof(double) * NN);
    for (int64_t i = 0; i < N; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < N; ++j) acc += Pt[i * N + j] * J->a[o + j];
      sa[t * N + i] = acc;
    }
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j)
        S[i * N + j] = Pt[i * N + j] * J->w[o + j] + sa[t * N + i] * J->b[o + j] + J->v[o + i] * J->k[o + j];
  }
  /* S now holds S_T; rebuild S_t on the way back as P_{t+1} unless a reset sits at t+1 */
  double* St = (double*)malloc(sizeof(double) * NN);
  if (!St) { J->failed = 1; return; }
  if (J->dsT)
    memcpy(D, J->dsT + unit * NN, sizeof(double) * NN);
  else
    memset(D, 0, sizeof(double) * NN);
  for (int64_t t = T - 1; t >= 0; --t) {
    const int64_t o = tok(J, b, t, h);
    const double *w = J->w + o, *k = J->k + o, *v = J->v + o;
    const double *a = J->a + o, *bb = J->b + o, *r = J->r + o, *dy = J->dy + o;
    const double* Pt = P + t * NN;
    /* S_t = P_t G_t + v_t k_t^T, recomputed directly from P_t */
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j)
        St[i * N + j] = Pt[i * N + j] * w[j] + sa[t * N + i] * bb[j] + v[i] * k[j];
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) D[i * N + j] += dy[i] * r[j];
    for (int64_t j = 0; j < N; ++j) {
      double acc_r = 0.0, acc_k = 0.0, acc_b = 0.0, acc_w = 0.0;
      for (int64_t i = 0; i < N; ++i) {
        acc_r += St[i * N + j] * dy[i];
        acc_k += D[i * N + j] * v[i];
        acc_b += D[i * N + j] * sa[t * N + i];
        acc_w += D[i * N + j] * Pt[i * N + j];
      }
      J->dr[o + j] = acc_r;
      J->dk[o + j] = acc_k;
      J->db[o + j] = acc_b;
      J->dw[o + j] = acc_w;
    }
    for (int64_t i = 0; i < N; ++i) {
      double acc_v = 0.0, acc_s = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        acc_v += D[i * N + j] * k[j];
        acc_s += D[i * N + j] * bb[j];
      }
      J->dv[o + i] = acc_v;
      dsa[i] = acc_s;
    }
    for (int64_t j = 0; j < N; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < N; ++i) acc += Pt[i * N + j] * dsa[i];
      J->da[o + j] = acc;
    }
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = 0; j < N; ++j) D[i * N + j] = D[i * N + j] * w[j] + dsa[i] * a[j];
    if (J->reset && J->reset[b * T + t]) memset(D, 0, sizeof(double) * NN);
  }
  free(St);
  if (J->ds0) memcpy(J->ds0 + unit * NN, D, sizeof(double) * NN);
}

static void* backward_worker(void* arg) {
  job_t* J = (job_t*)arg;
  const int64_t N = J->N, NN = N * N, T = J->T;
  double* P = (double*)malloc(sizeof(double) * NN * (size_t)(T + 1));
  double* D = (double*)malloc(sizeof(double) * NN);
  double* sa = (double*)malloc(sizeof(double) * N * (size_t)T);
  double* dsa = (double*)malloc(sizeof(double) * N);
  if (!P || !D || !sa || !dsa) {
    J->failed = 1;
  } else {
    for (int64_t u; (u = take_unit(J)) < J->B * J->H;) backward_unit(J, u / J->H, u % J->H, P, D, sa, dsa);
  }
  free(P);
  free(D);
  free(sa);
  free(dsa);
  return NULL;
}

/* --------------------------------------------------------------- driver */
static int run(job_t* J, void* (*fn)(void*), int nthreads) {
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > J->B * J->H) nthreads = (int)(J->B * J->H);
  if (nthreads < 1) nthreads = 1;
  J->next_unit = 0;
  J->failed = 0;
  pthread_mutex_init(&J->lock, NULL);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, fn, J) == 0) ++started;
  if (started == 0) fn(J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J->lock);
  return J->failed ? -1 : started > 0 ? started : 1;
}

/* Returns the number of threads used, or -1 on allocation failure. */
int wkv7_oracle_forward(int64_t B, int64_t T, int64_t H, int64_t N, const double* r, const double* w,
                        const double* k, const double* v, const double* a, const double* b,
                        const double* s0, const uint8_t* reset, double* y, double* s_out, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.B = B; J.T = T; J.H = H; J.N = N;
  J.r = r; J.w = w; J.k = k; J.v = v; J.a = a; J.b = b;
  J.s0 = s0; J.reset = reset; J.y = y; J.s_out = s_out;
  if (T == 0) {
    /* no tokens: the final state is the initial one */
    if (s_out) {
      if (s0) memcpy(s_out, s0, sizeof(double) * B * H * N * N);
      else memset(s_out, 0, sizeof(double) * B * H * N * N);
    }
    return 1;
  }
  return run(&J, forward_worker, nthreads);
}

int wkv7_oracle_backward(int64_t B, int64_t T, int64_t H, int64_t N, const double* r, const double* w,
                         const double* k, const double* v, const double* a, const double* b,
                         const double* s0, const uint8_t* reset, const double* dy, const double* dsT,
                         double* dr, double* dw, double* dk, double* dv, double* da, double* db,
                         double* ds0, int nthreads) {
  job_t J;
  memset(&J, 0, sizeof(J));
  J.B = B; J.T = T; J.H = H; J.N = N;
  J.r = r; J.w = w; J.k = k; J.v = v; J.a = a; J.b = b;
  J.s0 = s0; J.reset = reset; J.dy = dy; J.dsT = dsT;
  J.dr = dr; J.dw = dw; J.dk = dk; J.dv = dv; J.da = da; J.db = db; J.ds0 = ds0;
  if (T == 0) {
    if (ds0) {
      if (dsT) memcpy(ds0, dsT, sizeof(double) * B * H * N * N);
      else memset(ds0, 0, sizeof(double) * B * H * N * N);
    }
    return 1;
  }
  return run(&J, backward_worker, nthreads);
}

/*
 * Single-token decode step on a resident state (rwkv-metal page: one token on
 * a carried state; ragged batches padded on the right, the padded rows' results
 * unchanged).  state is [B,H,N,N] in/out, the
 * token inputs and y are [B,H,N].  Rows with active[b] == 0 keep their state
 * untouched and get y = 0.  active may be NULL (all rows active).
 */
void wkv7_oracle_step(int64_t B, int64_t H, int64_t N, const double* r, const double* w, const double* k,
                      const double* v, const double* a, const double* b, double* state,
                      const uint8_t* active, double* y) {
  double* sa = (double*)malloc(sizeof(double) * N);
  if (!sa) return;
  for (int64_t bi = 0; bi < B; ++bi) {
    for (int64_t h = 0; h < H; ++h) {
      const int64_t o = (bi * H + h) * N;
      double* S = state + (bi * H + h) * N * N;
      if (active && !active[bi]) {
        for (int64_t i = 0; i < N; ++i) y[o + i] = 0.0;
        continue;
      }
      for (int64_t i = 0; i < N; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < N; ++j) acc += S[i * N + j] * a[o + j];
        sa[i] = acc;
      }
      for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < N; ++j)
          S[i * N + j] = S[i * N + j] * w[o + j] + sa[i] * b[o + j] + v[o + i] * k[o + j];
      for (int64_t i = 0; i < N; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < N; ++j) acc += S[i * N + j] * r[o + j];
        y[o + i] = acc;
      }
    }
  }
  free(sa);
}
