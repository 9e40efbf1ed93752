/*
 * wkv7_oracle.c -- float64 CPU oracle for the RWKV-7 (x070) state recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * definition that the CUDA library is checked against.  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load it.  It shares no
 * code, header, table or helper with the CUDA library, and the library never
 * calls it.
 *
 * What it computes (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401,
 * section 7.1, "the two core operators of x070": the state is decayed by w,
 * gets the rank-one term state.a b^T and the write v k^T, and is read out
 * with r; RWKV-LM README copy, oa0.com/c/1004164, the note that the state
 * and w must be kept in fp32 or better because w can be very close to 1;
 * Swarma wiki RWKV entry, "Delta Rule" section, vector-valued gating of the
 * state):
 *
 *   for every batch row b and head h, with S an N x N matrix whose row i is a
 *   value channel and whose column j is a key channel,
 *     S = s_in[b,h]            (zero when s_in is NULL)
 *     for t = 0 .. T-1:
 *       sa_i   = sum_j S[i][j] * a_t[j]                  (S before the update)
 *       S[i][j] = S[i][j] * w_t[j] + sa_i * b_t[j] + v_t[i] * k_t[j]
 *       y_t[i] = sum_j S[i][j] * r_t[j]                  (S after the update)
 *     s_out[b,h] = S
 *
 * Layouts (row-major, contiguous):
 *   r, w, k, v, a, b, y : [B, T, H, N]   element (b,t,h,n) at ((b*T+t)*H+h)*N+n
 *   s_in, s_out         : [B, H, N, N]   element (b,h,i,j) at ((b*H+h)*N+i)*N+j
 *
 * Arithmetic: every operand is widened to ORACLE_REAL (double by default; the
 * same source built with -DORACLE_REAL="long double" gives the higher-
 * precision copy the tests use to bound this file's own rounding).  The loops
 * run in the plain order above.  Build without -ffast-math and with
 * -ffp-contract=off.
 *
 * Threads split the (b, h) pairs; each pair is computed by exactly one thread
 * in the fixed order above, so results do not depend on the thread count.
 */

#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_REAL
#define ORACLE_REAL double
#endif
typedef ORACLE_REAL real_t;

/* Where the operands come from: float32 or float64 arrays. */
enum { SRC_F32 = 0, SRC_F64 = 1 };

typedef struct {
  int B, T, H, N;
  int src;
  const void *r, *w, *k, *v, *a, *b;
  const double *s_in;
  double *y, *s_out;
  int first_pair, end_pair; /* this worker's (b*H + h) range */
  int status;
} job_t;

static real_t load(const void *base, int src, size_t idx) {
  if (src == SRC_F32) return (real_t)((const float *)base)[idx];
  return (real_t)((const double *)base)[idx];
}

/* One (b, h) pair, token by token. */
static int run_pair(const job_t *jb, int pair) {
  const int T = jb->T, H = jb->H, N = jb->N;
  const int bb = pair / H, hh = pair % H;
  real_t *S = (real_t *)malloc(sizeof(real_t) * (size_t)N * N);
  real_t *vec = (real_t *)malloc(sizeof(real_t) * (size_t)N * 7);
  if (!S || !vec) {
    free(S);
    free(vec);
    return 1;
  }
  real_t *r = vec, *w = vec + N, *k = vec + 2 * N, *v = vec + 3 * N;
  real_t *a = vec + 4 * N, *b = vec + 5 * N, *sa = vec + 6 * N;

  const size_t sbase = (size_t)pair * N * N;
  for (int e = 0; e < N * N; ++e) S[e] = jb->s_in ? (real_t)jb->s_in[sbase + e] : (real_t)0;

  for (int t = 0; t < T; ++t) {
    const size_t xbase = (((size_t)bb * T + t) * H + hh) * (size_t)N;
    for (int n = 0; n < N; ++n) {
      r[n] = load(jb->r, jb->src, xbase + n);
      w[n] = load(jb->w, jb->src, xbase + n);
      k[n] = load(jb->k, jb->src, xbase + n);
      v[n] = load(jb->v, jb->src, xbase + n);
      a[n] = load(jb->a, jb->src, xbase + n);
      b[n] = load(jb->b, jb->src, xbase + n);
    }
    /* sa = S a, with the state as it was before this token */
    for (int i = 0; i < N; ++i) {
      real_t acc = 0;
      for (int j = 0; j < N; ++j) acc += S[(size_t)i * N + j] * a[j];
      sa[i] = acc;
    }
    /* S <- S diag(w) + sa b^T + v k^T */
    for (int i = 0; i < N; ++i)
      for (int j = 0; j < N; ++j) {
        real_t s = S[(size_t)i * N + j];
        S[(size_t)i * N + j] = s * w[j] + sa[i] * b[j] + v[i] * k[j];
      }
    /* y = S r, with the updated state */
    for (int i = 0; i < N; ++i) {
      real_t acc = 0;
      for (int j = 0; j < N; ++j) acc += S[(size_t)i * N + j] * r[j];
      jb->y[xbase + i] = (double)acc;
    }
  }
  for (int e = 0; e < N * N; ++e) jb->s_out[sbase + e] = (double)S[e];
  free(S);
  free(vec);
  return 0;
}

static void *worker(void *arg) {
  job_t *jb = (job_t *)arg;
  jb->status = 0;
  for (int p = jb->first_pair; p < jb->end_pair; ++p)
    if (run_pair(jb, p)) {
      jb->status = 1;
      break;
    }
  return NULL;
}

static int run(int B, int T, int H, int N, int src, const void *r, const void *w, const void *k,
               const void *v, const void *a, const void *b, const double *s_in, double *y,
               double *s_out, int nthreads) {
  if (B <= 0 || H <= 0 || N <= 0 || T < 0) return 1;
  if (!s_out || (T > 0 && (!r || !w || !k || !v || !a || !b || !y))) return 1;
  const int pairs = B * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > pairs) nthreads = pairs;

  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return 2;
  }
  for (int i = 0; i < nthreads; ++i) {
    job_t *jb = &jobs[i];
    jb->B = B; jb->T = T; jb->H = H; jb->N = N; jb->src = src;
    jb->r = r; jb->w = w; jb->k = k; jb->v = v; jb->a = a; jb->b = b;
    jb->s_in = s_in; jb->y = y; jb->s_out = s_out;
    jb->first_pair = (int)((long long)pairs * i / nthreads);
    jb->end_pair = (int)((long long)pairs * (i + 1) / nthreads);
  }
  int started = 0;
  for (int i = 1; i < nthreads; ++i) {
    if (pthread_create(&tids[i], NULL, worker, &jobs[i]) != 0) break;
    started = i;
  }
  worker(&jobs[0]);
  /* any worker that could not be started runs here */
  for (int i = started + 1; i < nthreads; ++i) worker(&jobs[i]);
  for (int i = 1; i <= started; ++i) pthread_join(tids[i], NULL);
  int status = 0;
  for (int i = 0; i < nthreads; ++i) status |= jobs[i].status;
  free(jobs);
  free(tids);
  return status ? 2 : 0;
}

/* float64 operands.  Returns 0 on success, 1 on a bad argument, 2 when memory
 * or threads could not be had.  s_in may be NULL (zero initial state). */
int wkv7_oracle_f64(int B, int T, int H, int N, const double *r, const double *w, const double *k,
                    const double *v, const double *a, const double *b, const double *s_in,
                    double *y, double *s_out, int nthreads) {
  return run(B, T, H, N, SRC_F64, r, w, k, v, a, b, s_in, y, s_out, nthreads);
}

/* float32 operands (exact copies of fp32 or bf16 inputs), float64 arithmetic
 * and outputs.  Same return codes as wkv7_oracle_f64. */
int wkv7_oracle_f32in(int B, int T, int H, int N, const float *r, const float *w, const float *k,
                      const float *v, const float *a, const float *b, const double *s_in,
                      double *y, double *s_out, int nthreads) {
  return run(B, T, H, N, SRC_F32, r, w, k, v, a, b, s_in, y, s_out, nthreads);
}

/* sizeof(real_t), so a caller can tell the double and long double builds apart. */
int wkv7_oracle_real_bytes(void) { return (int)sizeof(real_t); }
