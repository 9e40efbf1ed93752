/*
 * wkv7_oracle_bwd.c -- float64 CPU oracle for the gradients of the RWKV-7 (x070) state recurrence.
 *
 * TEST INFRASTRUCTURE ONLY, like wkv7_oracle.c beside it: the slow, plain reverse-mode
 * differentiation that the CUDA backward is checked against.  It shares no code with the CUDA
 * library, and the library never calls it.
 *
 * The forward it differentiates is the token loop of wkv7_oracle.c (RWKV-7 G0 7.2B walkthrough,
 * lshu.cn/news/198401, section 7.1): per (b, h),
 *     sa = S a_t;   S <- S diag(w_t) + sa b_t^T + v_t k_t^T;   y_t = S r_t
 * from S = s_in to s_out.  The pages give no backward; this file is the chain rule applied to
 * that loop, for the scalar  L = sum_t <dy_t, y_t> + <ds_out, s_out>.  With S' the state after
 * token t and S the state before it, walking t from T-1 down to 0 with G = dL/dS' (starting from
 * ds_out):
 *     G += dy_t r_t^T                       (y_t = S' r_t)
 *     dr_t = S'^T dy_t
 *     dv_t = G k_t,   dk_t = G^T v_t          (the write v_t k_t^T)
 *     db_t = G^T sa,  g_sa = G b_t            (the rank-one term sa b_t^T)
 *     dw_t[j] = sum_i G[i][j] S[i][j]         (the decay S diag(w_t))
 *     da_t = S^T g_sa                         (sa = S a_t)
 *     G <- G diag(w_t) + g_sa a_t^T           (dL/dS, the next G)
 * and finally ds_in = G.
 *
 * The states S are recomputed: the forward keeps the state at every 64th token, and the walk
 * back recomputes one 64-token block at a time from its saved state (the same operations in the
 * same order, so the recomputed states are the forward's states exactly).
 *
 * Layouts as in wkv7_oracle.c: token tensors [B, T, H, N], states [B, H, N, N], row-major.
 * Threads split the (b, h) pairs; results do not depend on the thread count.  Build without
 * -ffast-math and with -ffp-contract=off.
 */
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

enum { BLK = 64 };

typedef struct {
  int B, T, H, N;
  const double *r, *w, *k, *v, *a, *b, *s_in, *dy, *ds_out;
  double *dr, *dw, *dk, *dv, *da, *db, *ds_in;
  int first_pair, end_pair;
  int status;
} bjob_t;

/* One forward token: S (N x N) updated in place; sa (N) receives S a before the update. */
static void step(int N, double *S, double *sa, const double *w, const double *k, const double *v,
                 const double *a, const double *b) {
  for (int i = 0; i < N; ++i) {
    double acc = 0;
    for (int j = 0; j < N; ++j) acc += S[(size_t)i * N + j] * a[j];
    sa[i] = acc;
  }
  for (int i = 0; i < N; ++i)
    for (int j = 0; j < N; ++j) {
      const double s = S[(size_t)i * N + j];
      S[(size_t)i * N + j] = s * w[j] + sa[i] * b[j] + v[i] * k[j];
    }
}

static int run_pair(const bjob_t *jb, int pair) {
  const int T = jb->T, H = jb->H, N = jb->N;
  const int bb = pair / H, hh = pair % H;
  const size_t NN = (size_t)N * N;
  const int nblk = (T + BLK - 1) / BLK;
  double *ckpt = (double *)malloc(sizeof(double) * NN * (size_t)(nblk > 0 ? nblk : 1));
  double *states = (double *)malloc(sizeof(double) * NN * (BLK + 1));
  double *G = (double *)malloc(sizeof(double) * NN);
  double *sa = (double *)malloc(sizeof(double) * (size_t)N * 2);
  if (!ckpt || !states || !G || !sa) {
    free(ckpt);
    free(states);
    free(G);
    free(sa);
    return 1;
  }
  double *gsa = sa + N;
  const size_t sbase = (size_t)pair * NN;
#define TOK(t) ((((size_t)bb * T + (t)) * H + hh) * (size_t)N)

  /* forward, keeping the state before every block */
  double *S = states; /* scratch for the forward sweep */
  for (size_t e = 0; e < NN; ++e) S[e] = jb->s_in ? jb->s_in[sbase + e] : 0.0;
  for (int t = 0; t < T; ++t) {
    if (t % BLK == 0) memcpy(ckpt + (size_t)(t / BLK) * NN, S, sizeof(double) * NN);
    const size_t x = TOK(t);
    step(N, S, sa, jb->w + x, jb->k + x, jb->v + x, jb->a + x, jb->b + x);
  }

  for (size_t e = 0; e < NN; ++e) G[e] = jb->ds_out ? jb->ds_out[sbase + e] : 0.0;
  for (int blk = nblk - 1; blk >= 0; --blk) {
    const int t0 = blk * BLK;
    const int L = (T - t0) < BLK ? (T - t0) : BLK;
    /* states[u] = state before token t0 + u, u = 0 .. L */
    memcpy(states, ckpt + (size_t)blk * NN, sizeof(double) * NN);
    for (int u = 0; u < L; ++u) {
      memcpy(states + (size_t)(u + 1) * NN, states + (size_t)u * NN, sizeof(double) * NN);
      const size_t x = TOK(t0 + u);
      step(N, states + (size_t)(u + 1) * NN, sa, jb->w + x, jb->k + x, jb->v + x, jb->a + x, jb->b + x);
    }
    for (int u = L - 1; u >= 0; --u) {
      const size_t x = TOK(t0 + u);
      const double *Sp = states + (size_t)u * NN;       /* before the token */
      const double *Sn = states + (size_t)(u + 1) * NN; /* after the token */
      const double *r = jb->r + x, *w = jb->w + x, *k = jb->k + x, *v = jb->v + x;
      const double *a = jb->a + x, *b = jb->b + x, *dy = jb->dy + x;
      /* y_t = S' r_t */
      for (int i = 0; i < N; ++i)
        for (int j = 0; j < N; ++j) G[(size_t)i * N + j] += dy[i] * r[j];
      for (int j = 0; j < N; ++j) {
        double acc = 0;
        for (int i = 0; i < N; ++i) acc += Sn[(size_t)i * N + j] * dy[i];
        jb->dr[x + j] = acc;
      }
      /* the write v_t k_t^T */
      for (int i = 0; i < N; ++i) {
        double acc = 0;
        for (int j = 0; j < N; ++j) acc += G[(size_t)i * N + j] * k[j];
        jb->dv[x + i] = acc;
      }
      for (int j = 0; j < N; ++j) {
        double acc = 0;
        for (int i = 0; i < N; ++i) acc += G[(size_t)i * N + j] * v[i];
        jb->dk[x + j] = acc;
      }
      /* the rank-one term sa b_t^T, sa = S a_t */
      for (int i = 0; i < N; ++i) {
        double acc = 0;
        for (int j = 0; j < N; ++j) acc += Sp[(size_t)i * N + j] * a[j];
        sa[i] = acc;
      }
      for (int j = 0; j < N; ++j) {
        double acc = 0;
        for (int i = 0; i < N; ++i) acc += G[(size_t)i * N + j] * sa[i];
        jb->db[x + j] = acc;
      }
      for (int i = 0; i < N; ++i) {
        double acc = 0;
        for (int j = 0; j < N; ++j) acc += G[(size_t)i * N + j] * b[j];
        gsa[i] = acc;
      }
      /* the decay S diag(w_t) */
      for (int j = 0; j < N; ++j) {
        double acc = 0;
        for (int i = 0; i < N; ++i) acc += G[(size_t)i * N + j] * Sp[(size_t)i * N + j];
        jb->dw[x + j] = acc;
      }
      for (int j = 0; j < N; ++j) {
        double acc = 0;
        for (int i = 0; i < N; ++i) acc += Sp[(size_t)i * N + j] * gsa[i];
        jb->da[x + j] = acc;
      }
      /* dL/dS for the state before the token */
      for (int i = 0; i < N; ++i)
        for (int j = 0; j < N; ++j) G[(size_t)i * N + j] = G[(size_t)i * N + j] * w[j] + gsa[i] * a[j];
    }
  }
  if (jb->ds_in)
    for (size_t e = 0; e < NN; ++e) jb->ds_in[sbase + e] = G[e];
#undef TOK
  free(ckpt);
  free(states);
  free(G);
  free(sa);
  return 0;
}

static void *worker(void *arg) {
  bjob_t *jb = (bjob_t *)arg;
  jb->status = 0;
  for (int p = jb->first_pair; p < jb->end_pair; ++p)
    if (run_pair(jb, p)) {
      jb->status = 1;
      break;
    }
  return NULL;
}

/* Gradients of L = sum <dy, y> + <ds_out, s_out> with respect to r, w, k, v, a, b ([B,T,H,N])
 * and s_in ([B,H,N,N]; ds_in may be NULL).  s_in and ds_out may be NULL (zero).  Returns 0 on
 * success, 1 on a bad argument, 2 when memory or threads could not be had. */
int wkv7_oracle_bwd_f64(int B, int T, int H, int N, const double *r, const double *w, const double *k,
                        const double *v, const double *a, const double *b, const double *s_in, const double *dy,
                        const double *ds_out, double *dr, double *dw, double *dk, double *dv, double *da,
                        double *db, double *ds_in, int nthreads) {
  if (B <= 0 || H <= 0 || N <= 0 || T < 0) return 1;
  if (T > 0 && (!r || !w || !k || !v || !a || !b || !dy || !dr || !dw || !dk || !dv || !da || !db)) return 1;
  const int pairs = B * H;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > pairs) nthreads = pairs;
  bjob_t *jobs = (bjob_t *)calloc((size_t)nthreads, sizeof(bjob_t));
  pthread_t *tids = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return 2;
  }
  for (int i = 0; i < nthreads; ++i) {
    bjob_t *jb = &jobs[i];
    jb->B = B; jb->T = T; jb->H = H; jb->N = N;
    jb->r = r; jb->w = w; jb->k = k; jb->v = v; jb->a = a; jb->b = b;
    jb->s_in = s_in; jb->dy = dy; jb->ds_out = ds_out;
    jb->dr = dr; jb->dw = dw; jb->dk = dk; jb->dv = dv; jb->da = da; jb->db = db; jb->ds_in = ds_in;
    jb->first_pair = (int)((long long)pairs * i / nthreads);
    jb->end_pair = (int)((long long)pairs * (i + 1) / nthreads);
  }
  int started = 0;
  for (int i = 1; i < nthreads; ++i) {
    if (pthread_create(&tids[i], NULL, worker, &jobs[i]) != 0) break;
    started = i;
  }
  worker(&jobs[0]);
  for (int i = started + 1; i < nthreads; ++i) worker(&jobs[i]);
  for (int i = 1; i <= started; ++i) pthread_join(tids[i], NULL);
  int status = 0;
  for (int i = 0; i < nthreads; ++i) status |= jobs[i].status;
  free(jobs);
  free(tids);
  return status ? 2 : 0;
}
