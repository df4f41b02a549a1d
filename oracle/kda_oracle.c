/*
 * KDA forward oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU restatement of the Kimi Delta Attention recurrence
 * (Kimi K3 technical report, section 2.1.1, Eq. 1):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = scale * S_t^T q_t,            alpha_t = exp(g_t)  (Eq. 5),
 *
 * evaluated token by token in the order the equation is printed: decay the
 * state row-wise by alpha_t (one factor per key channel), erase along k_t
 * using the decayed state, write beta_t k_t v_t^T, then read the output from
 * the post-update state (the report keeps the diagonal of the intra-chunk
 * mask because every output reads the state after its own token).  The output
 * scale (dk^-1/2 by default) multiplies o only, never the state.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use
 * this file; the CUDA library shares no code with it.  Build:
 *     gcc -O2 -fPIC -shared -o liboracle.so kda_oracle.c -lm -lpthread
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  const double *q, *k, *v, *g, *beta, *h0;
  double *o, *hT;
  int B, H, T, dk, dv, erase;
  double scale;
  int next;                 /* next (b,h) chain to run; guarded by mu */
  pthread_mutex_t mu;
  int failed;
} job_t;

/* One (b,h) chain.  Layouts (row-major): q,k,g [T,dk]; v [T,dv]; beta [T];
 * h0, hT [dk,dv] (h0 may be NULL = zeros); o [T,dv]. */
static int run_chain(const double *q, const double *k, const double *v, const double *g,
                     const double *beta, const double *h0, double *o, double *hT, int T, int dk,
                     int dv, double scale, int erase) {
  double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
  double *p = (double *)malloc(sizeof(double) * (size_t)dv);
  if (!S || !p) {
    free(S);
    free(p);
    return -1;
  }
  if (h0)
    memcpy(S, h0, sizeof(double) * (size_t)dk * dv);
  else
    memset(S, 0, sizeof(double) * (size_t)dk * dv);

  for (int t = 0; t < T; ++t) {
    const double *qt = q + (size_t)t * dk, *kt = k + (size_t)t * dk, *gt = g + (size_t)t * dk;
    const double *vt = v + (size_t)t * dv;
    const double bt = beta[t];
    /* Diag(alpha_t) S_{t-1}: alpha acts on the key dimension (rows of S). */
    for (int i = 0; i < dk; ++i) {
      const double a = exp(gt[i]);
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
    }
    /* (I - beta k k^T) applied to the decayed state. */
    if (erase) {
      for (int j = 0; j < dv; ++j) p[j] = 0.0;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) p[j] += kt[i] * S[(size_t)i * dv + j];
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] -= bt * kt[i] * p[j];
    }
    /* + beta k v^T */
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += bt * kt[i] * vt[j];
    /* o_t = scale * S_t^T q_t */
    for (int j = 0; j < dv; ++j) p[j] = 0.0;
    for (int i = 0; i < dk; ++i)
      for (int j = 0; j < dv; ++j) p[j] += qt[i] * S[(size_t)i * dv + j];
    for (int j = 0; j < dv; ++j) o[(size_t)t * dv + j] = scale * p[j];
  }
  if (hT) memcpy(hT, S, sizeof(double) * (size_t)dk * dv);
  free(S);
  free(p);
  return 0;
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int c = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (c >= J->B * J->H) break;
    const size_t T = (size_t)J->T, dk = (size_t)J->dk, dv = (size_t)J->dv;
    const int rc = run_chain(J->q + c * T * dk, J->k + c * T * dk, J->v + c * T * dv,
                             J->g + c * T * dk, J->beta + c * T, J->h0 ? J->h0 + c * dk * dv : NULL,
                             J->o + c * T * dv, J->hT ? J->hT + c * dk * dv : NULL, J->T, J->dk,
                             J->dv, J->scale, J->erase);
    if (rc) {
      pthread_mutex_lock(&J->mu);
      J->failed = 1;
      pthread_mutex_unlock(&J->mu);
    }
  }
  return NULL;
}

/*
 * Run B*H independent chains of length T.  Layouts: q,k,g [B,H,T,dk];
 * v [B,H,T,dv]; beta [B,H,T]; h0 [B,H,dk,dv] or NULL; o [B,H,T,dv];
 * hT [B,H,dk,dv] or NULL.  erase = 0 drops the delta-rule erase term (plain
 * gated linear attention; used only to pin the oracle).  Chains are spread
 * over nthreads POSIX threads.  Returns 0, or -1 on bad arguments / OOM.
 */
int kda_oracle_recurrent(const double *q, const double *k, const double *v, const double *g,
                         const double *beta, const double *h0, double *o, double *hT, int B,
                         int H, int T, int dk, int dv, double scale, int erase, int nthreads) {
  if (!q || !k || !v || !g || !beta || !o || B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1)
    return -1;
  if (B * H == 0) return 0;
  job_t J = {q, k, v, g, beta, h0, o, hT, B, H, T, dk, dv, erase, scale, 0,
             PTHREAD_MUTEX_INITIALIZER, 0};
  if (nthreads < 1) nthreads = 1;
  if (nthreads > B * H) nthreads = B * H;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -1;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
  if (started == 0) worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  return J.failed ? -1 : 0;
}
