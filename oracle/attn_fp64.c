/*
 * Oracle for exact attention, plain fp64 on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load this library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes is the plain definition of attention,
 *     out_i = softmax(scale * q_i . K^T) V ,
 * from "Lesson 8: Context Parallelism", section 1 (the attention formula
 * that every query must see every key).  Blockwise ring attention with the
 * online-softmax merge reaches exactly this value (same lesson, section 3,
 * and "Sequence parallelism and ring attention", FAQ on online softmax), so
 * the oracle is that definition written out, with no blocking, no online
 * rescaling and no chunk order:
 *
 *   for each requested query row (b, h, i):
 *     J    = allowed keys: j < kv_len[b] (when lengths are given) and, when
 *            causal, kpos[j] <= qpos[i] ("Lesson 8", section 4: query i sees
 *            keys j <= i)
 *     s_j  = scale * sum_d q[b,i,h,d] * k[b,j,g,d]      with g = h / (Hq/Hkv)
 *     m    = max_j s_j ,  Z = sum_j exp(s_j - m)
 *     out  = sum_j exp(s_j - m) v[b,j,g,:] / Z ,   lse = m + ln Z
 *
 * The whole score row is materialised before it is normalised.  Inputs are
 * float32 arrays holding the exact values of the device inputs (bf16 values
 * are exact in float32); every operation is done in double.
 *
 * Layouts (row-major, last index fastest):
 *   q   [B, Sq , Hq , D]      k, v [B, Skv, Hkv, D]
 *   qpos[Sq]  (global position of each query row; NULL means the row index)
 *   kpos[Skv] (global position of each key row;   NULL means the row index)
 *   kv_len[B] (keys j >= kv_len[b] are not allowed; NULL means all Skv)
 *   rows [nrows][3] = (b, h, i)
 *   out  [nrows][D]  lse [nrows]
 * A row with no allowed key gets out = 0 and lse = -inf.
 */
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

typedef struct {
  const float *q, *k, *v;
  int B, Sq, Skv, Hq, Hkv, D;
  const int64_t *qpos, *kpos;
  int causal;
  const int64_t *kv_len;
  double scale;
  const int32_t *rows;
  int64_t r0, r1;
  double *out, *lse;
  int err;
} job_t;

static void one_row(const job_t *J, int64_t r, double *s /* [Skv] */) {
  const int b = J->rows[3 * r + 0], h = J->rows[3 * r + 1], i = J->rows[3 * r + 2];
  const int G = J->Hq / J->Hkv;
  const int g = h / G;
  const int D = J->D;
  const float *qi = J->q + (((int64_t)b * J->Sq + i) * J->Hq + h) * D;
  const int64_t qp = J->qpos ? J->qpos[i] : i;
  const int64_t nkeys = J->kv_len ? J->kv_len[b] : J->Skv;
  double *o = J->out + r * D;
  for (int d = 0; d < D; ++d) o[d] = 0.0;

  /* 1. materialise the score row over the allowed keys */
  double m = -INFINITY;
  int any = 0;
  for (int64_t j = 0; j < J->Skv; ++j) {
    const int64_t kp = J->kpos ? J->kpos[j] : j;
    const int allowed = (j < nkeys) && (!J->causal || kp <= qp);
    if (!allowed) { s[j] = -INFINITY; continue; }
    const float *kj = J->k + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += (double)qi[d] * (double)kj[d];
    s[j] = J->scale * acc;
    if (s[j] > m) m = s[j];
    any = 1;
  }
  if (!any) { J->lse[r] = -INFINITY; return; }

  /* 2. exponentiate against the row max and sum */
  double Z = 0.0;
  for (int64_t j = 0; j < J->Skv; ++j) {
    if (s[j] == -INFINITY) { s[j] = 0.0; continue; }
    s[j] = exp(s[j] - m);
    Z += s[j];
  }
  /* 3. weighted sum of the value rows, then normalise */
  for (int64_t j = 0; j < J->Skv; ++j) {
    if (s[j] == 0.0) continue;
    const float *vj = J->v + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
    const double w = s[j];
    for (int d = 0; d < D; ++d) o[d] += w * (double)vj[d];
  }
  for (int d = 0; d < D; ++d) o[d] /= Z;
  J->lse[r] = m + log(Z);
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  double *s = (double *)malloc(sizeof(double) * (size_t)(J->Skv > 0 ? J->Skv : 1));
  if (!s) { J->err = 1; return NULL; }
  for (int64_t r = J->r0; r < J->r1; ++r) one_row(J, r, s);
  free(s);
  return NULL;
}

/* Number of host cores this process may run on. */
int oracle_cores(void) {
  cpu_set_t set;
  if (sched_getaffinity(0, sizeof(set), &set) == 0) return CPU_COUNT(&set);
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

/* Returns 0 on success, nonzero on a bad argument or an allocation failure. */
int oracle_attn_rows(const float *q, const float *k, const float *v,
                     int B, int Sq, int Skv, int Hq, int Hkv, int D,
                     const int64_t *qpos, const int64_t *kpos, int causal,
                     const int64_t *kv_len, double scale,
                     const int32_t *rows, int64_t nrows,
                     double *out, double *lse, int nthreads) {
  if (B <= 0 || Sq <= 0 || Skv < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return 1;
  if (Hq % Hkv != 0) return 1;
  for (int64_t r = 0; r < nrows; ++r) {
    const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= Sq) return 1;
  }
  if (nthreads <= 0) nthreads = oracle_cores();
  if (nthreads > nrows) nthreads = nrows > 0 ? (int)nrows : 1;
  if (nthreads < 1) nthreads = 1;
  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return 2; }
  int err = 0;
  for (int t = 0; t < nthreads; ++t) {
    job_t *J = &jobs[t];
    J->q = q; J->k = k; J->v = v;
    J->B = B; J->Sq = Sq; J->Skv = Skv; J->Hq = Hq; J->Hkv = Hkv; J->D = D;
    J->qpos = qpos; J->kpos = kpos; J->causal = causal; J->kv_len = kv_len;
    J->scale = scale; J->rows = rows;
    J->r0 = nrows * t / nthreads; J->r1 = nrows * (t + 1) / nthreads;
    J->out = out; J->lse = lse;
    if (pthread_create(&th[t], NULL, worker, J) != 0) { J->r1 = J->r0; err = 3; th[t] = 0; }
  }
  for (int t = 0; t < nthreads; ++t) {
    if (th[t]) pthread_join(th[t], NULL);
    if (jobs[t].err) err = 2;
  }
  free(jobs); free(th);
  return err;
}

/*
 * Backward of the same attention: the gradients of L = sum(dout * out) with
 * respect to q, k and v.  The pages give no backward; this is the calculus of
 * the definition above, written out with the whole score row materialised:
 *
 *   for each query row (b, h, i), g = h / (Hq/Hkv), over its allowed keys J:
 *     s_j    = scale * q_i . k_j ,  lse = log sum_j exp(s_j)
 *     p_j    = exp(s_j - lse)                    (the softmax weights)
 *     dp_j   = dout_i . v_j
 *     delta  = sum_j p_j dp_j                    (= dout_i . out_i)
 *     ds_j   = p_j (dp_j - delta)                (derivative through softmax)
 *     dq_i   = scale * sum_j ds_j k_j
 *     dk_j  += scale * ds_j q_i                  (summed over rows and the
 *     dv_j  += p_j dout_i                         query heads of group g)
 *
 * Layouts as above; dout [B, Sq, Hq, D]; dq [B, Sq, Hq, D] and dk, dv
 * [B, Skv, Hkv, D] are double and are overwritten.  Threads split the
 * (b, kv head) pairs, so the dk / dv sums need no locks.
 */
typedef struct {
  const float *q, *k, *v, *dout;
  int B, Sq, Skv, Hq, Hkv, D;
  const int64_t *qpos, *kpos;
  int causal;
  double scale;
  double *dq, *dk, *dv;
  int t, nthreads, err;
} bjob_t;

static void *bwd_worker(void *arg) {
  bjob_t *J = (bjob_t *)arg;
  const int G = J->Hq / J->Hkv, D = J->D;
  double *s = (double *)malloc(sizeof(double) * (size_t)(J->Skv > 0 ? J->Skv : 1));
  double *dp = (double *)malloc(sizeof(double) * (size_t)(J->Skv > 0 ? J->Skv : 1));
  if (!s || !dp) { free(s); free(dp); J->err = 1; return NULL; }
  for (int bg = J->t; bg < J->B * J->Hkv; bg += J->nthreads) {
    const int b = bg / J->Hkv, g = bg % J->Hkv;
    for (int h = g * G; h < (g + 1) * G; ++h) {
      for (int i = 0; i < J->Sq; ++i) {
        const float *qi = J->q + (((int64_t)b * J->Sq + i) * J->Hq + h) * D;
        const float *oi = J->dout + (((int64_t)b * J->Sq + i) * J->Hq + h) * D;
        const int64_t qp = J->qpos ? J->qpos[i] : i;
        double m = -INFINITY;
        for (int j = 0; j < J->Skv; ++j) {
          const int64_t kp = J->kpos ? J->kpos[j] : j;
          if (J->causal && kp > qp) { s[j] = -INFINITY; continue; }
          const float *kj = J->k + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += (double)qi[d] * (double)kj[d];
          s[j] = J->scale * acc;
          if (s[j] > m) m = s[j];
        }
        double *dqi = J->dq + (((int64_t)b * J->Sq + i) * J->Hq + h) * D;
        for (int d = 0; d < D; ++d) dqi[d] = 0.0;
        if (m == -INFINITY) continue;              /* no allowed key: no gradient */
        double Z = 0.0;
        for (int j = 0; j < J->Skv; ++j)
          if (s[j] != -INFINITY) Z += exp(s[j] - m);
        const double lse = m + log(Z);
        double delta = 0.0;
        for (int j = 0; j < J->Skv; ++j) {
          if (s[j] == -INFINITY) { dp[j] = 0.0; continue; }
          const float *vj = J->v + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
          double acc = 0.0;
          for (int d = 0; d < D; ++d) acc += (double)oi[d] * (double)vj[d];
          dp[j] = acc;
          delta += exp(s[j] - lse) * acc;
        }
        for (int j = 0; j < J->Skv; ++j) {
          if (s[j] == -INFINITY) continue;
          const double p = exp(s[j] - lse);
          const double ds = p * (dp[j] - delta);
          const float *kj = J->k + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
          double *dkj = J->dk + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
          double *dvj = J->dv + (((int64_t)b * J->Skv + j) * J->Hkv + g) * D;
          for (int d = 0; d < D; ++d) {
            dqi[d] += J->scale * ds * (double)kj[d];
            dkj[d] += J->scale * ds * (double)qi[d];
            dvj[d] += p * (double)oi[d];
          }
        }
      }
    }
  }
  free(s);
  free(dp);
  return NULL;
}

/* Returns 0 on success, nonzero on a bad argument or an allocation failure. */
int oracle_attn_bwd(const float *q, const float *k, const float *v, const float *dout,
                    int B, int Sq, int Skv, int Hq, int Hkv, int D,
                    const int64_t *qpos, const int64_t *kpos, int causal, double scale,
                    double *dq, double *dk, double *dv, int nthreads) {
  if (B <= 0 || Sq <= 0 || Skv < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return 1;
  for (int64_t e = 0; e < (int64_t)B * Skv * Hkv * D; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
  if (nthreads <= 0) nthreads = oracle_cores();
  if (nthreads > B * Hkv) nthreads = B * Hkv;
  if (nthreads < 1) nthreads = 1;
  bjob_t *jobs = (bjob_t *)calloc((size_t)nthreads, sizeof(bjob_t));
  pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return 2; }
  int err = 0;
  for (int t = 0; t < nthreads; ++t) {
    bjob_t *J = &jobs[t];
    J->q = q; J->k = k; J->v = v; J->dout = dout;
    J->B = B; J->Sq = Sq; J->Skv = Skv; J->Hq = Hq; J->Hkv = Hkv; J->D = D;
    J->qpos = qpos; J->kpos = kpos; J->causal = causal; J->scale = scale;
    J->dq = dq; J->dk = dk; J->dv = dv;
    J->t = t; J->nthreads = nthreads;
    if (pthread_create(&th[t], NULL, bwd_worker, J) != 0) { err = 3; th[t] = 0; }
  }
  for (int t = 0; t < nthreads; ++t) {
    if (th[t]) pthread_join(th[t], NULL);
    if (jobs[t].err) err = 2;
  }
  free(jobs); free(th);
  return err;
}

/*
 * dq of selected query rows only (the same calculus as oracle_attn_bwd, for
 * one row at a time: its scores, lse, dp_j, delta and ds_j need only that
 * row), so large problems can be checked on sampled rows.
 * rows [nrows][3] = (b, h, i); dq [nrows][D] double.
 */
typedef struct {
  const float *q, *k, *v, *dout;
  int B, S, Hq, Hkv, D, causal;
  double scale;
  const int32_t *rows;
  int64_t r0, r1;
  double *dq;
  int err;
} qjob_t;

static void *dq_rows_worker(void *arg) {
  qjob_t *J = (qjob_t *)arg;
  const int G = J->Hq / J->Hkv, D = J->D;
  double *s = (double *)malloc(sizeof(double) * (size_t)J->S);
  double *dp = (double *)malloc(sizeof(double) * (size_t)J->S);
  if (!s || !dp) { free(s); free(dp); J->err = 1; return NULL; }
  for (int64_t r = J->r0; r < J->r1; ++r) {
    const int b = J->rows[3 * r], h = J->rows[3 * r + 1], i = J->rows[3 * r + 2], g = h / G;
    const float *qi = J->q + (((int64_t)b * J->S + i) * J->Hq + h) * D;
    const float *oi = J->dout + (((int64_t)b * J->S + i) * J->Hq + h) * D;
    double *dqi = J->dq + r * D;
    for (int d = 0; d < D; ++d) dqi[d] = 0.0;
    const int nj = J->causal ? i + 1 : J->S;
    double m = -INFINITY;
    for (int j = 0; j < nj; ++j) {
      const float *kj = J->k + (((int64_t)b * J->S + j) * J->Hkv + g) * D;
      const float *vj = J->v + (((int64_t)b * J->S + j) * J->Hkv + g) * D;
      double a = 0.0, c = 0.0;
      for (int d = 0; d < D; ++d) {
        a += (double)qi[d] * (double)kj[d];
        c += (double)oi[d] * (double)vj[d];
      }
      s[j] = J->scale * a;
      dp[j] = c;
      if (s[j] > m) m = s[j];
    }
    if (nj == 0) continue;
    double Z = 0.0;
    for (int j = 0; j < nj; ++j) Z += exp(s[j] - m);
    const double lse = m + log(Z);
    double delta = 0.0;
    for (int j = 0; j < nj; ++j) delta += exp(s[j] - lse) * dp[j];
    for (int j = 0; j < nj; ++j) {
      const double ds = exp(s[j] - lse) * (dp[j] - delta);
      const float *kj = J->k + (((int64_t)b * J->S + j) * J->Hkv + g) * D;
      for (int d = 0; d < D; ++d) dqi[d] += J->scale * ds * (double)kj[d];
    }
  }
  free(s);
  free(dp);
  return NULL;
}

int oracle_attn_bwd_dq_rows(const float *q, const float *k, const float *v, const float *dout,
                            int B, int S, int Hq, int Hkv, int D, int causal, double scale,
                            const int32_t *rows, int64_t nrows, double *dq, int nthreads) {
  if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return 1;
  for (int64_t r = 0; r < nrows; ++r) {
    const int b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
    if (b < 0 || b >= B || h < 0 || h >= Hq || i < 0 || i >= S) return 1;
  }
  if (nthreads <= 0) nthreads = oracle_cores();
  if (nthreads > nrows) nthreads = nrows > 0 ? (int)nrows : 1;
  if (nthreads < 1) nthreads = 1;
  qjob_t *jobs = (qjob_t *)calloc((size_t)nthreads, sizeof(qjob_t));
  pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !th) { free(jobs); free(th); return 2; }
  int err = 0;
  for (int t = 0; t < nthreads; ++t) {
    qjob_t *J = &jobs[t];
    J->q = q; J->k = k; J->v = v; J->dout = dout;
    J->B = B; J->S = S; J->Hq = Hq; J->Hkv = Hkv; J->D = D; J->causal = causal; J->scale = scale;
    J->rows = rows; J->r0 = nrows * t / nthreads; J->r1 = nrows * (t + 1) / nthreads; J->dq = dq;
    if (pthread_create(&th[t], NULL, dq_rows_worker, J) != 0) { err = 3; th[t] = 0; }
  }
  for (int t = 0; t < nthreads; ++t) {
    if (th[t]) pthread_join(th[t], NULL);
    if (jobs[t].err) err = 2;
  }
  free(jobs); free(th);
  return err;
}
