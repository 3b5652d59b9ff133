/*
 * attn_oracle.c — TEST INFRASTRUCTURE ONLY. The plain, slow fp64 CPU oracle for
 * exact attention. Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may call it; the library's CUDA path never does.
 *
 * What it computes is the definition of standard attention, which the IO-aware
 * method reproduces exactly up to rounding order:
 *   - "Flash Attention" glossary page, first paragraph: the result is the same as
 *     standard attention; second paragraph: standard attention forms the full
 *     N x N score matrix, the IO-aware method never writes it out.
 *   - "FlashAttention-3 (PT)", section "O problema do mecanismo de atenção": the
 *     self-attention that is quadratic in sequence length.
 *
 * For one query row i of head (b, h), with Nq query rows and Nk keys per head:
 *   allowed(i) = { j : lo <= j < min(Nk, hi) and (not causal or j <= i + Nk - Nq) }
 *   z_j  = scale * sum_c q[i][c] * k[j][c]                    (fp64)
 *   m    = max_{j in allowed} z_j
 *   l    = sum_{j in allowed} exp(z_j - m)
 *   O[c] = sum_{j in allowed} exp(z_j - m) * v[j][c] / l
 *   LSE  = m + ln(l)                                           (natural log)
 * The causal rule and the natural-log LSE are readings: the pages state neither.
 * Key j is visible to query i iff j <= i + (Nk - Nq): the queries are the last Nq
 * positions of the key sequence. For Nq = Nk this is the square, top-left
 * aligned mask j <= i.
 *
 * The key range [lo, hi) restricts attention to a slice of the keys: the
 * partial result over one block of keys that the online softmax of the
 * "Flash Attention" glossary page (second paragraph) accumulates, here produced
 * on its own. A row with no allowed key gets O = 0 and LSE = -inf (the empty
 * sum). lo = 0, hi = Nk is ordinary attention.
 *
 * Layout: q is contiguous [B][H][Nq][d] fp64, k and v [B][H][Nk][d]; o is
 * [rows][d] and lse is [rows], where the row list holds flat ids
 * r = (b*H + h)*Nq + i (NULL = every row in order). Work is split over rows
 * across `nthreads` POSIX threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

typedef struct {
  const double *q, *k, *v;
  int Nq, Nk, d, causal, lo, hi;
  double scale;
  const int64_t* rows;
  int64_t row_begin, row_end;
  double *o, *lse;
  int status;
} oracle_job;

static void attend_one_row(const oracle_job* jb, int64_t out_idx, int64_t flat, double* z) {
  const int Nq = jb->Nq, Nk = jb->Nk, d = jb->d;
  const int64_t bh = flat / Nq;
  const int i = (int)(flat % Nq);
  const double* qi = jb->q + flat * d;
  const double* kh = jb->k + bh * (int64_t)Nk * d;
  const double* vh = jb->v + bh * (int64_t)Nk * d;
  /* allowed keys are first..last */
  const int first = jb->lo;
  int last = (jb->hi < Nk ? jb->hi : Nk) - 1;
  if (jb->causal && i + (Nk - Nq) < last) last = i + (Nk - Nq);
  double* oi = jb->o + out_idx * d;
  if (last < first) {
    for (int c = 0; c < d; ++c) oi[c] = 0.0;
    jb->lse[out_idx] = -INFINITY;
    return;
  }

  double m = -INFINITY;
  for (int j = first; j <= last; ++j) {
    const double* kj = kh + (int64_t)j * d;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];
    z[j] = jb->scale * dot;
    if (z[j] > m) m = z[j];
  }
  double l = 0.0;
  for (int j = first; j <= last; ++j) {
    z[j] = exp(z[j] - m); /* z now holds the unnormalised weights */
    l += z[j];
  }
  for (int c = 0; c < d; ++c) oi[c] = 0.0;
  for (int j = first; j <= last; ++j) {
    const double* vj = vh + (int64_t)j * d;
    for (int c = 0; c < d; ++c) oi[c] += z[j] * vj[c];
  }
  for (int c = 0; c < d; ++c) oi[c] /= l;
  jb->lse[out_idx] = m + log(l);
}

static void* run_job(void* arg) {
  oracle_job* jb = (oracle_job*)arg;
  double* z = (double*)malloc(sizeof(double) * (size_t)jb->Nk);
  if (z == NULL) {
    jb->status = 1;
    return NULL;
  }
  for (int64_t r = jb->row_begin; r < jb->row_end; ++r) {
    const int64_t flat = jb->rows ? jb->rows[r] : r;
    attend_one_row(jb, r, flat, z);
  }
  free(z);
  jb->status = 0;
  return NULL;
}

/* Returns 0 on success, 1 on bad arguments, 2 on allocation/thread failure. */
int oracle_attn_range_rows(const double* q, const double* k, const double* v, int B, int H, int Nq, int Nk,
                           int d, int causal, double scale, int lo, int hi, const int64_t* rows, int64_t nrows,
                           double* o, double* lse, int nthreads) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || lo < 0 || hi < lo || !q || !k || !v || !o || !lse) return 1;
  const int64_t total = (int64_t)B * H * Nq;
  if (rows == NULL) nrows = total;
  for (int64_t r = 0; rows && r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= total) return 1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);

  oracle_job* jobs = (oracle_job*)calloc((size_t)nthreads, sizeof(oracle_job));
  pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return 2;
  }
  int rc = 0;
  int started = 0;
  for (int t = 0; t < nthreads; ++t) {
    oracle_job* jb = &jobs[t];
    jb->q = q; jb->k = k; jb->v = v;
    jb->Nq = Nq; jb->Nk = Nk; jb->d = d; jb->causal = causal; jb->scale = scale;
    jb->lo = lo; jb->hi = hi;
    jb->rows = rows;
    jb->row_begin = nrows * t / nthreads;
    jb->row_end = nrows * (t + 1) / nthreads;
    jb->o = o; jb->lse = lse;
    jb->status = 2;
    if (pthread_create(&tids[t], NULL, run_job, jb) != 0) {
      rc = 2;
      break;
    }
    ++started;
  }
  for (int t = 0; t < started; ++t) {
    pthread_join(tids[t], NULL);
    if (jobs[t].status != 0) rc = 2;
  }
  free(jobs);
  free(tids);
  return rc;
}

/* Square attention (Nq = Nk = N) over every key. */
int oracle_attn_rows(const double* q, const double* k, const double* v, int B, int H, int N, int d,
                     int causal, double scale, const int64_t* rows, int64_t nrows, double* o, double* lse,
                     int nthreads) {
  return oracle_attn_range_rows(q, k, v, B, H, N, N, d, causal, scale, 0, N, rows, nrows, o, lse, nthreads);
}
