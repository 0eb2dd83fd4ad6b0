/*
 * attn_oracle.c -- plain fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (the plain definition, no blocking, no fusion):
 *   O = softmax(Q K^T * scale) V, row by row, in fp64.
 *     - Qiita "Flash Attention" tutorial, section 2.2 (Self-Attention):
 *       Attention(Q,K,V) = softmax(Q K^T / sqrt(d)) V.
 *     - hysenlabs "FlashAttention: GPU-specific backends and the attention API",
 *       section on outputs/operations: the functions compute
 *       softmax(Q @ K^T * softmax_scale) @ V, options causal / window_size,
 *       and MQA/GQA when the number of Q heads is divisible by the number of
 *       KV heads.
 *     - same page, section on constraints/changelog: since v2.1 the causal
 *       mask is aligned to the bottom-right corner when Nq != Nk.
 *   Softmax is the two-pass form: row max m, l = sum exp(S - m),
 *   P = exp(S - m) / l.  LSE_i = m_i + ln(l_i) (natural log, scale included).
 *
 *   Backward (the calculus of the loss L = sum(dO * O); no page prints these
 *   formulas, abeam.tech FlashAttention summary, "backward uses recomputation",
 *   only says P is recomputed from saved statistics):
 *     D_i   = sum_c dO_ic O_ic
 *     dP_ij = dO_i . V_j
 *     dS_ij = P_ij (dP_ij - D_i)
 *     dQ_i  = scale * sum_j dS_ij K_j
 *     dK_j  = scale * sum_i dS_ij Q_i     (summed over the Q heads of a KV group)
 *     dV_j  = sum_i P_ij dO_i             (summed over the Q heads of a KV group)
 *
 *   Blockwise recurrence (oracle_attn_fwd_blockwise): the online softmax of the
 *   Qiita tutorial, section 4.3 (running max and running sum rescaled by
 *   exp(old max - new max)), with the output accumulator rescaled by the same
 *   factor as the abeam.tech summary describes ("computing softmax blockwise
 *   correctly": the output vector is rescaled and accumulated).  It exists only
 *   so the tests can show the recurrence equals the two-pass definition.
 *
 * Readings where the pages are silent:
 *   - layout: Q,O,dO,dQ [B,Nq,Hq,d]; K,V,dK,dV [B,Nk,Hkv,d]; LSE [B,Hq,Nq];
 *     d contiguous.
 *   - visibility: with delta = Nk - Nq, key j is visible to query i iff
 *       (wr < 0 || j <= i + delta + wr) && (wl < 0 || j >= i + delta - wl),
 *     wr = 0 when causal; bounds inclusive; negative = unbounded.
 *   - a row with no visible key has O = 0, LSE = -inf and zero gradients.
 *   - GQA head mapping: kv head = q head / (Hq / Hkv).
 *
 * Threads: rows are split over plain pthreads; dK/dV are accumulated in
 * per-thread buffers and summed in thread order, so results are reproducible.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  long B, Nq, Nk, Hq, Hkv, d;
  double scale;
  long wl, wr; /* effective window bounds, negative = unbounded */
} oshape;

static void make_shape(oshape* s, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                       double scale, int causal, int win_l, int win_r) {
  s->B = B; s->Nq = Nq; s->Nk = Nk; s->Hq = Hq; s->Hkv = Hkv; s->d = d;
  s->scale = scale;
  s->wl = win_l < 0 ? -1 : win_l;
  s->wr = causal ? 0 : (win_r < 0 ? -1 : win_r);
}

static int bad_shape(int B, int Nq, int Nk, int Hq, int Hkv, int d) {
  if (B < 1 || Nq < 1 || Nk < 1 || Hq < 1 || Hkv < 1 || d < 1) return 1;
  if (Hq % Hkv != 0) return 1;
  return 0;
}

static int visible(const oshape* s, long i, long j) {
  long delta = s->Nk - s->Nq;
  if (s->wr >= 0 && j > i + delta + s->wr) return 0;
  if (s->wl >= 0 && j < i + delta - s->wl) return 0;
  return 1;
}

static const double* qrow(const oshape* s, const double* q, long b, long i, long h) {
  return q + ((b * s->Nq + i) * s->Hq + h) * s->d;
}
static const double* krow(const oshape* s, const double* k, long b, long j, long hk) {
  return k + ((b * s->Nk + j) * s->Hkv + hk) * s->d;
}

/* S row, two-pass softmax.  Fills p[j] (normalised, 0 where masked) and
 * returns LSE; returns -inf (and p = 0) when nothing is visible. */
static double softmax_row(const oshape* s, const double* q, const double* k,
                          long b, long h, long i, double* p) {
  long hk = h / (s->Hq / s->Hkv);
  const double* qi = qrow(s, q, b, i, h);
  double m = -INFINITY;
  for (long j = 0; j < s->Nk; ++j) {
    if (!visible(s, i, j)) { p[j] = -INFINITY; continue; }
    const double* kj = krow(s, k, b, j, hk);
    double acc = 0.0;
    for (long c = 0; c < s->d; ++c) acc += qi[c] * kj[c];
    p[j] = acc * s->scale;
    if (p[j] > m) m = p[j];
  }
  if (m == -INFINITY) {
    for (long j = 0; j < s->Nk; ++j) p[j] = 0.0;
    return -INFINITY;
  }
  double l = 0.0;
  for (long j = 0; j < s->Nk; ++j) {
    p[j] = (p[j] == -INFINITY) ? 0.0 : exp(p[j] - m);
    l += p[j];
  }
  for (long j = 0; j < s->Nk; ++j) p[j] /= l;
  return m + log(l);
}

/* ------------------------------------------------------------------ forward */

typedef struct {
  const oshape* s;
  const double *q, *k, *v;
  double *o, *lse;
  long row_begin, row_end; /* flattened (b, h, i) rows */
  long block_n;            /* 0 = two-pass definition, >0 = blockwise recurrence */
} fwd_task;

static void fwd_row_twopass(const oshape* s, const double* q, const double* k,
                            const double* v, double* o, double* lse, long b,
                            long h, long i, double* p) {
  long hk = h / (s->Hq / s->Hkv);
  double L = softmax_row(s, q, k, b, h, i, p);
  double* oi = o + ((b * s->Nq + i) * s->Hq + h) * s->d;
  for (long c = 0; c < s->d; ++c) oi[c] = 0.0;
  for (long j = 0; j < s->Nk; ++j) {
    if (p[j] == 0.0) continue;
    const double* vj = krow(s, v, b, j, hk);
    for (long c = 0; c < s->d; ++c) oi[c] += p[j] * vj[c];
  }
  lse[(b * s->Hq + h) * s->Nq + i] = L;
}

/* Online softmax over key blocks of size bn: running max m, running sum l and
 * an output accumulator, all rescaled by exp(m_old - m_new) when a block
 * raises the max; the division by l happens once at the end. */
static void fwd_row_blockwise(const oshape* s, const double* q, const double* k,
                              const double* v, double* o, double* lse, long b,
                              long h, long i, long bn, double* sblk) {
  long hk = h / (s->Hq / s->Hkv);
  const double* qi = qrow(s, q, b, i, h);
  double* oi = o + ((b * s->Nq + i) * s->Hq + h) * s->d;
  double m = -INFINITY, l = 0.0;
  for (long c = 0; c < s->d; ++c) oi[c] = 0.0;
  for (long j0 = 0; j0 < s->Nk; j0 += bn) {
    long j1 = j0 + bn < s->Nk ? j0 + bn : s->Nk;
    double bmax = -INFINITY;
    for (long j = j0; j < j1; ++j) {
      double x = -INFINITY;
      if (visible(s, i, j)) {
        const double* kj = krow(s, k, b, j, hk);
        double acc = 0.0;
        for (long c = 0; c < s->d; ++c) acc += qi[c] * kj[c];
        x = acc * s->scale;
      }
      sblk[j - j0] = x;
      if (x > bmax) bmax = x;
    }
    double m_new = m > bmax ? m : bmax;
    if (m_new == -INFINITY) continue; /* nothing visible yet */
    double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
    l *= alpha;
    for (long c = 0; c < s->d; ++c) oi[c] *= alpha;
    for (long j = j0; j < j1; ++j) {
      if (sblk[j - j0] == -INFINITY) continue;
      double pj = exp(sblk[j - j0] - m_new);
      l += pj;
      const double* vj = krow(s, v, b, j, hk);
      for (long c = 0; c < s->d; ++c) oi[c] += pj * vj[c];
    }
    m = m_new;
  }
  if (m == -INFINITY) {
    lse[(b * s->Hq + h) * s->Nq + i] = -INFINITY;
    return;
  }
  for (long c = 0; c < s->d; ++c) oi[c] /= l;
  lse[(b * s->Hq + h) * s->Nq + i] = m + log(l);
}

static void* fwd_worker(void* arg) {
  fwd_task* t = (fwd_task*)arg;
  const oshape* s = t->s;
  long buflen = t->block_n > 0 ? t->block_n : s->Nk;
  double* buf = (double*)malloc(sizeof(double) * (size_t)buflen);
  if (!buf) return (void*)1;
  for (long r = t->row_begin; r < t->row_end; ++r) {
    long i = r % s->Nq;
    long h = (r / s->Nq) % s->Hq;
    long b = r / (s->Nq * s->Hq);
    if (t->block_n > 0)
      fwd_row_blockwise(s, t->q, t->k, t->v, t->o, t->lse, b, h, i, t->block_n, buf);
    else
      fwd_row_twopass(s, t->q, t->k, t->v, t->o, t->lse, b, h, i, buf);
  }
  free(buf);
  return NULL;
}

static int run_fwd(const double* q, const double* k, const double* v, double* o,
                   double* lse, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                   double scale, int causal, int win_l, int win_r, int nthreads,
                   long block_n) {
  if (bad_shape(B, Nq, Nk, Hq, Hkv, d)) return 1;
  if (!q || !k || !v || !o || !lse) return 1;
  oshape s;
  make_shape(&s, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r);
  long rows = s.B * s.Hq * s.Nq;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > rows) nthreads = (int)rows;
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  fwd_task* tk = (fwd_task*)malloc(sizeof(fwd_task) * (size_t)nthreads);
  if (!th || !tk) { free(th); free(tk); return 2; }
  int rc = 0;
  for (int t = 0; t < nthreads; ++t) {
    tk[t].s = &s; tk[t].q = q; tk[t].k = k; tk[t].v = v; tk[t].o = o; tk[t].lse = lse;
    tk[t].row_begin = rows * t / nthreads;
    tk[t].row_end = rows * (t + 1) / nthreads;
    tk[t].block_n = block_n;
    pthread_create(&th[t], NULL, fwd_worker, &tk[t]);
  }
  for (int t = 0; t < nthreads; ++t) {
    void* ret = NULL;
    pthread_join(th[t], &ret);
    if (ret) rc = 2;
  }
  free(th); free(tk);
  return rc;
}

int oracle_attn_fwd(const double* q, const double* k, const double* v, double* o,
                    double* lse, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                    double scale, int causal, int win_l, int win_r, int nthreads) {
  return run_fwd(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l,
                 win_r, nthreads, 0);
}

int oracle_attn_fwd_blockwise(const double* q, const double* k, const double* v,
                              double* o, double* lse, int B, int Nq, int Nk, int Hq,
                              int Hkv, int d, double scale, int causal, int win_l,
                              int win_r, int block_n, int nthreads) {
  if (block_n < 1) return 1;
  return run_fwd(q, k, v, o, lse, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l,
                 win_r, nthreads, block_n);
}

/* ----------------------------------------------------------------- backward */

typedef struct {
  const oshape* s;
  const double *q, *k, *v, *dout;
  double* dq;
  double *dk_part, *dv_part; /* this thread's [Nk, d] slice for the current (b, hkv) */
  long b, hk;
  long row_begin, row_end;   /* flattened (h in group, i) rows of the group */
  int failed;
} bwd_task;

static void* bwd_worker(void* arg) {
  bwd_task* t = (bwd_task*)arg;
  const oshape* s = t->s;
  long G = s->Hq / s->Hkv;
  double* p = (double*)malloc(sizeof(double) * (size_t)s->Nk);
  double* orow = (double*)malloc(sizeof(double) * (size_t)s->d);
  if (!p || !orow) { free(p); free(orow); t->failed = 1; return NULL; }
  for (long r = t->row_begin; r < t->row_end; ++r) {
    long i = r % s->Nq;
    long h = t->hk * G + r / s->Nq;
    const double* qi = qrow(s, t->q, t->b, i, h);
    const double* doi = qrow(s, t->dout, t->b, i, h);
    double* dqi = t->dq + ((t->b * s->Nq + i) * s->Hq + h) * s->d;
    for (long c = 0; c < s->d; ++c) dqi[c] = 0.0;
    double L = softmax_row(s, t->q, t->k, t->b, h, i, p);
    if (L == -INFINITY) continue;
    /* O_i = sum_j P_ij V_j, then D_i = dO_i . O_i */
    for (long c = 0; c < s->d; ++c) orow[c] = 0.0;
    for (long j = 0; j < s->Nk; ++j) {
      if (p[j] == 0.0) continue;
      const double* vj = krow(s, t->v, t->b, j, t->hk);
      for (long c = 0; c < s->d; ++c) orow[c] += p[j] * vj[c];
    }
    double D = 0.0;
    for (long c = 0; c < s->d; ++c) D += doi[c] * orow[c];
    for (long j = 0; j < s->Nk; ++j) {
      if (p[j] == 0.0) continue;
      const double* vj = krow(s, t->v, t->b, j, t->hk);
      const double* kj = krow(s, t->k, t->b, j, t->hk);
      double dP = 0.0;
      for (long c = 0; c < s->d; ++c) dP += doi[c] * vj[c];
      double dS = p[j] * (dP - D);
      double* dkj = t->dk_part + j * s->d;
      double* dvj = t->dv_part + j * s->d;
      for (long c = 0; c < s->d; ++c) {
        dqi[c] += s->scale * dS * kj[c];
        dkj[c] += s->scale * dS * qi[c];
        dvj[c] += p[j] * doi[c];
      }
    }
  }
  free(p); free(orow);
  return NULL;
}

int oracle_attn_bwd(const double* q, const double* k, const double* v,
                    const double* dout, double* dq, double* dk, double* dv, int B,
                    int Nq, int Nk, int Hq, int Hkv, int d, double scale, int causal,
                    int win_l, int win_r, int nthreads) {
  if (bad_shape(B, Nq, Nk, Hq, Hkv, d)) return 1;
  if (!q || !k || !v || !dout || !dq || !dk || !dv) return 1;
  oshape s;
  make_shape(&s, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r);
  long G = s.Hq / s.Hkv;
  long rows = G * s.Nq; /* rows per (b, hkv) group */
  if (nthreads < 1) nthreads = 1;
  if (nthreads > rows) nthreads = (int)rows;
  size_t slice = (size_t)s.Nk * (size_t)s.d;
  double* parts = (double*)malloc(sizeof(double) * slice * 2 * (size_t)nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  bwd_task* tk = (bwd_task*)malloc(sizeof(bwd_task) * (size_t)nthreads);
  if (!parts || !th || !tk) { free(parts); free(th); free(tk); return 2; }
  int rc = 0;
  for (long b = 0; b < s.B && rc == 0; ++b) {
    for (long hk = 0; hk < s.Hkv && rc == 0; ++hk) {
      memset(parts, 0, sizeof(double) * slice * 2 * (size_t)nthreads);
      for (int t = 0; t < nthreads; ++t) {
        tk[t].s = &s; tk[t].q = q; tk[t].k = k; tk[t].v = v; tk[t].dout = dout;
        tk[t].dq = dq;
        tk[t].dk_part = parts + slice * 2 * (size_t)t;
        tk[t].dv_part = parts + slice * (2 * (size_t)t + 1);
        tk[t].b = b; tk[t].hk = hk;
        tk[t].row_begin = rows * t / nthreads;
        tk[t].row_end = rows * (t + 1) / nthreads;
        tk[t].failed = 0;
        pthread_create(&th[t], NULL, bwd_worker, &tk[t]);
      }
      for (int t = 0; t < nthreads; ++t) {
        pthread_join(th[t], NULL);
        if (tk[t].failed) rc = 2;
      }
      /* sum the per-thread slices in thread order */
      for (long j = 0; j < s.Nk; ++j) {
        double* dkj = dk + ((b * s.Nk + j) * s.Hkv + hk) * s.d;
        double* dvj = dv + ((b * s.Nk + j) * s.Hkv + hk) * s.d;
        for (long c = 0; c < s.d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
        for (int t = 0; t < nthreads; ++t) {
          const double* pk = parts + slice * 2 * (size_t)t + j * s.d;
          const double* pv = parts + slice * (2 * (size_t)t + 1) + j * s.d;
          for (long c = 0; c < s.d; ++c) { dkj[c] += pk[c]; dvj[c] += pv[c]; }
        }
      }
    }
  }
  free(parts); free(th); free(tk);
  return rc;
}

/* ------------------------------------------------------ selected rows only */
/*
 * The same row-by-row definition as above, evaluated only for a list of
 * absolute query rows (O, LSE, dQ) or key rows (dK, dV), so large problems can
 * be checked on a sample.  Each selected row is computed exactly as in the
 * full functions (same code path, same order), so a selected row equals the
 * full function's row bit for bit.
 *   o_rows  [B, nq, Hq, d], lse_rows [B, Hq, nq], dq_rows [B, nq, Hq, d]
 *   dk_rows [B, nk, Hkv, d], dv_rows [B, nk, Hkv, d]
 */
typedef struct {
  const oshape* s;
  const double *q, *k, *v, *dout;
  const int* qrows; int nq;
  const int* krows; int nk;
  double *o_rows, *lse_rows, *dq_rows;
  double *dk_part, *dv_part; /* this thread's [B, nk, Hkv, d] accumulators */
  long task_begin, task_end; /* flattened (b, h, i) over all Nq query rows */
  int mode;                  /* 0: fwd rows, 1: dq rows, 2: dk/dv rows */
  int failed;
} rows_task;

static void* rows_worker(void* arg) {
  rows_task* t = (rows_task*)arg;
  const oshape* s = t->s;
  double* p = (double*)malloc(sizeof(double) * (size_t)s->Nk);
  double* orow = (double*)malloc(sizeof(double) * (size_t)s->d);
  if (!p || !orow) { free(p); free(orow); t->failed = 1; return NULL; }
  for (long task = t->task_begin; task < t->task_end; ++task) {
    long b, h, i, r = -1;
    if (t->mode == 2) {
      /* every query row (b, h, i) contributes to the selected key rows */
      i = task % s->Nq; h = (task / s->Nq) % s->Hq; b = task / (s->Nq * s->Hq);
    } else {
      r = task % t->nq; h = (task / t->nq) % s->Hq; b = task / (t->nq * s->Hq);
      i = t->qrows[r];
    }
    long hk = h / (s->Hq / s->Hkv);
    if (t->mode == 0) {
      double L = softmax_row(s, t->q, t->k, b, h, i, p);
      double* oi = t->o_rows + ((b * t->nq + r) * s->Hq + h) * s->d;
      for (long c = 0; c < s->d; ++c) oi[c] = 0.0;
      for (long j = 0; j < s->Nk; ++j) {
        if (p[j] == 0.0) continue;
        const double* vj = krow(s, t->v, b, j, hk);
        for (long c = 0; c < s->d; ++c) oi[c] += p[j] * vj[c];
      }
      t->lse_rows[(b * s->Hq + h) * t->nq + r] = L;
      continue;
    }
    const double* qi = qrow(s, t->q, b, i, h);
    const double* doi = qrow(s, t->dout, b, i, h);
    if (t->mode == 2) {
      /* skip query rows that see none of the selected keys */
      int any = 0;
      for (int kk = 0; kk < t->nk && !any; ++kk) any = visible(s, i, t->krows[kk]);
      if (!any) continue;
    }
    double L = softmax_row(s, t->q, t->k, b, h, i, p);
    double* dqi = (t->mode == 1) ? t->dq_rows + ((b * t->nq + r) * s->Hq + h) * s->d : NULL;
    if (dqi) for (long c = 0; c < s->d; ++c) dqi[c] = 0.0;
    if (L == -INFINITY) continue;
    for (long c = 0; c < s->d; ++c) orow[c] = 0.0;
    for (long j = 0; j < s->Nk; ++j) {
      if (p[j] == 0.0) continue;
      const double* vj = krow(s, t->v, b, j, hk);
      for (long c = 0; c < s->d; ++c) orow[c] += p[j] * vj[c];
    }
    double D = 0.0;
    for (long c = 0; c < s->d; ++c) D += doi[c] * orow[c];
    if (t->mode == 1) {
      for (long j = 0; j < s->Nk; ++j) {
        if (p[j] == 0.0) continue;
        const double* vj = krow(s, t->v, b, j, hk);
        const double* kj = krow(s, t->k, b, j, hk);
        double dP = 0.0;
        for (long c = 0; c < s->d; ++c) dP += doi[c] * vj[c];
        double dS = p[j] * (dP - D);
        for (long c = 0; c < s->d; ++c) dqi[c] += s->scale * dS * kj[c];
      }
    } else {
      for (int kk = 0; kk < t->nk; ++kk) {
        long j = t->krows[kk];
        if (p[j] == 0.0) continue;
        const double* vj = krow(s, t->v, b, j, hk);
        double dP = 0.0;
        for (long c = 0; c < s->d; ++c) dP += doi[c] * vj[c];
        double dS = p[j] * (dP - D);
        double* dkj = t->dk_part + ((b * t->nk + kk) * s->Hkv + hk) * s->d;
        double* dvj = t->dv_part + ((b * t->nk + kk) * s->Hkv + hk) * s->d;
        for (long c = 0; c < s->d; ++c) {
          dkj[c] += s->scale * dS * qi[c];
          dvj[c] += p[j] * doi[c];
        }
      }
    }
  }
  free(p); free(orow);
  return NULL;
}

static int run_rows(const double* q, const double* k, const double* v, const double* dout,
                    double* o_rows, double* lse_rows, double* dq_rows, double* dk_rows,
                    double* dv_rows, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                    double scale, int causal, int win_l, int win_r, const int* qrows,
                    int nq, const int* krows, int nk, int mode, int nthreads) {
  if (bad_shape(B, Nq, Nk, Hq, Hkv, d)) return 1;
  oshape s;
  make_shape(&s, B, Nq, Nk, Hq, Hkv, d, scale, causal, win_l, win_r);
  for (int r = 0; r < nq; ++r) if (qrows[r] < 0 || qrows[r] >= Nq) return 1;
  for (int r = 0; r < nk; ++r) if (krows[r] < 0 || krows[r] >= Nk) return 1;
  long tasks = (mode == 2) ? s.B * s.Hq * s.Nq : s.B * s.Hq * (long)nq;
  if (tasks == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > tasks) nthreads = (int)tasks;
  size_t kslice = (size_t)B * (size_t)nk * (size_t)Hkv * (size_t)d;
  double* parts = NULL;
  if (mode == 2) {
    parts = (double*)calloc(kslice * 2 * (size_t)nthreads + 1, sizeof(double));
    if (!parts) return 2;
  }
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  rows_task* tk = (rows_task*)malloc(sizeof(rows_task) * (size_t)nthreads);
  if (!th || !tk) { free(th); free(tk); free(parts); return 2; }
  for (int t = 0; t < nthreads; ++t) {
    rows_task* x = &tk[t];
    x->s = &s; x->q = q; x->k = k; x->v = v; x->dout = dout;
    x->qrows = qrows; x->nq = nq; x->krows = krows; x->nk = nk;
    x->o_rows = o_rows; x->lse_rows = lse_rows; x->dq_rows = dq_rows;
    x->dk_part = parts ? parts + kslice * 2 * (size_t)t : NULL;
    x->dv_part = parts ? parts + kslice * (2 * (size_t)t + 1) : NULL;
    x->task_begin = tasks * t / nthreads;
    x->task_end = tasks * (t + 1) / nthreads;
    x->mode = mode; x->failed = 0;
    pthread_create(&th[t], NULL, rows_worker, x);
  }
  int rc = 0;
  for (int t = 0; t < nthreads; ++t) {
    pthread_join(th[t], NULL);
    if (tk[t].failed) rc = 2;
  }
  if (mode == 2 && rc == 0) {
    for (size_t e = 0; e < kslice; ++e) { dk_rows[e] = 0.0; dv_rows[e] = 0.0; }
    for (int t = 0; t < nthreads; ++t)
      for (size_t e = 0; e < kslice; ++e) {
        dk_rows[e] += parts[kslice * 2 * (size_t)t + e];
        dv_rows[e] += parts[kslice * (2 * (size_t)t + 1) + e];
      }
  }
  free(th); free(tk); free(parts);
  return rc;
}

int oracle_attn_fwd_rows(const double* q, const double* k, const double* v, double* o_rows,
                         double* lse_rows, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                         double scale, int causal, int win_l, int win_r, const int* rows,
                         int nrows, int nthreads) {
  if (!q || !k || !v || !o_rows || !lse_rows || !rows) return 1;
  return run_rows(q, k, v, NULL, o_rows, lse_rows, NULL, NULL, NULL, B, Nq, Nk, Hq, Hkv, d,
                  scale, causal, win_l, win_r, rows, nrows, NULL, 0, 0, nthreads);
}

int oracle_attn_dq_rows(const double* q, const double* k, const double* v, const double* dout,
                        double* dq_rows, int B, int Nq, int Nk, int Hq, int Hkv, int d,
                        double scale, int causal, int win_l, int win_r, const int* rows,
                        int nrows, int nthreads) {
  if (!q || !k || !v || !dout || !dq_rows || !rows) return 1;
  return run_rows(q, k, v, dout, NULL, NULL, dq_rows, NULL, NULL, B, Nq, Nk, Hq, Hkv, d,
                  scale, causal, win_l, win_r, rows, nrows, NULL, 0, 1, nthreads);
}

int oracle_attn_dkdv_rows(const double* q, const double* k, const double* v, const double* dout,
                          double* dk_rows, double* dv_rows, int B, int Nq, int Nk, int Hq,
                          int Hkv, int d, double scale, int causal, int win_l, int win_r,
                          const int* krows, int nkrows, int nthreads) {
  if (!q || !k || !v || !dout || !dk_rows || !dv_rows || !krows) return 1;
  return run_rows(q, k, v, dout, NULL, NULL, NULL, dk_rows, dv_rows, B, Nq, Nk, Hq, Hkv, d,
                  scale, causal, win_l, win_r, NULL, 0, krows, nkrows, 2, nthreads);
}
