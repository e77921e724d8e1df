/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact attention forward.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * bench's CPU-baseline leg, never by the product library.  No tiling, fusion
 * or reordering beyond what each function's comment states, so that it can be
 * checked against the pages by eye.  Page legend and layouts: attn_oracle.h.
 *
 * Readings taken where the pages are silent (restated in the design notes):
 *   - causal means key j <= query i, diagonal included, queries and keys
 *     aligned (no page defines it; the masked-scores form of [MHA-CUDA 2.2]
 *     is applied to the lower triangle);
 *   - the window is the band |i - j| <= w of [LONGSEQ 2.1], applied as an
 *     additive -inf mask as in [MHA-CUDA 2.2] (the page multiplies its 0/1
 *     band into the scores, which would leave masked keys with weight e^0);
 *   - the scale is a caller argument, 1/sqrt(d) in the pages' formula;
 *   - LSE is the natural-log log-sum-exp of the scaled logits over the allowed
 *     keys; a row with no allowed key (impossible for the three masks, which
 *     always allow the diagonal) gets out = 0 and LSE = -inf.
 */
#include "attn_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* Mask predicate: may query i attend to key j?  [MHA-CUDA 2.2], [LONGSEQ 2.1] */
static int allowed(int64_t i, int64_t j, int mask_kind, int64_t window) {
  if (mask_kind == ORACLE_MASK_CAUSAL) return j <= i;
  if (mask_kind == ORACLE_MASK_WINDOW) return (i - j <= window) && (j - i <= window);
  if (mask_kind == ORACLE_MASK_CAUSAL_WINDOW) return (j <= i) && (i - j <= window);
  return 1;
}

static int check_args(const float* q, const float* k, const float* v,
                      const void* out, const void* lse, int64_t B, int64_t H,
                      int64_t L, int64_t d, int mask_kind, int64_t window) {
  if (!q || !k || !v || !out || !lse) return -1;
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return -1;
  if (mask_kind < ORACLE_MASK_NONE || mask_kind > ORACLE_MASK_CAUSAL_WINDOW) return -1;
  if ((mask_kind == ORACLE_MASK_WINDOW || mask_kind == ORACLE_MASK_CAUSAL_WINDOW) && window < 0)
    return -1;
  return 0;
}

/*
 * One query row by the definition [MHA-CUDA 1]:
 *   s_j = scale * <q_i, k_j>            for allowed j
 *   m   = max_j s_j                     (subtracted for stability [MOSAIC 5.1])
 *   l   = sum_j exp(s_j - m)
 *   o   = sum_j exp(s_j - m) v_j / l
 *   lse = m + ln l
 * `s` is scratch of length L.
 */
static void definition_row(const float* qi, const float* kh, const float* vh,
                           int64_t L, int64_t d, double scale, int mask_kind,
                           int64_t window, int64_t i, double* s, double* o,
                           double* lse) {
  double m = -INFINITY;
  int64_t n_allowed = 0;
  for (int64_t j = 0; j < L; ++j) {
    if (!allowed(i, j, mask_kind, window)) continue;
    const float* kj = kh + j * d;
    double dot = 0.0;
    for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kj[c];
    s[j] = scale * dot;
    if (s[j] > m) m = s[j];
    ++n_allowed;
  }
  for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
  if (n_allowed == 0) {
    *lse = -INFINITY;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < L; ++j) {
    if (!allowed(i, j, mask_kind, window)) continue;
    double p = exp(s[j] - m);
    l += p;
    const float* vj = vh + j * d;
    for (int64_t c = 0; c < d; ++c) o[c] += p * (double)vj[c];
  }
  for (int64_t c = 0; c < d; ++c) o[c] /= l;
  *lse = m + log(l);
}

/* ---- thread pool over a list of rows ---------------------------------- */

typedef struct {
  const float *q, *k, *v;
  const int64_t *bh_idx, *row_idx; /* NULL: dense enumeration of all rows */
  double *out, *lse;
  int64_t L, d, nrows;
  double scale;
  int mask_kind;
  int64_t window;
  int64_t first, last; /* this worker's half-open slice of rows */
  int status;
} row_job;

static void* row_worker(void* arg) {
  row_job* job = (row_job*)arg;
  double* s = (double*)malloc((size_t)job->L * sizeof(double));
  if (!s) {
    job->status = -2;
    return NULL;
  }
  for (int64_t r = job->first; r < job->last; ++r) {
    int64_t bh, i;
    if (job->bh_idx) {
      bh = job->bh_idx[r];
      i = job->row_idx[r];
    } else {
      bh = r / job->L;
      i = r % job->L;
    }
    const int64_t head = bh * job->L * job->d;
    definition_row(job->q + head + i * job->d, job->k + head, job->v + head,
                   job->L, job->d, job->scale, job->mask_kind, job->window, i,
                   s, job->out + r * job->d, job->lse + r);
  }
  free(s);
  job->status = 0;
  return NULL;
}

static int run_rows(const float* q, const float* k, const float* v,
                    const int64_t* bh_idx, const int64_t* row_idx,
                    int64_t nrows, double* out, double* lse, int64_t L,
                    int64_t d, double scale, int mask_kind, int64_t window,
                    int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 1024) nthreads = 1024;
  if ((int64_t)nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
  row_job* jobs = (row_job*)calloc((size_t)nthreads, sizeof(row_job));
  pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return -2;
  }
  int64_t per = nrows / nthreads, extra = nrows % nthreads, start = 0;
  for (int t = 0; t < nthreads; ++t) {
    row_job* j = &jobs[t];
    j->q = q; j->k = k; j->v = v;
    j->bh_idx = bh_idx; j->row_idx = row_idx;
    j->out = out; j->lse = lse;
    j->L = L; j->d = d; j->nrows = nrows;
    j->scale = scale; j->mask_kind = mask_kind; j->window = window;
    j->first = start;
    j->last = start + per + (t < extra ? 1 : 0);
    start = j->last;
  }
  int started = 0, status = 0;
  for (int t = 1; t < nthreads; ++t) {
    if (pthread_create(&tids[t], NULL, row_worker, &jobs[t]) != 0) {
      jobs[t].status = 1; /* run it on this thread below */
    } else {
      ++started;
    }
  }
  row_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) {
    if (jobs[t].status == 1) row_worker(&jobs[t]);
    else pthread_join(tids[t], NULL);
  }
  (void)started;
  for (int t = 0; t < nthreads; ++t)
    if (jobs[t].status != 0) status = jobs[t].status;
  free(jobs);
  free(tids);
  return status;
}

int oracle_attn_fwd(const float* q, const float* k, const float* v, double* out,
                    double* lse, int64_t B, int64_t H, int64_t L, int64_t d,
                    double scale, int mask_kind, int64_t window, int nthreads) {
  if (check_args(q, k, v, out, lse, B, H, L, d, mask_kind, window)) return -1;
  return run_rows(q, k, v, NULL, NULL, B * H * L, out, lse, L, d, scale,
                  mask_kind, window, nthreads);
}

int oracle_attn_rows(const float* q, const float* k, const float* v,
                     const int64_t* bh_idx, const int64_t* row_idx,
                     int64_t nrows, double* out, double* lse, int64_t B,
                     int64_t H, int64_t L, int64_t d, double scale,
                     int mask_kind, int64_t window, int nthreads) {
  if (check_args(q, k, v, out, lse, B, H, L, d, mask_kind, window)) return -1;
  if (!bh_idx || !row_idx || nrows < 0) return -1;
  for (int64_t r = 0; r < nrows; ++r)
    if (bh_idx[r] < 0 || bh_idx[r] >= B * H || row_idx[r] < 0 || row_idx[r] >= L)
      return -1;
  if (nrows == 0) return 0;
  return run_rows(q, k, v, bh_idx, row_idx, nrows, out, lse, L, d, scale,
                  mask_kind, window, nthreads);
}

/*
 * K/V-blockwise online softmax, one row at a time [MOSAIC 3.2].  For each key
 * block:  m_new = max(m, max_j s_j);  alpha = exp(m - m_new);
 *         l = alpha*l + sum_j exp(s_j - m_new);
 *         acc = alpha*acc + sum_j exp(s_j - m_new) v_j;  m = m_new.
 * The page's sketch never updates its max and never rescales; the rescale by
 * alpha is what makes the result equal the definition.  A block in which no
 * key is allowed (and no earlier one either) leaves the state untouched.
 */
int oracle_attn_kv_blockwise(const float* q, const float* k, const float* v,
                             double* out, double* lse, int64_t B, int64_t H,
                             int64_t L, int64_t d, double scale, int mask_kind,
                             int64_t window, int64_t block) {
  if (check_args(q, k, v, out, lse, B, H, L, d, mask_kind, window)) return -1;
  if (block <= 0) return -1;
  double* s = (double*)malloc((size_t)block * sizeof(double));
  double* acc = (double*)malloc((size_t)d * sizeof(double));
  if (!s || !acc) {
    free(s);
    free(acc);
    return -2;
  }
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const float* kh = k + bh * L * d;
    const float* vh = v + bh * L * d;
    for (int64_t i = 0; i < L; ++i) {
      const float* qi = q + (bh * L + i) * d;
      double m = -INFINITY, l = 0.0;
      for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
      for (int64_t j0 = 0; j0 < L; j0 += block) {
        int64_t j1 = j0 + block < L ? j0 + block : L;
        double m_blk = -INFINITY;
        for (int64_t j = j0; j < j1; ++j) {
          if (!allowed(i, j, mask_kind, window)) {
            s[j - j0] = -INFINITY;
            continue;
          }
          double dot = 0.0;
          for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];
          s[j - j0] = scale * dot;
          if (s[j - j0] > m_blk) m_blk = s[j - j0];
        }
        double m_new = m_blk > m ? m_blk : m;
        if (m_new == -INFINITY) continue; /* nothing allowed yet */
        double alpha = exp(m - m_new);    /* exp(-inf) = 0 on the first block */
        l *= alpha;
        for (int64_t c = 0; c < d; ++c) acc[c] *= alpha;
        for (int64_t j = j0; j < j1; ++j) {
          if (s[j - j0] == -INFINITY) continue;
          double p = exp(s[j - j0] - m_new);
          l += p;
          for (int64_t c = 0; c < d; ++c) acc[c] += p * (double)vh[j * d + c];
        }
        m = m_new;
      }
      double* o = out + (bh * L + i) * d;
      if (l == 0.0) {
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        lse[bh * L + i] = -INFINITY;
      } else {
        for (int64_t c = 0; c < d; ++c) o[c] = acc[c] / l;
        lse[bh * L + i] = m + log(l);
      }
    }
  }
  free(s);
  free(acc);
  return 0;
}

/*
 * Query-blockwise attention [BPT]: rows [i0, min(i0 + block, L)) form a score
 * block against all L keys (materialised, block x L), masked with -inf, each
 * row normalised by its own max and sum, then multiplied by V.
 */
int oracle_attn_q_blockwise(const float* q, const float* k, const float* v,
                            double* out, double* lse, int64_t B, int64_t H,
                            int64_t L, int64_t d, double scale, int mask_kind,
                            int64_t window, int64_t block) {
  if (check_args(q, k, v, out, lse, B, H, L, d, mask_kind, window)) return -1;
  if (block <= 0) return -1;
  int64_t rows_max = block < L ? block : L;
  double* S = (double*)malloc((size_t)(rows_max * L) * sizeof(double));
  if (!S) return -2;
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const float* kh = k + bh * L * d;
    const float* vh = v + bh * L * d;
    for (int64_t i0 = 0; i0 < L; i0 += block) {
      int64_t i1 = i0 + block < L ? i0 + block : L;
      /* scores of the whole block */
      for (int64_t i = i0; i < i1; ++i) {
        const float* qi = q + (bh * L + i) * d;
        for (int64_t j = 0; j < L; ++j) {
          double dot = 0.0;
          for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];
          S[(i - i0) * L + j] = allowed(i, j, mask_kind, window) ? scale * dot : -INFINITY;
        }
      }
      /* row softmax, then P V */
      for (int64_t i = i0; i < i1; ++i) {
        double* Si = S + (i - i0) * L;
        double m = -INFINITY;
        for (int64_t j = 0; j < L; ++j)
          if (Si[j] > m) m = Si[j];
        double* o = out + (bh * L + i) * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        if (m == -INFINITY) {
          lse[bh * L + i] = -INFINITY;
          continue;
        }
        double l = 0.0;
        for (int64_t j = 0; j < L; ++j) {
          Si[j] = (Si[j] == -INFINITY) ? 0.0 : exp(Si[j] - m);
          l += Si[j];
        }
        for (int64_t j = 0; j < L; ++j) {
          double p = Si[j] / l;
          for (int64_t c = 0; c < d; ++c) o[c] += p * (double)vh[j * d + c];
        }
        lse[bh * L + i] = m + log(l);
      }
    }
  }
  free(S);
  return 0;
}

/*
 * The definition restricted to the keys j in [key_lo, key_hi): the partial
 * result a key shard holds ([MOSAIC 2.1], before its tree reduction).  out is
 * that range's softmax-weighted average of V (normalised within the range),
 * lse its natural-log log-sum-exp; a row with no allowed key in the range gets
 * out = 0 and lse = -inf.  One thread, plain loops.
 */
int oracle_attn_partial(const float* q, const float* k, const float* v, double* out,
                        double* lse, int64_t B, int64_t H, int64_t L, int64_t d,
                        double scale, int mask_kind, int64_t window, int64_t key_lo,
                        int64_t key_hi) {
  if (check_args(q, k, v, out, lse, B, H, L, d, mask_kind, window)) return -1;
  if (key_lo < 0 || key_hi > L || key_hi < key_lo) return -1;
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const float* kh = k + bh * L * d;
    const float* vh = v + bh * L * d;
    for (int64_t i = 0; i < L; ++i) {
      const float* qi = q + (bh * L + i) * d;
      double* o = out + (bh * L + i) * d;
      double m = -INFINITY;
      for (int64_t j = key_lo; j < key_hi; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];
        if (scale * dot > m) m = scale * dot;
      }
      for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
      if (m == -INFINITY) {
        lse[bh * L + i] = -INFINITY;
        continue;
      }
      double l = 0.0;
      for (int64_t j = key_lo; j < key_hi; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)kh[j * d + c];
        double p = exp(scale * dot - m);
        l += p;
        for (int64_t c = 0; c < d; ++c) o[c] += p * (double)vh[j * d + c];
      }
      for (int64_t c = 0; c < d; ++c) o[c] /= l;
      lse[bh * L + i] = m + log(l);
    }
  }
  return 0;
}

/* ---- the multi-head attention layer [MHA-CUDA 2.1, 2.2] -------------- */

/*
 * The layer's steps in the page's order, all in fp64:
 *   qkv = x W_qkv^T + b_qkv                       (Linear(E, 3E))
 *   q, k, v = qkv[..., 0:E], [E:2E], [2E:3E]      (chunk(3, dim=-1))
 *   head h of each = columns [h d, (h+1) d)       (view(B, L, H, d).transpose)
 *   context[b, i, h d + c] = definition row i of head h, scale 1/sqrt(d)
 *   y = context W_out^T + b_out                   (Linear(E, E))
 * Biases may be NULL (zero).  Single-threaded; for small problems.
 */
int oracle_mha_fwd(const float* x, const float* w_qkv, const float* b_qkv, const float* w_out,
                   const float* b_out, double* y, int64_t B, int64_t L, int64_t E, int64_t H,
                   int mask_kind, int64_t window) {
  if (!x || !w_qkv || !w_out || !y || B <= 0 || L <= 0 || E <= 0 || H <= 0 || E % H) return -1;
  if (mask_kind < ORACLE_MASK_NONE || mask_kind > ORACLE_MASK_CAUSAL_WINDOW) return -1;
  if ((mask_kind == ORACLE_MASK_WINDOW || mask_kind == ORACLE_MASK_CAUSAL_WINDOW) && window < 0)
    return -1;
  const int64_t d = E / H;
  const double scale = 1.0 / sqrt((double)d);
  double* qkv = (double*)malloc((size_t)(B * L * 3 * E) * sizeof(double));
  double* ctx = (double*)malloc((size_t)(B * L * E) * sizeof(double));
  double* s = (double*)malloc((size_t)L * sizeof(double));
  if (!qkv || !ctx || !s) {
    free(qkv);
    free(ctx);
    free(s);
    return -2;
  }
  for (int64_t r = 0; r < B * L; ++r)
    for (int64_t j = 0; j < 3 * E; ++j) {
      double acc = b_qkv ? (double)b_qkv[j] : 0.0;
      for (int64_t c = 0; c < E; ++c) acc += (double)x[r * E + c] * (double)w_qkv[j * E + c];
      qkv[r * 3 * E + j] = acc;
    }
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < H; ++h)
      for (int64_t i = 0; i < L; ++i) {
        const double* qi = qkv + (b * L + i) * 3 * E + h * d;
        double m = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
          if (!allowed(i, j, mask_kind, window)) continue;
          const double* kj = qkv + (b * L + j) * 3 * E + E + h * d;
          double dot = 0.0;
          for (int64_t c = 0; c < d; ++c) dot += qi[c] * kj[c];
          s[j] = scale * dot;
          if (s[j] > m) m = s[j];
        }
        double* o = ctx + (b * L + i) * E + h * d;
        for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
        double l = 0.0;
        for (int64_t j = 0; j < L; ++j) {
          if (!allowed(i, j, mask_kind, window)) continue;
          const double p = exp(s[j] - m);
          l += p;
          const double* vj = qkv + (b * L + j) * 3 * E + 2 * E + h * d;
          for (int64_t c = 0; c < d; ++c) o[c] += p * vj[c];
        }
        for (int64_t c = 0; c < d; ++c) o[c] /= l;
      }
  for (int64_t r = 0; r < B * L; ++r)
    for (int64_t j = 0; j < E; ++j) {
      double acc = b_out ? (double)b_out[j] : 0.0;
      for (int64_t c = 0; c < E; ++c) acc += ctx[r * E + c] * (double)w_out[j * E + c];
      y[r * E + j] = acc;
    }
  free(qkv);
  free(ctx);
  free(s);
  return 0;
}

/* ---- backward by recomputation [LONGSEQ 3.1], [MOSAIC 2.2] ------------ */

/*
 * Gradients of O = softmax(scale Q K^T + mask) V given dO, from the
 * definition (the pages recompute the attention weights instead of storing
 * them; here every row's weights are recomputed from Q and K):
 *   P_ij  = exp(s_ij - lse_i) for allowed j, s_ij = scale <q_i, k_j>
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i
 * All [B, H, L, d] in fp64; single-threaded.
 */
int oracle_attn_bwd(const float* q, const float* k, const float* v, const float* dout,
                    double* dq, double* dk, double* dv, int64_t B, int64_t H, int64_t L,
                    int64_t d, double scale, int mask_kind, int64_t window) {
  if (check_args(q, k, v, dq, dk, B, H, L, d, mask_kind, window) || !dout || !dv) return -1;
  double* P = (double*)malloc((size_t)L * sizeof(double));
  double* dP = (double*)malloc((size_t)L * sizeof(double));
  if (!P || !dP) {
    free(P);
    free(dP);
    return -2;
  }
  const int64_t n = B * H * L * d;
  for (int64_t e = 0; e < n; ++e) dq[e] = dk[e] = dv[e] = 0.0;
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const int64_t head = bh * L * d;
    for (int64_t i = 0; i < L; ++i) {
      const float* qi = q + head + i * d;
      const float* gi = dout + head + i * d;
      double m = -INFINITY;
      for (int64_t j = 0; j < L; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += (double)qi[c] * (double)k[head + j * d + c];
        P[j] = scale * dot;
        if (P[j] > m) m = P[j];
      }
      if (m == -INFINITY) continue; /* no allowed key: no gradient */
      double l = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        P[j] = exp(P[j] - m);
        l += P[j];
      }
      double D = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        P[j] /= l;
        double dot = 0.0;
        for (int64_t c = 0; c < d; ++c) dot += (double)gi[c] * (double)v[head + j * d + c];
        dP[j] = dot;
        D += P[j] * dot;
      }
      for (int64_t j = 0; j < L; ++j) {
        if (!allowed(i, j, mask_kind, window)) continue;
        const double ds = P[j] * (dP[j] - D);
        for (int64_t c = 0; c < d; ++c) {
          dv[head + j * d + c] += P[j] * (double)gi[c];
          dq[head + i * d + c] += scale * ds * (double)k[head + j * d + c];
          dk[head + j * d + c] += scale * ds * (double)qi[c];
        }
      }
    }
  }
  free(P);
  free(dP);
  return 0;
}

