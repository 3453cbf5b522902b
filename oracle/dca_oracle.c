/*
 * dca_oracle.c -- plain float64 CPU reference of Dual Chunk Attention (DCA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is
 * checked against.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load it; the product path never calls it and shares
 * no code, header, table or constant with it.
 *
 * Sources (web pages on Qwen2.5-1M; cited by title and section):
 *   [MIZ] "Qwen2.5-1M 不重训外推 1M" (mizuki-eaf.pages.dev), sections
 *         "核心思想", "Intra-Chunk Attention：块内正常来",
 *         "Successive-Chunk Attention：相邻块的边界过渡",
 *         "Inter-Chunk Attention：远距离的善意谎言", "为什么不需要重训？",
 *         "DCA + YaRN", "Chunked Prefill".
 *   [QBIT] news article on the Qwen2.5-1M release (7a8v.yksolo.com),
 *         section "如何炼成的？" (RoPE base raised to 10,000,000; DCA remaps
 *         too-large relative positions to smaller ones).
 *   [YDL] "Qwen-2.5 explained" (yudonglee.me), section 三 (GQA, RoPE base 1e7).
 *
 * What is computed, per query row i and query head h (all arithmetic fp64):
 *   1. theta_k = base^(-2k/d), k < d/2                               [QBIT, YDL]
 *   2. R(p) rotates the pair (x_k, x_{k+d/2}) by the angle p*theta_k
 *      (half-split pairing; the pages name no pairing, this is a reading).
 *   3. DCA position map for a key j <= i, with n = index // s, r = index % s
 *      (chunks of size s start at token 0)                             [MIZ 核心思想]
 *        key position     Pk(j)   = j mod s        (periodic key index)  [MIZ Inter]
 *        query position   Pq(i,j) = r_i            if n_i == n_j         [MIZ Intra]
 *                                 = s + r_i        if n_i - n_j == 1 and the
 *                                                  pair is inside the local
 *                                                  window w              [MIZ Successive]
 *                                 = c - 1          otherwise (large fixed
 *                                                  query index)          [MIZ Inter]
 *      Window reading A (default): the pair is inside the window when r_i < w.
 *      Window reading B (option):  the pair is inside the window when i - j < w.
 *      Either way the in-window distance Pq - Pk equals the true distance i - j.
 *   4. logit(i,j) = tau * m^2 * < R(Pq) q_i , R(Pk) k_j >,  tau = 1/sqrt(d),
 *      m = 1 if f <= 1 else 0.1*ln(f) + 1 (YaRN attention temperature; the
 *      pages only say YaRN scales the scores and is orthogonal to DCA; the
 *      formula for m is the one of the YaRN paper they cite)         [MIZ DCA + YaRN]
 *   5. out_i = sum_{j<=i} softmax_j(logit(i,.)) v_j, exact two-pass softmax
 *      (max first, then exponentials), causal including j = i.
 *   6. GQA: query head h reads KV head h // (Hq/Hkv).                   [YDL 三]
 *   7. Chunked prefill: a query block of Lq rows starting at absolute row
 *      q_start attends to a KV cache of Lk rows; the formula above is applied
 *      to absolute indices, so block results equal the one-shot rows. [MIZ Chunked Prefill]
 *
 * Sparse variant (dca_oracle_sparse_attention): the vertical-slash sparse
 * attention that the Qwen2.5-1M framework runs on top of DCA ("Qwen2.5-1M
 * 不重训外推 1M", sections "跟 NSA / 其他稀疏注意力的区别" and "稀疏注意力 +
 * 核优化": a few key columns draw most of the attention, per-head sparse
 * configurations are searched offline, and at inference only the selected
 * keys are attended).  For query head h with vertical key set V_h and slash
 * offset set S_h, row i attends exactly the member keys
 *      M_h(i) = { j <= i : j in V_h }  U  { i - o : o in S_h, o <= i }  U  { i }
 * (each key once; the row's own key always, so no row is empty), with the
 * DCA logits above and a softmax over M_h(i).
 *
 * Key selection for the sparse variant (dca_oracle_vs_scores): the estimate
 * from which the per-head vertical and slash sets are chosen.  For the last
 * n_last rows i of the query block and query head h, p_ij is the softmax over
 * keys j <= i of the logits, either the DCA logits above or -- the
 * refinement of "稀疏注意力 + 核优化", which restores continuous relative
 * positions at this stage -- plain RoPE logits with the true positions
 * (query rotated by i, key by j).  Then
 *      vertical_h[j] = sum_rows p_ij,   slash_h[o] = sum_rows p_{i, i-o}.
 * The n_v keys and n_s offsets of largest score (ties: the smaller index)
 * form the head's pattern (dca_oracle_topk).
 *
 * The oracle also carries a `mutation` argument used only by tests that
 * check that the pins catch plausible mistakes (each value plants one known
 * mistake).  mutation = 0 is the oracle proper.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_DT_BF16 0
#define ORACLE_DT_F32 1
#define ORACLE_DT_F64 2

/* mutations planted for the pin tests (never used otherwise) */
#define MUT_NONE 0
#define MUT_SIN_SIGN 1        /* wrong sign of the sine term in R(p)            */
#define MUT_KEY_NOT_PERIODIC 2/* key position j instead of j mod s              */
#define MUT_QUERY_C 3         /* large query index c instead of c - 1           */
#define MUT_WINDOW_LE 4       /* window test r_i <= w instead of r_i < w        */
#define MUT_PAIR_ADJACENT 5   /* pairs (2k, 2k+1) instead of (k, k + d/2)        */
#define MUT_NO_MSCALE_SQ 6    /* logits scaled by m instead of m^2              */
#define MUT_SUCC_AS_INTER 7   /* successive pairs always take the inter rule    */
#define MUT_NONCAUSAL_DIAG 8  /* diagonal j = i excluded                        */
#define MUT_GQA_INTERLEAVED 9 /* head h reads KV head h % Hkv                   */
#define MUT_THETA_D 10        /* theta_k = base^(-k/d)                          */
/* sparse variant */
#define MUT_SP_NO_DEDUP 11    /* a key that is vertical and on a slash counted twice */
#define MUT_SP_VERT_ACAUSAL 12/* vertical keys j > i included                   */
#define MUT_SP_OFFSET_OFF1 13 /* slash offset o selects j = i - o - 1            */
#define MUT_SP_NO_SELF 14     /* the row's own key not added                      */

static double to_f64(const void* p, int dtype, int64_t idx) {
  if (dtype == ORACLE_DT_BF16) {
    uint16_t b = ((const uint16_t*)p)[idx];
    uint32_t u = ((uint32_t)b) << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  if (dtype == ORACLE_DT_F32) return (double)((const float*)p)[idx];
  return ((const double*)p)[idx];
}

/* YaRN attention-temperature factor m(f); logits are multiplied by m^2.
 * Parity unpinned by the pages: they say YaRN scales the attention scores but
 * print no formula; this is the YaRN paper's formula (0.1 ln f + 1). */
double dca_oracle_mscale(double f) {
  if (f <= 1.0) return 1.0;
  return 0.1 * log(f) + 1.0;
}

/* DCA position map of [MIZ]; returns the relation class
 * (0 intra, 1 successive, 2 inter) and writes the query / key positions. */
int dca_oracle_position(int64_t i, int64_t j, int64_t s, int64_t w, int64_t c,
                        int reading, int mutation, int64_t* pq, int64_t* pk) {
  int64_t ni = i / s, nj = j / s, ri = i % s;
  *pk = (mutation == MUT_KEY_NOT_PERIODIC) ? j : j % s;
  if (ni == nj) {
    *pq = ri;
    return 0;
  }
  if (ni - nj == 1 && mutation != MUT_SUCC_AS_INTER) {
    int in_window;
    if (reading == 1)
      in_window = (i - j) < w;
    else if (mutation == MUT_WINDOW_LE)
      in_window = ri <= w;
    else
      in_window = ri < w;
    if (in_window) {
      *pq = s + ri;
      return 1;
    }
  }
  *pq = (mutation == MUT_QUERY_C) ? c : c - 1;
  return 2;
}

/* R(p) x for one head vector of length d, fp64. */
static void rotate(const double* x, double* y, int d, int64_t p,
                   const double* theta, int mutation) {
  int half = d / 2;
  for (int k = 0; k < half; ++k) {
    int a = k, b = k + half;
    if (mutation == MUT_PAIR_ADJACENT) {
      a = 2 * k;
      b = 2 * k + 1;
    }
    double ang = (double)p * theta[k];
    double cs = cos(ang), sn = sin(ang);
    if (mutation == MUT_SIN_SIGN) sn = -sn;
    y[a] = x[a] * cs - x[b] * sn;
    y[b] = x[a] * sn + x[b] * cs;
  }
}

typedef struct {
  /* inputs */
  const void *q, *k, *v;
  int dtype;
  int64_t q_start, Lq, Lk;
  int Hq, Hkv, d;
  int64_t s, w, c;
  double base, yarn;
  int reading, mutation;
  const int64_t* rows;
  int64_t n_rows;
  const int* heads;
  int n_heads;
  double* out;
  double* lse;
  /* sparse pattern (NULL v_ptr: dense) -- CSR per query head, sorted lists */
  const int64_t *v_ptr, *v_idx, *s_ptr, *s_off;
  int64_t krot_rows;  /* rows of krot (keys 0 .. krot_rows - 1 are rotated) */
  /* shared state */
  const double* theta;
  const double* krot; /* rotated keys of the current KV head: [jmax+1][d] */
  int kv_head;        /* KV head whose keys are in krot */
  const int64_t* work;/* (row index, head index) pairs for this KV head */
  int64_t n_work;
  int64_t next;       /* work counter */
  pthread_mutex_t mu;
  int status;
} job_t;

static int kv_of_head(const job_t* J, int h) {
  int G = J->Hq / J->Hkv;
  if (J->mutation == MUT_GQA_INTERLEAVED) return h % J->Hkv;
  return h / G;
}

/* One (row, head) output: the definition written out. */
static void one_row(job_t* J, int64_t ridx, int hidx, double* scratch) {
  const int d = J->d;
  const int64_t t = J->rows[ridx];
  const int64_t i = J->q_start + t;
  const int h = J->heads[hidx];
  double* logit = scratch;               /* [i+1] */
  double* qraw = scratch + (i + 1);      /* [d] */
  double* qvar = qraw + d;               /* [3][d]: intra, successive, inter */
  int64_t qpos_cached[3] = {-1, -1, -1};
  double tau = 1.0 / sqrt((double)d);
  double m = dca_oracle_mscale(J->yarn);
  double scale = tau * ((J->mutation == MUT_NO_MSCALE_SQ) ? m : m * m);

  for (int e = 0; e < d; ++e)
    qraw[e] = to_f64(J->q, J->dtype, (t * J->Hq + h) * (int64_t)d + e);

  int64_t jend = i; /* causal: keys 0..i */
  if (J->mutation == MUT_NONCAUSAL_DIAG) jend = i - 1;
  double mx = -INFINITY;
  for (int64_t j = 0; j <= jend; ++j) {
    int64_t pq, pk;
    int cls = dca_oracle_position(i, j, J->s, J->w, J->c, J->reading,
                                  J->mutation, &pq, &pk);
    double* qv = qvar + cls * d;
    if (qpos_cached[cls] != pq) { /* at most a few distinct query positions per row */
      rotate(qraw, qv, d, pq, J->theta, J->mutation);
      qpos_cached[cls] = pq;
    }
    /* krot holds R(j mod s) k_j; the key-not-periodic mutation is applied
       through pk below by re-rotating when it differs from j mod s. */
    const double* kr = J->krot + j * (int64_t)d;
    double kbuf[1024];
    if (pk != j % J->s) {
      double kraw[1024];
      for (int e = 0; e < d; ++e)
        kraw[e] = to_f64(J->k, J->dtype, (j * J->Hkv + J->kv_head) * (int64_t)d + e);
      rotate(kraw, kbuf, d, pk, J->theta, J->mutation);
      kr = kbuf;
    }
    double dot = 0.0;
    for (int e = 0; e < d; ++e) dot += qv[e] * kr[e];
    logit[j] = scale * dot;
    if (logit[j] > mx) mx = logit[j];
  }
  double* o = J->out + (ridx * J->n_heads + hidx) * (int64_t)d;
  for (int e = 0; e < d; ++e) o[e] = 0.0;
  if (jend < 0) { /* only reachable under the non-causal-diagonal mutation */
    if (J->lse) J->lse[ridx * J->n_heads + hidx] = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int64_t j = 0; j <= jend; ++j) {
    double p = exp(logit[j] - mx);
    sum += p;
    for (int e = 0; e < d; ++e)
      o[e] += p * to_f64(J->v, J->dtype, (j * J->Hkv + J->kv_head) * (int64_t)d + e);
  }
  for (int e = 0; e < d; ++e) o[e] /= sum;
  if (J->lse) J->lse[ridx * J->n_heads + hidx] = mx + log(sum);
}

static int cmp_i64(const void* a, const void* b) {
  int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return (x > y) - (x < y);
}

/* One (row, head) output of the sparse variant: the member set written out,
 * then the same logits and softmax as one_row over those keys only. */
static void one_row_sparse(job_t* J, int64_t ridx, int hidx, double* scratch, int64_t* cand) {
  const int d = J->d;
  const int64_t t = J->rows[ridx];
  const int64_t i = J->q_start + t;
  const int h = J->heads[hidx];
  /* member keys */
  int64_t n = 0;
  for (int64_t e = J->v_ptr[h]; e < J->v_ptr[h + 1]; ++e) {
    int64_t j = J->v_idx[e];
    if (j <= i || (J->mutation == MUT_SP_VERT_ACAUSAL && j < J->krot_rows)) cand[n++] = j;
  }
  for (int64_t e = J->s_ptr[h]; e < J->s_ptr[h + 1]; ++e) {
    int64_t o = J->s_off[e];
    int64_t j = (J->mutation == MUT_SP_OFFSET_OFF1) ? i - o - 1 : i - o;
    if (o <= i && j >= 0) cand[n++] = j;
  }
  if (J->mutation != MUT_SP_NO_SELF) cand[n++] = i;
  qsort(cand, (size_t)n, sizeof(int64_t), cmp_i64);
  int64_t m = 0;
  for (int64_t e = 0; e < n; ++e)
    if (J->mutation == MUT_SP_NO_DEDUP || m == 0 || cand[e] != cand[m - 1]) cand[m++] = cand[e];

  double* logit = scratch;          /* [m] */
  double* qraw = scratch + m;       /* [d] */
  double* qvar = qraw + d;          /* [3][d] */
  int64_t qpos_cached[3] = {-1, -1, -1};
  double scale = (1.0 / sqrt((double)d)) * dca_oracle_mscale(J->yarn) * dca_oracle_mscale(J->yarn);
  for (int e = 0; e < d; ++e)
    qraw[e] = to_f64(J->q, J->dtype, (t * J->Hq + h) * (int64_t)d + e);
  double mx = -INFINITY;
  for (int64_t e = 0; e < m; ++e) {
    int64_t j = cand[e], pq, pk;
    int cls = dca_oracle_position(i, j, J->s, J->w, J->c, J->reading, MUT_NONE, &pq, &pk);
    double* qv = qvar + cls * d;
    if (qpos_cached[cls] != pq) {
      rotate(qraw, qv, d, pq, J->theta, MUT_NONE);
      qpos_cached[cls] = pq;
    }
    const double* kr = J->krot + j * (int64_t)d;
    double dot = 0.0;
    for (int c2 = 0; c2 < d; ++c2) dot += qv[c2] * kr[c2];
    logit[e] = scale * dot;
    if (logit[e] > mx) mx = logit[e];
  }
  double* o = J->out + (ridx * J->n_heads + hidx) * (int64_t)d;
  for (int e = 0; e < d; ++e) o[e] = 0.0;
  if (m == 0) {
    if (J->lse) J->lse[ridx * J->n_heads + hidx] = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int64_t e = 0; e < m; ++e) {
    double p = exp(logit[e] - mx);
    sum += p;
    for (int c2 = 0; c2 < d; ++c2)
      o[c2] += p * to_f64(J->v, J->dtype, (cand[e] * J->Hkv + J->kv_head) * (int64_t)d + c2);
  }
  for (int e = 0; e < d; ++e) o[e] /= sum;
  if (J->lse) J->lse[ridx * J->n_heads + hidx] = mx + log(sum);
}

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  int64_t imax = 0;
  for (int64_t r = 0; r < J->n_rows; ++r)
    if (J->q_start + J->rows[r] > imax) imax = J->q_start + J->rows[r];
  int64_t most = 0; /* candidate keys of a sparse row (before removing repeats) */
  if (J->v_ptr)
    for (int hh = 0; hh < J->Hq; ++hh) {
      int64_t c2 = (J->v_ptr[hh + 1] - J->v_ptr[hh]) + (J->s_ptr[hh + 1] - J->s_ptr[hh]) + 1;
      if (c2 > most) most = c2;
    }
  int64_t nlog = imax + 1 > most ? imax + 1 : most;
  double* scratch = (double*)malloc(sizeof(double) * (size_t)(nlog + 4 * J->d));
  int64_t* cand = NULL;
  if (J->v_ptr) {
    cand = (int64_t*)malloc(sizeof(int64_t) * (size_t)(most + 1));
    if (!cand) {
      free(scratch);
      scratch = NULL;
    }
  }
  if (!scratch) {
    pthread_mutex_lock(&J->mu);
    J->status = -3;
    pthread_mutex_unlock(&J->mu);
    return NULL;
  }
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int64_t w = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (w >= J->n_work) break;
    if (J->v_ptr)
      one_row_sparse(J, J->work[2 * w], (int)J->work[2 * w + 1], scratch, cand);
    else
      one_row(J, J->work[2 * w], (int)J->work[2 * w + 1], scratch);
  }
  free(scratch);
  free(cand);
  return NULL;
}

typedef struct {
  job_t* J;
  double* krot;
  int64_t j0, j1;
} rot_job_t;

static void* rot_worker(void* arg) {
  rot_job_t* R = (rot_job_t*)arg;
  job_t* J = R->J;
  const int d = J->d;
  double kraw[1024];
  for (int64_t j = R->j0; j < R->j1; ++j) {
    for (int e = 0; e < d; ++e)
      kraw[e] = to_f64(J->k, J->dtype, (j * J->Hkv + J->kv_head) * (int64_t)d + e);
    rotate(kraw, R->krot + j * (int64_t)d, d, j % J->s, J->theta, J->mutation);
  }
  return NULL;
}

/*
 * Full entry point.  Layouts (row-major, contiguous):
 *   q    [Lq][Hq][d]    query block; row t has absolute index q_start + t
 *   k, v [Lk][Hkv][d]   KV cache (unrotated keys)
 *   rows [n_rows]       block row indices t to evaluate
 *   heads[n_heads]      query heads to evaluate
 *   out  [n_rows][n_heads][d] fp64,  lse [n_rows][n_heads] (natural log) or NULL
 * Returns 0 on success, -1 on a bad argument, -3 on allocation failure.
 */
static int attention_impl(const void* q, const void* k, const void* v, int dtype,
                          int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv,
                          int d, int64_t s, int64_t w, int64_t c, double base,
                          double yarn, int reading, int mutation,
                          const int64_t* v_ptr, const int64_t* v_idx,
                          const int64_t* s_ptr, const int64_t* s_off,
                          const int64_t* rows, int64_t n_rows, const int* heads,
                          int n_heads, double* out, double* lse, int n_threads) {
  if (!q || !k || !v || !out || !rows || !heads) return -1;
  if (dtype < 0 || dtype > 2 || d <= 0 || d % 2 || d > 1024) return -1;
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
  if (s < 1 || w < 0 || c < 1 || q_start < 0 || Lq < 0 || Lk < q_start + Lq) return -1;
  if (n_threads < 1) n_threads = 1;
  for (int64_t r = 0; r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= Lq) return -1;
  for (int hh = 0; hh < n_heads; ++hh)
    if (heads[hh] < 0 || heads[hh] >= Hq) return -1;

  double* theta = (double*)malloc(sizeof(double) * (size_t)(d / 2));
  if (!theta) return -3;
  for (int kk = 0; kk < d / 2; ++kk) {
    double expo = (mutation == MUT_THETA_D) ? -(double)kk / d : -2.0 * kk / d;
    theta[kk] = pow(base, expo);
  }

  job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.v = v; J.dtype = dtype;
  J.q_start = q_start; J.Lq = Lq; J.Lk = Lk;
  J.Hq = Hq; J.Hkv = Hkv; J.d = d;
  J.s = s; J.w = w; J.c = c; J.base = base; J.yarn = yarn;
  J.reading = reading; J.mutation = mutation;
  J.rows = rows; J.n_rows = n_rows; J.heads = heads; J.n_heads = n_heads;
  J.out = out; J.lse = lse; J.theta = theta;
  J.v_ptr = v_ptr; J.v_idx = v_idx; J.s_ptr = s_ptr; J.s_off = s_off;
  pthread_mutex_init(&J.mu, NULL);

  int64_t imax = -1;
  for (int64_t r = 0; r < n_rows; ++r)
    if (q_start + rows[r] > imax) imax = q_start + rows[r];
  /* keys 0 .. imax are rotated; the acausal-vertical mutation reaches up to Lk - 1 */
  if (v_ptr && mutation == MUT_SP_VERT_ACAUSAL && imax >= 0) imax = Lk - 1;
  J.krot_rows = imax + 1;

  int64_t* work = (int64_t*)malloc(sizeof(int64_t) * 2 * (size_t)(n_rows * n_heads + 1));
  double* krot = (double*)malloc(sizeof(double) * (size_t)(imax + 1) * d + 8);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
  rot_job_t* rj = (rot_job_t*)malloc(sizeof(rot_job_t) * (size_t)n_threads);
  int status = 0;
  if (!work || !krot || !th || !rj) status = -3;

  /* one KV head at a time: rotate its keys once, then every (row, head) of it */
  for (int g = 0; status == 0 && g < Hkv && n_rows > 0; ++g) {
    int64_t nw = 0;
    for (int64_t r = 0; r < n_rows; ++r)
      for (int hh = 0; hh < n_heads; ++hh) {
        J.kv_head = g; /* kv_of_head reads only Hq/Hkv/mutation */
        if (kv_of_head(&J, heads[hh]) != g) continue;
        work[2 * nw] = r;
        work[2 * nw + 1] = hh;
        ++nw;
      }
    if (nw == 0) continue;
    J.kv_head = g;
    int64_t per = (imax + 1 + n_threads - 1) / n_threads;
    for (int t = 0; t < n_threads; ++t) {
      rj[t].J = &J;
      rj[t].krot = krot;
      rj[t].j0 = t * per < imax + 1 ? t * per : imax + 1;
      rj[t].j1 = (t + 1) * per < imax + 1 ? (t + 1) * per : imax + 1;
      pthread_create(&th[t], NULL, rot_worker, &rj[t]);
    }
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
    J.krot = krot;
    J.work = work;
    J.n_work = nw;
    J.next = 0;
    for (int t = 0; t < n_threads; ++t) pthread_create(&th[t], NULL, worker, &J);
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
    if (J.status) status = J.status;
  }
  free(work);
  free(krot);
  free(th);
  free(rj);
  free(theta);
  pthread_mutex_destroy(&J.mu);
  return status;
}

int dca_oracle_attention_mut(const void* q, const void* k, const void* v, int dtype,
                             int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv,
                             int d, int64_t s, int64_t w, int64_t c, double base,
                             double yarn, int reading, int mutation,
                             const int64_t* rows, int64_t n_rows, const int* heads,
                             int n_heads, double* out, double* lse, int n_threads) {
  return attention_impl(q, k, v, dtype, q_start, Lq, Lk, Hq, Hkv, d, s, w, c, base, yarn,
                        reading, mutation, NULL, NULL, NULL, NULL, rows, n_rows, heads,
                        n_heads, out, lse, n_threads);
}

/*
 * Sparse variant.  v_ptr, s_ptr [Hq + 1] (CSR offsets), v_idx [v_ptr[Hq]]
 * vertical key indices in [0, Lk) and s_off [s_ptr[Hq]] slash offsets in
 * [0, Lk), each head's list sorted ascending without repeats.  Other
 * arguments and outputs as dca_oracle_attention_mut.
 */
int dca_oracle_sparse_attention(const void* q, const void* k, const void* v, int dtype,
                                int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv,
                                int d, int64_t s, int64_t w, int64_t c, double base,
                                double yarn, int reading, int mutation,
                                const int64_t* v_ptr, const int64_t* v_idx,
                                const int64_t* s_ptr, const int64_t* s_off,
                                const int64_t* rows, int64_t n_rows, const int* heads,
                                int n_heads, double* out, double* lse, int n_threads) {
  if (!v_ptr || !s_ptr || Hq <= 0) return -1;
  for (int h = 0; h < Hq; ++h) {
    if (v_ptr[h + 1] < v_ptr[h] || s_ptr[h + 1] < s_ptr[h]) return -1;
    for (int64_t e = v_ptr[h]; e < v_ptr[h + 1]; ++e)
      if (v_idx[e] < 0 || v_idx[e] >= Lk || (e > v_ptr[h] && v_idx[e] <= v_idx[e - 1])) return -1;
    for (int64_t e = s_ptr[h]; e < s_ptr[h + 1]; ++e)
      if (s_off[e] < 0 || s_off[e] >= Lk || (e > s_ptr[h] && s_off[e] <= s_off[e - 1])) return -1;
  }
  return attention_impl(q, k, v, dtype, q_start, Lq, Lk, Hq, Hkv, d, s, w, c, base, yarn,
                        reading, mutation, v_ptr, v_idx, s_ptr, s_off, rows, n_rows, heads,
                        n_heads, out, lse, n_threads);
}

/*
 * Vertical / slash scores of the key selection (definition in the header).
 * q [Lq][Hq][d] query block (row t at absolute index q_start + t), k
 * [Lk][Hkv][d]; the last n_last rows of the block are the estimate's rows.
 * continuous = 0: DCA logits; 1: RoPE logits at the true positions.
 * vert, slash [Hq][Lk] fp64 outputs.  Returns 0, -1 on bad arguments,
 * -3 on allocation failure.  Single-threaded per head, parallel over heads.
 */
typedef struct {
  const void *q, *k;
  int dtype;
  int64_t q_start, Lq, Lk, n_last;
  int Hq, Hkv, d;
  int64_t s, w, c;
  double base, yarn;
  int reading, continuous;
  const double* theta;
  double *vert, *slash;
  int next;
  pthread_mutex_t mu;
  int status;
} vs_job_t;

static void vs_head(vs_job_t* J, int h) {
  const int d = J->d;
  const int G = J->Hq / J->Hkv, g = h / G;
  double* logit = (double*)malloc(sizeof(double) * (size_t)J->Lk);
  double* kraw = (double*)malloc(sizeof(double) * (size_t)d);
  double* kr = (double*)malloc(sizeof(double) * (size_t)d);
  double* qraw = (double*)malloc(sizeof(double) * (size_t)d);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  if (!logit || !kraw || !kr || !qraw || !qv) {
    pthread_mutex_lock(&J->mu);
    J->status = -3;
    pthread_mutex_unlock(&J->mu);
    free(logit); free(kraw); free(kr); free(qraw); free(qv);
    return;
  }
  double scale = (1.0 / sqrt((double)d)) * dca_oracle_mscale(J->yarn) * dca_oracle_mscale(J->yarn);
  double* vert = J->vert + (int64_t)h * J->Lk;
  double* slash = J->slash + (int64_t)h * J->Lk;
  for (int64_t j = 0; j < J->Lk; ++j) vert[j] = slash[j] = 0.0;
  for (int64_t t = J->Lq - J->n_last; t < J->Lq; ++t) {
    const int64_t i = J->q_start + t;
    for (int e = 0; e < d; ++e) qraw[e] = to_f64(J->q, J->dtype, (t * J->Hq + h) * (int64_t)d + e);
    double mx = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
      int64_t pq, pk;
      if (J->continuous) {
        pq = i;
        pk = j;
      } else {
        dca_oracle_position(i, j, J->s, J->w, J->c, J->reading, MUT_NONE, &pq, &pk);
      }
      rotate(qraw, qv, d, pq, J->theta, MUT_NONE);
      for (int e = 0; e < d; ++e) kraw[e] = to_f64(J->k, J->dtype, (j * J->Hkv + g) * (int64_t)d + e);
      rotate(kraw, kr, d, pk, J->theta, MUT_NONE);
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += qv[e] * kr[e];
      logit[j] = scale * dot;
      if (logit[j] > mx) mx = logit[j];
    }
    double sum = 0.0;
    for (int64_t j = 0; j <= i; ++j) sum += exp(logit[j] - mx);
    for (int64_t j = 0; j <= i; ++j) {
      const double p = exp(logit[j] - mx) / sum;
      vert[j] += p;
      slash[i - j] += p;
    }
  }
  free(logit); free(kraw); free(kr); free(qraw); free(qv);
}

static void* vs_worker(void* arg) {
  vs_job_t* J = (vs_job_t*)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int h = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (h >= J->Hq) break;
    vs_head(J, h);
  }
  return NULL;
}

int dca_oracle_vs_scores(const void* q, const void* k, int dtype, int64_t q_start, int64_t Lq,
                         int64_t Lk, int Hq, int Hkv, int d, int64_t s, int64_t w, int64_t c,
                         double base, double yarn, int reading, int64_t n_last, int continuous,
                         double* vert, double* slash, int n_threads) {
  if (!q || !k || !vert || !slash) return -1;
  if (dtype < 0 || dtype > 2 || d <= 0 || d % 2 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
  if (s < 1 || w < 0 || c < 1 || q_start < 0 || Lq < 1 || Lk < q_start + Lq) return -1;
  if (n_last < 1 || n_last > Lq) return -1;
  if (n_threads < 1) n_threads = 1;
  double* theta = (double*)malloc(sizeof(double) * (size_t)(d / 2));
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
  if (!theta || !th) {
    free(theta);
    free(th);
    return -3;
  }
  for (int kk = 0; kk < d / 2; ++kk) theta[kk] = pow(base, -2.0 * kk / d);
  vs_job_t J;
  memset(&J, 0, sizeof J);
  J.q = q; J.k = k; J.dtype = dtype; J.q_start = q_start; J.Lq = Lq; J.Lk = Lk;
  J.n_last = n_last; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.s = s; J.w = w; J.c = c;
  J.base = base; J.yarn = yarn; J.reading = reading; J.continuous = continuous;
  J.theta = theta; J.vert = vert; J.slash = slash;
  pthread_mutex_init(&J.mu, NULL);
  for (int t = 0; t < n_threads; ++t) pthread_create(&th[t], NULL, vs_worker, &J);
  for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
  pthread_mutex_destroy(&J.mu);
  free(theta);
  free(th);
  return J.status;
}

/* The n indices of largest score among score[0 .. len) (ties: the smaller
 * index), written ascending to out[0 .. n): sort by (score descending,
 * index ascending), keep the first n, sort those by index.  Returns n, or -1. */
typedef struct {
  double v;
  int64_t j;
} sj_t;

static int cmp_score_desc(const void* a, const void* b) {
  const sj_t* x = (const sj_t*)a;
  const sj_t* y = (const sj_t*)b;
  if (x->v != y->v) return x->v > y->v ? -1 : 1;
  return (x->j > y->j) - (x->j < y->j);
}

int dca_oracle_topk(const double* score, int64_t len, int64_t n, int64_t* out) {
  if (!score || !out || n < 0 || n > len) return -1;
  sj_t* a = (sj_t*)malloc(sizeof(sj_t) * (size_t)(len > 0 ? len : 1));
  if (!a) return -1;
  for (int64_t j = 0; j < len; ++j) {
    a[j].v = score[j];
    a[j].j = j;
  }
  qsort(a, (size_t)len, sizeof(sj_t), cmp_score_desc);
  for (int64_t r = 0; r < n; ++r) out[r] = a[r].j;
  qsort(out, (size_t)n, sizeof(int64_t), cmp_i64);
  free(a);
  return (int)n;
}

int dca_oracle_attention(const void* q, const void* k, const void* v, int dtype,
                         int64_t q_start, int64_t Lq, int64_t Lk, int Hq, int Hkv, int d,
                         int64_t s, int64_t w, int64_t c, double base, double yarn,
                         int reading, const int64_t* rows, int64_t n_rows,
                         const int* heads, int n_heads, double* out, double* lse,
                         int n_threads) {
  return dca_oracle_attention_mut(q, k, v, dtype, q_start, Lq, Lk, Hq, Hkv, d, s, w, c,
                                  base, yarn, reading, MUT_NONE, rows, n_rows, heads,
                                  n_heads, out, lse, n_threads);
}
