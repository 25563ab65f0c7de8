/*
 * lychee_oracle.c -- plain, slow, fp64 CPU oracle for the hybrid-head sparse
 * decode-attention step of LycheeDecode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file: it exists so that tests, the smoke check and the CPU-baseline leg of
 * the benchmark can check the CUDA library against an independent restatement of
 * the method.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it follows (page "LycheeDecode: Accelerating Long-Context LLM Inference
 * via Hybrid-Head Sparse Decoding", paper.rainbus.top/paper/2602.04541, the
 * seven-step method description):
 *   step (1)  layer 0: every head is a retrieval head; its full attention
 *             initialises the key-token set S of that head position;
 *   step (3)  retrieval head: A = softmax(q K^T / sqrt(d_k)) over the whole
 *             cache, O = A V, and S for the same head position of the next
 *             layer is argsTopK(A, k);
 *   step (4)  sparse head: O = softmax(q K[S]^T / sqrt(d_k)) V[S] over the
 *             incoming set only, and S is passed on unchanged;
 *   step (7)  roles are fixed at inference (E[z] > 0.5); here they are an input.
 * The key-token budget (30% of the sequence length) comes from the same page's
 * reproduction paragraph; the caller passes k.
 *
 * Readings where the page is silent (each one is listed in the design notes):
 *   - argsTopK is taken on the logits s_j (softmax is strictly increasing, so
 *     the set is the same and fp64 probabilities cannot underflow into false
 *     ties); ties go to the lower position; the set is returned in ascending
 *     position order and padded with -1 up to the row capacity k.
 *   - k_b = min(k_per_seq[b] (or k), n_b).
 *   - GQA: query head h reads KV head floor(h / G), G = Hq / Hkv.
 *   - A sparse head reads its own layer's K/V at the inherited positions; only
 *     the index set is shared between layers.
 *   - A set row ends at its first -1 (or at the row capacity k); a sparse head
 *     attends over all of it, which may be fewer than k_b positions, or more
 *     (a block-granular set when k_b < B).  A head with an empty set outputs 0.
 *   - Block-granular selection (the block-sparse decoding kernel of the same
 *     page; the block-level maximum scores and the k/B top blocks of the
 *     HySparse page, B = 64): a block's score is the largest logit among its
 *     positions, the max(1, floor(k_b / B)) best blocks (ties: lower block
 *     index) are taken whole, and the set lists their positions in ascending
 *     order.  Selected when the caller passes block = B > 1.
 *
 * All arithmetic is fp64.  Inputs are bf16 (raw 16-bit patterns) or fp32 and are
 * widened exactly to double when read.  The only parallelism is an optional
 * OpenMP loop over independent (batch, head) pairs; the arithmetic inside one
 * head is the same for every thread count.
 *
 * Parity pins (tests/test_oracle_pins.py): closed forms (uniform weights, n=1,
 * constant V, the two-token logistic case, GQA group constants), a library
 * special case (torch fp64 softmax(qK^T/sqrt(d))V), sparse-with-all-positions ==
 * retrieval, brute-force top-k on tiny n, and the pass-through / layer-0 rules.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_BF16 0
#define OR_FP32 1
#define OR_ROLE_SPARSE 0
#define OR_ROLE_RETRIEVAL 1

/* return codes */
#define OR_OK 0
#define OR_EARG (-1)     /* bad shape / argument */
#define OR_EINDEX (-2)   /* an incoming index is out of range or repeated */
#define OR_ELAYER0 (-3)  /* a layer-0 head is not a retrieval head (stack) */
#define OR_ENOMEM (-4)

/* Read element i of an array of dtype `dt`, widened exactly to double. */
static double rd(const void *base, size_t i, int dt) {
  if (dt == OR_BF16) {
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[i];
}

/* s_j = (sum_i q_i K_{row_j, i}) / sqrt(d) for the listed rows (step (3)/(4)). */
static void logits_rows(const void *q, size_t q_off, const void *K, size_t k_off, int d,
                        int dt, const int32_t *rows, int nrows, double *s) {
  double scale = 1.0 / sqrt((double)d);
  for (int j = 0; j < nrows; ++j) {
    size_t r = (size_t)rows[j];
    double acc = 0.0;
    for (int i = 0; i < d; ++i)
      acc += rd(q, q_off + (size_t)i, dt) * rd(K, k_off + r * (size_t)d + (size_t)i, dt);
    s[j] = acc * scale;
  }
}

/* p_j = exp(s_j - max s), returns Z = sum p_j. */
static double softmax_unnormalised(const double *s, int n, double *p) {
  double m = -INFINITY;
  for (int j = 0; j < n; ++j)
    if (s[j] > m) m = s[j];
  double z = 0.0;
  for (int j = 0; j < n; ++j) {
    p[j] = exp(s[j] - m);
    z += p[j];
  }
  return z;
}

/* O = (sum_j p_j V_{row_j}) / Z. */
static void weighted_values(const double *p, double z, const void *V, size_t v_off, int d,
                            int dt, const int32_t *rows, int nrows, double *out) {
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int j = 0; j < nrows; ++j) {
    size_t r = (size_t)rows[j];
    for (int i = 0; i < d; ++i) out[i] += p[j] * rd(V, v_off + r * (size_t)d + (size_t)i, dt);
  }
  for (int i = 0; i < d; ++i) out[i] /= z;
}

/* ---- argsTopK ------------------------------------------------------------ */

typedef struct {
  double s;
  int32_t j;
} keyed;

/* Order: larger s first; equal s -> lower position first.  A total order. */
static int by_score_then_position(const void *a, const void *b) {
  const keyed *x = (const keyed *)a, *y = (const keyed *)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->j > y->j) - (x->j < y->j);
}

static int ascending_i32(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

/* idx[0:kk] = the kk positions ranked first by (-s, j), in ascending position
 * order; idx[kk:cap] = -1.  kk = min(k, n).  Returns kk, or OR_ENOMEM. */
int oracle_topk(const double *s, int n, int k, int cap, int32_t *idx) {
  int kk = k < n ? k : n;
  if (kk < 0) kk = 0;
  keyed *tmp = (keyed *)malloc(sizeof(keyed) * (size_t)(n > 0 ? n : 1));
  if (!tmp) return OR_ENOMEM;
  for (int j = 0; j < n; ++j) {
    tmp[j].s = s[j];
    tmp[j].j = j;
  }
  qsort(tmp, (size_t)n, sizeof(keyed), by_score_then_position);
  for (int t = 0; t < kk; ++t) idx[t] = tmp[t].j;
  qsort(idx, (size_t)kk, sizeof(int32_t), ascending_i32);
  for (int t = kk; t < cap; ++t) idx[t] = -1;
  free(tmp);
  return kk;
}

/* Block-granular argsTopK: blocks [B c, min(B c + B, n)) scored by their largest
 * s_j; the kblk = max(1, floor(kb / B)) blocks ranked first by (larger score,
 * then lower block index) are taken whole.  idx[0:m] = their positions in
 * ascending order, idx[m:cap] = -1.  Returns m, or a negative code (the set
 * must fit in cap). */
int oracle_block_select(const double *s, int n, int kb, int block, int cap, int32_t *idx) {
  if (n < 1 || block < 1 || kb < 1) return OR_EARG;
  int nblk = (n + block - 1) / block;
  int kblk = kb / block;
  if (kblk < 1) kblk = 1;
  if (kblk > nblk) kblk = nblk;
  double *bs = (double *)calloc((size_t)nblk, sizeof(double));
  int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)nblk);
  int m = 0, rc = OR_OK;
  if (!bs || !sel) {
    rc = OR_ENOMEM;
    goto done;
  }
  for (int c = 0; c < nblk; ++c) {
    double best = -INFINITY;
    for (int j = c * block; j < n && j < (c + 1) * block; ++j)
      if (s[j] > best) best = s[j];
    bs[c] = best;
  }
  if (oracle_topk(bs, nblk, kblk, nblk, sel) < 0) {
    rc = OR_ENOMEM;
    goto done;
  }
  for (int i = 0; i < kblk; ++i)
    for (int j = sel[i] * block; j < n && j < (sel[i] + 1) * block; ++j) {
      if (m >= cap) {
        rc = OR_EARG;
        goto done;
      }
      idx[m++] = j;
    }
  for (int t = m; t < cap; ++t) idx[t] = -1;
done:
  free(bs);
  free(sel);
  return rc ? rc : m;
}

/* ---- one head ------------------------------------------------------------ */

/* Full (retrieval) attention of query head h of sequence b over rows [0, n).
 * out[d]; s_all[n] receives the logits (may be NULL); idx_out[cap] the top-k set
 * (block > 1: the block-granular set). */
static int retrieval_head(const void *q, size_t q_off, const void *K, const void *V,
                          size_t kv_off, int n, int d, int dt, int kb, int cap, int block,
                          double *out, double *s_all, int32_t *idx_out) {
  int32_t *rows = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  double *s = (double *)malloc(sizeof(double) * (size_t)n);
  double *p = (double *)malloc(sizeof(double) * (size_t)n);
  int rc = OR_OK;
  if (!rows || !s || !p) {
    rc = OR_ENOMEM;
    goto done;
  }
  for (int j = 0; j < n; ++j) rows[j] = j;
  logits_rows(q, q_off, K, kv_off, d, dt, rows, n, s);
  double z = softmax_unnormalised(s, n, p);
  weighted_values(p, z, V, kv_off, d, dt, rows, n, out);
  if (s_all) memcpy(s_all, s, sizeof(double) * (size_t)n);
  if (idx_out) {
    const int m = block > 1 ? oracle_block_select(s, n, kb, block, cap, idx_out)
                            : oracle_topk(s, n, kb, cap, idx_out);
    if (m < 0) rc = m;
  }
done:
  free(rows);
  free(s);
  free(p);
  return rc;
}

/* Sparse attention over the whole set S it was handed (method step (4)): the
 * row's entries before its first -1, within the row capacity cap (distinct and
 * in [0, n); a non-negative entry after a -1 is an error).  The budget k_b does
 * not bound the set: a block-granular set may hold more than k_b positions.  An
 * empty set gives out = 0.  idx_out (may be NULL) receives S unchanged (all cap
 * entries). */
static int sparse_head(const void *q, size_t q_off, const void *K, const void *V,
                       size_t kv_off, int n, int d, int dt, const int32_t *S, int cap,
                       double *out, int32_t *idx_out) {
  if (cap < 1) return OR_EARG;
  int m = 0;
  while (m < cap && S[m] >= 0) ++m;
  for (int t = m; t < cap; ++t)
    if (S[t] >= 0) return OR_EINDEX;
  if (m == 0) {
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (idx_out) memcpy(idx_out, S, sizeof(int32_t) * (size_t)cap);
    return OR_OK;
  }
  unsigned char *seen = (unsigned char *)calloc((size_t)n, 1);
  double *s = (double *)malloc(sizeof(double) * (size_t)m);
  double *p = (double *)malloc(sizeof(double) * (size_t)m);
  int rc = OR_OK;
  if (!seen || !s || !p) {
    rc = OR_ENOMEM;
    goto done;
  }
  for (int t = 0; t < m; ++t) {
    int32_t j = S[t];
    if (j < 0 || j >= n || seen[j]) {
      rc = OR_EINDEX;
      goto done;
    }
    seen[j] = 1;
  }
  logits_rows(q, q_off, K, kv_off, d, dt, S, m, s);
  double z = softmax_unnormalised(s, m, p);
  weighted_values(p, z, V, kv_off, d, dt, S, m, out);
  if (idx_out) memcpy(idx_out, S, sizeof(int32_t) * (size_t)cap);
done:
  free(seen);
  free(s);
  free(p);
  return rc;
}

/* ---- one layer ----------------------------------------------------------- */

static int budget(const int32_t *k_per_seq, int b, int k, int n) {
  int kb = k_per_seq ? k_per_seq[b] : k;
  if (kb > k) kb = k;
  return kb < n ? kb : n;
}

static int check_shape(int B, int Hq, int Hkv, int d, int N_max, int k, int dt) {
  if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || N_max < 1 || k < 1) return OR_EARG;
  if (Hq % Hkv != 0) return OR_EARG;
  if (dt != OR_BF16 && dt != OR_FP32) return OR_EARG;
  return OR_OK;
}

/*
 * One hybrid-head layer (steps (3) and (4)).
 *   q        [B, Hq, d]             dtype dt
 *   K, V     [B, Hkv, N_max, d]     dtype dt
 *   seqlens  [B]                    1 <= n_b <= N_max
 *   k_per_seq[B] or NULL            k_b = min(k_per_seq[b] or k, n_b)
 *   role     [Hq]                   1 = retrieval, 0 = sparse
 *   idx_in   [B, Hq, k]             rows of sparse heads are read (entries before the
 *                                   first -1, up to k)
 *   out      [B, Hq, d]   double
 *   logits   [B, Hq, N_max] double or NULL: s_j of retrieval heads for j < n_b
 *   idx_out  [B, Hq, k]             retrieval: top-k set; sparse: idx_in row copied
 *   block    1: token-level argsTopK; B > 1: block-granular selection (k >= B)
 *   nthreads OpenMP threads over (b, h) pairs (<= 0: library default)
 * Returns OR_OK or a negative code.
 */
int oracle_hybrid_layer(int B, int Hq, int Hkv, int d, int N_max, int k, int dt, int block,
                        const void *q, const void *K, const void *V, const int32_t *seqlens,
                        const int32_t *k_per_seq, const uint8_t *role, const int32_t *idx_in,
                        double *out, double *logits, int32_t *idx_out, int nthreads) {
  int rc = check_shape(B, Hq, Hkv, d, N_max, k, dt);
  if (rc) return rc;
  if (block < 1 || (block > 1 && k < block)) return OR_EARG;
  for (int b = 0; b < B; ++b)
    if (seqlens[b] < 1 || seqlens[b] > N_max) return OR_EARG;
  int G = Hq / Hkv;
  int err = OR_OK;
  int pairs = B * Hq;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int bh = 0; bh < pairs; ++bh) {
    int b = bh / Hq, h = bh % Hq, g = h / G;
    int n = seqlens[b];
    int kb = budget(k_per_seq, b, k, n);
    size_t q_off = ((size_t)b * Hq + h) * (size_t)d;
    size_t kv_off = ((size_t)b * Hkv + g) * (size_t)N_max * (size_t)d;
    size_t row = (size_t)b * Hq + h;
    int r;
    if (role[h] == OR_ROLE_RETRIEVAL) {
      r = retrieval_head(q, q_off, K, V, kv_off, n, d, dt, kb, k, block, out + row * (size_t)d,
                         logits ? logits + row * (size_t)N_max : NULL,
                         idx_out ? idx_out + row * (size_t)k : NULL);
    } else {
      if (!idx_in) {
        r = OR_EARG;
      } else {
        r = sparse_head(q, q_off, K, V, kv_off, n, d, dt, idx_in + row * (size_t)k, k,
                        out + row * (size_t)d, idx_out ? idx_out + row * (size_t)k : NULL);
      }
    }
    if (r) {
#ifdef _OPENMP
#pragma omp critical
#endif
      err = r;
    }
  }
  return err;
}

/*
 * L chained layers (steps (1), (3), (4)): S of head position h after layer l is
 * the input S of head position h at layer l+1.
 *   q          [L, B, Hq, d]
 *   Ks, Vs     L pointers to [B, Hkv, N_max, d]
 *   role       [L, Hq]; row 0 must be all retrieval (step (1))
 *   out        [L, B, Hq, d] double
 *   idx_layers [L, B, Hq, k] or NULL: S leaving each layer
 *   idx_final  [B, Hq, k]: S leaving layer L-1
 */
int oracle_stack(int L, int B, int Hq, int Hkv, int d, int N_max, int k, int dt, int block,
                 const void *q, const void *const *Ks, const void *const *Vs,
                 const int32_t *seqlens, const int32_t *k_per_seq, const uint8_t *role,
                 double *out, int32_t *idx_layers, int32_t *idx_final, int nthreads) {
  int rc = check_shape(B, Hq, Hkv, d, N_max, k, dt);
  if (rc) return rc;
  if (L < 1) return OR_EARG;
  for (int h = 0; h < Hq; ++h)
    if (role[h] != OR_ROLE_RETRIEVAL) return OR_ELAYER0;
  size_t set_elems = (size_t)B * Hq * k;
  int32_t *cur = (int32_t *)malloc(sizeof(int32_t) * set_elems);
  int32_t *nxt = (int32_t *)malloc(sizeof(int32_t) * set_elems);
  if (!cur || !nxt) {
    free(cur);
    free(nxt);
    return OR_ENOMEM;
  }
  for (size_t t = 0; t < set_elems; ++t) cur[t] = -1;
  size_t qsz = (dt == OR_BF16) ? 2 : 4;
  for (int l = 0; l < L && rc == OR_OK; ++l) {
    const char *ql = (const char *)q + (size_t)l * B * Hq * d * qsz;
    rc = oracle_hybrid_layer(B, Hq, Hkv, d, N_max, k, dt, block, ql, Ks[l], Vs[l], seqlens, k_per_seq,
                             role + (size_t)l * Hq, cur, out + (size_t)l * B * Hq * d, NULL, nxt,
                             nthreads);
    if (idx_layers) memcpy(idx_layers + (size_t)l * set_elems, nxt, sizeof(int32_t) * set_elems);
    int32_t *t = cur;
    cur = nxt;
    nxt = t;
  }
  if (rc == OR_OK && idx_final) memcpy(idx_final, cur, sizeof(int32_t) * set_elems);
  free(cur);
  free(nxt);
  return rc;
}

/* Attention weights A_j = softmax(s)_j of one query head over rows [0, n) of its
 * KV group (step (3)); used by the tests to pin normalisation. */
int oracle_attention_weights(int d, int n, int dt, const void *q, const void *Kg, double *A) {
  if (d < 1 || n < 1) return OR_EARG;
  int32_t *rows = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  double *s = (double *)malloc(sizeof(double) * (size_t)n);
  if (!rows || !s) {
    free(rows);
    free(s);
    return OR_ENOMEM;
  }
  for (int j = 0; j < n; ++j) rows[j] = j;
  logits_rows(q, 0, Kg, 0, d, dt, rows, n, s);
  double z = softmax_unnormalised(s, n, A);
  for (int j = 0; j < n; ++j) A[j] /= z;
  free(rows);
  free(s);
  return OR_OK;
}
