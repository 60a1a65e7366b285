/*
 * g4attn oracle -- a plain, slow float64 CPU restatement of the Gemma 4
 * decoder attention layer (prologue + sliding / global attention + decode).
 *
 * THIS IS TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load it.  The CUDA library never links,
 * includes or calls anything in this directory, and this file includes nothing
 * from the CUDA library: the two implementations share no code.
 *
 * Everything is computed in float64 from the exact values of the input bits
 * (bf16 or fp32).  Nothing is blocked, fused or reordered: every output row is
 * an explicit loop over the keys its query may see.
 *
 * Sources (page title, section):
 *  - "Gemma 4" (Keras port docs), "What changed from Gemma 3": plain-weight
 *    RMSNorm, zero-pad partial rope, K=V global MQA, blockwise bidirectional
 *    image attention on sliding layers only.
 *  - "gemma4-pt-claude" README, "Supported Models" (QK-norm and V-norm on all
 *    variants), "Key architectural features" (GQA, K=V), "Attention Backend
 *    Notes" (norms multiply by the weight, one-initialised), "KV Cache"
 *    (rolling sliding-window caches, overflow raises).
 *  - "Gemma 4" overview blog (vinija.ai), "Sliding-window attention",
 *    "Global attention layers", "Dual RoPE configurations" (2x2 rotation of
 *    each two-dimensional subspace), "Shared KV Cache".
 *
 * Readings taken where the pages are silent or ambiguous (each is a choice,
 * not a page fact): window = w keys including the query itself; the image
 * block is added to the window as a union; the global layer rotates the pairs
 * (k, k + d/2) for k < R = fraction*d/2 with frequency theta^(-2k/d) and leaves
 * the other pairs untouched (a zero-padded frequency vector); pairs are split
 * halves (rotate-half); positions are 0-based token indices; the KV head of
 * query head h is h / (Hq/Hkv); a chunk of a cached prefill sees keys up to
 * its own last position, so an image block cut by the chunk's end is seen up
 * to there (rows of earlier chunks are not recomputed).
 *
 * Parity status of the readings: the rotated-dimension selection, the pairing
 * convention, eps and the softmax scale are not fixed by any value the pages
 * print ("parity unpinned" for those choices); every other step is pinned by
 * the tests under tests/test_oracle.py (closed forms, invariants, brute force).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BF16 0
#define OR_FP32 1
#define OR_FP64 2 /* exact values, e.g. a cache holding oracle results */

#define OR_SLIDING 0
#define OR_GLOBAL 1
#define OR_BIDIRECTIONAL 2 /* the vision tower's attention: every key of the sequence */

#define OR_ROPE_ZEROPAD 0 /* the build's reading: zero-padded frequency vector */
#define OR_ROPE_PREFIX 1  /* alternative reading: rotate the first fraction*d dims */

typedef struct {
  int layer_type;          /* OR_SLIDING, OR_GLOBAL or OR_BIDIRECTIONAL */
  int window;              /* keys a sliding query sees, itself included */
  double rotary_fraction;  /* 1.0 on sliding layers, 0.25 on global layers */
  double rope_theta;       /* 1e4 sliding, 1e6 global */
  int k_eq_v;              /* V comes from the same raw vector as K */
  int num_heads;           /* Hq */
  int num_kv_heads;        /* Hkv */
  int head_dim;            /* d */
  double softmax_scale;
  double rms_eps;
  int rope_mode;           /* OR_ROPE_ZEROPAD (default) or OR_ROPE_PREFIX */
  int window_plus_one;     /* 1: the printed j in [i-w, i] reading (w+1 keys) */
  double logit_softcap;    /* 0: none; else s <- cap * tanh(s / cap) */
} or_layer;

/* Exact value of element i of a bf16 (raw bits), fp32 or fp64 array. */
static double or_load(const void *p, long i, int dtype) {
  if (dtype == OR_FP64) return ((const double *)p)[i];
  if (dtype == OR_FP32) return (double)((const float *)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* RMSNorm over one head: y = x / sqrt(mean(x^2) + eps) * w.  The weight is
 * used as it is (no 1 + w offset); w == NULL is the weightless V-norm. */
void or_rms_normalize(const double *x, int d, double eps, const double *w,
                      double *y) {
  double ss = 0.0;
  for (int k = 0; k < d; ++k) ss += x[k] * x[k];
  double r = sqrt(ss / (double)d + eps);
  for (int k = 0; k < d; ++k) y[k] = (x[k] / r) * (w ? w[k] : 1.0);
}

/* Number of rotated pairs R for a layer. */
int or_rotated_pairs(const or_layer *L) {
  return (int)llround(L->rotary_fraction * (double)L->head_dim / 2.0);
}

/* RoPE at integer position pos, in place on one head.
 * Zero-pad reading: pair k is (x[k], x[k + d/2]); for k < R its angle is
 * pos * theta^(-2k/d), for k >= R the frequency is zero and the pair passes
 * through untouched.  Each pair is multiplied by the 2x2 rotation
 * [[cos a, -sin a], [sin a, cos a]]. */
void or_rope(double *x, int d, long pos, const or_layer *L) {
  int R = or_rotated_pairs(L);
  if (L->rope_mode == OR_ROPE_PREFIX) {
    /* rotate the contiguous first rd = 2R dims as a rotate-half RoPE of
     * width rd with frequencies theta^(-2k/rd); the rest passes through */
    int rd = 2 * R;
    for (int k = 0; k < R; ++k) {
      double f = pow(L->rope_theta, -2.0 * (double)k / (double)rd);
      double a = (double)pos * f;
      double c = cos(a), s = sin(a);
      double x0 = x[k], x1 = x[k + R];
      x[k] = x0 * c - x1 * s;
      x[k + R] = x0 * s + x1 * c;
    }
    return;
  }
  int half = d / 2;
  for (int k = 0; k < half; ++k) {
    if (k >= R) continue; /* zero frequency: exact pass-through */
    double f = pow(L->rope_theta, -2.0 * (double)k / (double)d);
    double a = (double)pos * f;
    double c = cos(a), s = sin(a);
    double x0 = x[k], x1 = x[k + half];
    x[k] = x0 * c - x1 * s;
    x[k + half] = x0 * s + x1 * c;
  }
}

/* Query prologue for one (token, head): q_hat = RoPE_pos(RMSNorm(q) * w_q). */
void or_prologue_q(const or_layer *L, const void *q_raw, long off, int dtype,
                   const void *wq, int w_dtype, long pos, double *out) {
  int d = L->head_dim;
  double *x = (double *)malloc(sizeof(double) * 2 * d);
  double *w = x + d;
  for (int k = 0; k < d; ++k) {
    x[k] = or_load(q_raw, off + k, dtype);
    w[k] = or_load(wq, k, w_dtype);
  }
  or_rms_normalize(x, d, L->rms_eps, w, out);
  or_rope(out, d, pos, L);
  free(x);
}

/* Key/value prologue for one (token, KV head):
 *   k_hat = RoPE_pos(RMSNorm(k) * w_k),  v_hat = RMSNorm(v) (no weight).
 * With k_eq_v the value is normalised from the same raw vector as the key.
 * Either output may be NULL. */
void or_prologue_kv(const or_layer *L, const void *k_raw, const void *v_raw,
                    long off, int dtype, const void *wk, int w_dtype, long pos,
                    double *k_out, double *v_out) {
  int d = L->head_dim;
  double *x = (double *)malloc(sizeof(double) * 2 * d);
  double *w = x + d;
  if (k_out) {
    for (int k = 0; k < d; ++k) {
      x[k] = or_load(k_raw, off + k, dtype);
      w[k] = or_load(wk, k, w_dtype);
    }
    or_rms_normalize(x, d, L->rms_eps, w, k_out);
    or_rope(k_out, d, pos, L);
  }
  if (v_out) {
    const void *src = L->k_eq_v ? k_raw : v_raw;
    for (int k = 0; k < d; ++k) x[k] = or_load(src, off + k, dtype);
    or_rms_normalize(x, d, L->rms_eps, NULL, v_out);
  }
  free(x);
}

/* Keys query i may see, as the closed interval [*lo, *hi].
 * Sliding text row: the w most recent positions, itself included.
 * Sliding row inside an image block [s, e): the window united with the whole
 * block (both contain i, so the union is an interval).
 * Global row: every earlier position and itself; block ids are ignored.
 * Bidirectional row (the vision tower's ViT attention, "gemma4-pt-claude"
 * README, "Key architectural features"): every one of the T positions; block
 * ids are ignored.
 * ids is the row of block ids of this sequence (-1 = text) or NULL. */
void or_interval(const or_layer *L, const int *ids, int T, int i, int *lo,
                 int *hi) {
  if (L->layer_type == OR_GLOBAL) {
    *lo = 0;
    *hi = i;
    return;
  }
  if (L->layer_type == OR_BIDIRECTIONAL) {
    *lo = 0;
    *hi = T - 1;
    return;
  }
  int w = L->window + (L->window_plus_one ? 1 : 0);
  int a = i - w + 1;
  if (a < 0) a = 0;
  int b = i;
  if (ids && ids[i] >= 0) {
    int s = i, e = i + 1;
    while (s > 0 && ids[s - 1] == ids[i]) --s;
    while (e < T && ids[e] == ids[i]) ++e;
    if (s < a) a = s;
    if (e - 1 > b) b = e - 1;
  }
  *lo = a;
  *hi = b;
}

/* Masked softmax attention of one query over keys lo..hi (explicit loop):
 *   o = sum_j e^{s_j - M} v_j / sum_j e^{s_j - M},  s_j = scale * q . k_j,
 * and with a logit soft-cap c > 0 ("gemma4-pt-claude" README, "Attention
 * Backend": attn_logits_soft_cap; the page prints no formula, the reading
 * is the usual tanh cap, the form the "Gemma 4" Keras docs' argument table
 * names for the output-logit cap) s_j <- c * tanh(s_j / c) before the
 * softmax.
 * keep (indexed by key position, NULL = every key kept) drops padding keys
 * ("Gemma4ConditionalGenerate" arguments: attention_mask 1 = keep, 0 =
 * padding); a query left with no key gets o = 0.
 * kbase/vbase point to key/value rows spaced `stride` doubles apart.  The
 * two-pass form (max first) is the plain definition; no online rescaling. */
static void or_attend(const double *q, const double *kbase,
                      const double *vbase, long stride, int lo, int hi, int d,
                      double scale, double cap, const unsigned char *keep,
                      double *s_buf, double *o) {
  double m = -INFINITY;
  for (int j = lo; j <= hi; ++j) {
    if (keep && !keep[j]) continue;
    const double *kj = kbase + (long)j * stride;
    double dot = 0.0;
    for (int k = 0; k < d; ++k) dot += q[k] * kj[k];
    double s = scale * dot;
    if (cap > 0.0) s = cap * tanh(s / cap);
    s_buf[j - lo] = s;
    if (s > m) m = s;
  }
  double den = 0.0;
  for (int k = 0; k < d; ++k) o[k] = 0.0;
  if (m == -INFINITY) return; /* no key left */
  for (int j = lo; j <= hi; ++j) {
    if (keep && !keep[j]) continue;
    double p = exp(s_buf[j - lo] - m);
    den += p;
    const double *vj = vbase + (long)j * stride;
    for (int k = 0; k < d; ++k) o[k] += p * vj[k];
  }
  for (int k = 0; k < d; ++k) o[k] /= den;
}

/* ------------------------------------------------------------------ */
/* prefill                                                              */

typedef struct {
  const or_layer *L;
  int B, T;   /* T query rows per sequence (the chunk) */
  int p0;     /* position of the chunk's first row */
  const void *q_raw, *wq;
  int dtype, w_dtype;
  const int *block_ids;      /* [B][p0 + T] */
  const unsigned char *keep; /* [B][p0 + T] or NULL */
  const int *rows;
  int n_rows;
  const double *khat, *vhat; /* [B][p0 + T][Hkv][d] */
  double *out;               /* [B][n_rows][Hq][d] */
  int tid, nthreads;
  const double *qhat;        /* [B][T][Hq][d] post-prologue queries, or NULL */
} or_prefill_job;

static void *or_prefill_worker(void *arg) {
  or_prefill_job *J = (or_prefill_job *)arg;
  const or_layer *L = J->L;
  int d = L->head_dim, Hq = L->num_heads, Hkv = L->num_kv_heads;
  int g = Hq / Hkv;
  double *q = (double *)malloc(sizeof(double) * d);
  const int Tk = J->p0 + J->T; /* positions a row of the chunk may see */
  double *s = (double *)malloc(sizeof(double) * (Tk + 1));
  long items = (long)J->B * J->n_rows * Hq;
  for (long it = J->tid; it < items; it += J->nthreads) {
    int h = (int)(it % Hq);
    int r = (int)((it / Hq) % J->n_rows);
    int b = (int)(it / ((long)Hq * J->n_rows));
    int i = J->rows ? J->rows[r] : r; /* row of the chunk */
    int pos = J->p0 + i;
    long qoff = (((long)b * J->T + i) * Hq + h) * d;
    if (J->qhat)
      memcpy(q, J->qhat + qoff, sizeof(double) * d);
    else
      or_prologue_q(L, J->q_raw, qoff, J->dtype, J->wq, J->w_dtype, pos, q);
    int lo, hi;
    or_interval(L, J->block_ids ? J->block_ids + (long)b * Tk : NULL, Tk, pos,
                &lo, &hi);
    int kvh = h / g;
    const double *kb = J->khat + ((long)b * Tk * Hkv + kvh) * d;
    const double *vb = J->vhat + ((long)b * Tk * Hkv + kvh) * d;
    double *o = J->out + (((long)b * J->n_rows + r) * Hq + h) * d;
    or_attend(q, kb, vb, (long)Hkv * d, lo, hi, d, L->softmax_scale,
              L->logit_softcap, J->keep ? J->keep + (long)b * Tk : NULL, s, o);
  }
  free(q);
  free(s);
  return NULL;
}

typedef struct {
  const or_layer *L;
  int B, T;
  int p0; /* position of the first token */
  const void *k_raw, *v_raw, *wk;
  int dtype, w_dtype;
  double *khat, *vhat;
  int tid, nthreads;
} or_kv_job;

static void *or_kv_worker(void *arg) {
  or_kv_job *J = (or_kv_job *)arg;
  const or_layer *L = J->L;
  int d = L->head_dim, Hkv = L->num_kv_heads;
  long items = (long)J->B * J->T * Hkv;
  for (long it = J->tid; it < items; it += J->nthreads) {
    long t = J->p0 + (it / Hkv) % J->T;
    long off = it * d;
    or_prologue_kv(L, J->k_raw, J->v_raw, off, J->dtype, J->wk, J->w_dtype, t,
                   J->khat + off, J->vhat + off);
  }
  return NULL;
}

static void or_run(void *(*fn)(void *), void *jobs, size_t job_size,
                   int nthreads) {
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
  for (int t = 0; t < nthreads; ++t)
    pthread_create(&th[t], NULL, fn, (char *)jobs + job_size * t);
  for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* Post-prologue keys and values of T tokens at positions p0 .. p0+T-1:
 * khat, vhat [B][T][Hkv][d].  k_raw/v_raw are [B][T][Hkv][d] in `dtype`;
 * v_raw is ignored with k_eq_v. */
void or_prefill_kv_at(const or_layer *L, int B, int T, int p0, const void *k_raw,
                      const void *v_raw, const void *wk, int dtype, int w_dtype,
                      double *khat, double *vhat, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  or_kv_job *jobs = (or_kv_job *)calloc(nthreads, sizeof(or_kv_job));
  for (int t = 0; t < nthreads; ++t) {
    or_kv_job j = {L, B, T, p0, k_raw, v_raw, wk, dtype, w_dtype, khat, vhat,
                   t, nthreads};
    jobs[t] = j;
  }
  or_run(or_kv_worker, jobs, sizeof(or_kv_job), nthreads);
  free(jobs);
}

/* The same for a whole prompt (positions 0 .. T-1). */
void or_prefill_kv(const or_layer *L, int B, int T, const void *k_raw,
                   const void *v_raw, const void *wk, int dtype, int w_dtype,
                   double *khat, double *vhat, int nthreads) {
  or_prefill_kv_at(L, B, T, 0, k_raw, v_raw, wk, dtype, w_dtype, khat, vhat,
                   nthreads);
}

/* Cached (chunked) prefill ("gemma4-pt-claude" README, "Tests": a cached
 * path must reproduce the uncached forward pass, image spans included):
 * the T query rows of a chunk at positions p0 .. p0+T-1 attend, each over
 * the interval of its position in a prompt of p0 + T tokens, to keys held
 * for all p0 + T positions.  q_raw is [B][T][Hq][d]; block_ids, when given,
 * is [B][p0 + T] (an image block is seen up to the chunk's last position);
 * khat/vhat are [B][p0 + T][Hkv][d]; rows lists rows of the chunk (NULL =
 * all T, n_rows = T); out is [B][n_rows][Hq][d].  keep, when given, is the
 * padding mask [B][p0 + T] (1 = keep, 0 = padding key). */
void or_prefill_chunk_rows_masked(const or_layer *L, int B, int T, int p0,
                                  const void *q_raw, const void *wq, int dtype,
                                  int w_dtype, const int *block_ids,
                                  const unsigned char *keep,
                                  const double *khat, const double *vhat,
                                  const int *rows, int n_rows, double *out,
                                  int nthreads) {
  if (nthreads < 1) nthreads = 1;
  or_prefill_job *jobs =
      (or_prefill_job *)calloc(nthreads, sizeof(or_prefill_job));
  for (int t = 0; t < nthreads; ++t) {
    or_prefill_job j = {L,     B,       T,         p0,   q_raw,  wq,
                        dtype, w_dtype, block_ids, keep, rows,   n_rows,
                        khat,  vhat,    out,       t,    nthreads, NULL};
    jobs[t] = j;
  }
  or_run(or_prefill_worker, jobs, sizeof(or_prefill_job), nthreads);
  free(jobs);
}

/* The attention of or_prefill_chunk_rows_masked from given post-prologue
 * queries qhat [B][T][Hq][d] (float64) instead of raw ones: the same row
 * intervals, padding and soft-cap, the same loop.  Lets a caller model a
 * storage format of q_hat, k_hat, v_hat (values rounded before they are
 * attended), with every step after the prologue unchanged. */
void or_attend_rows(const or_layer *L, int B, int T, int p0, const double *qhat,
                    const int *block_ids, const unsigned char *keep,
                    const double *khat, const double *vhat, const int *rows,
                    int n_rows, double *out, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  or_prefill_job *jobs =
      (or_prefill_job *)calloc(nthreads, sizeof(or_prefill_job));
  for (int t = 0; t < nthreads; ++t) {
    or_prefill_job j = {L,      B,    T,         p0,   NULL,   NULL,
                        OR_FP64, OR_FP64, block_ids, keep, rows, n_rows,
                        khat,   vhat, out,       t,    nthreads, qhat};
    jobs[t] = j;
  }
  or_run(or_prefill_worker, jobs, sizeof(or_prefill_job), nthreads);
  free(jobs);
}

/* Post-prologue queries RoPE_pos(RMSNorm(q) * w_q) of every token, float64
 * [B][T][Hq][d], the tokens at positions p0 .. p0 + T - 1. */
void or_prologue_q_all(const or_layer *L, int B, int T, int p0, const void *q_raw,
                       const void *wq, int dtype, int w_dtype, double *out) {
  int d = L->head_dim, Hq = L->num_heads;
  for (long it = 0; it < (long)B * T * Hq; ++it) {
    long t = (it / Hq) % T;
    or_prologue_q(L, q_raw, it * d, dtype, wq, w_dtype, p0 + t, out + it * d);
  }
}

/* The same with every key kept. */
void or_prefill_chunk_rows(const or_layer *L, int B, int T, int p0,
                           const void *q_raw, const void *wq, int dtype,
                           int w_dtype, const int *block_ids,
                           const double *khat, const double *vhat,
                           const int *rows, int n_rows, double *out,
                           int nthreads) {
  or_prefill_chunk_rows_masked(L, B, T, p0, q_raw, wq, dtype, w_dtype,
                               block_ids, NULL, khat, vhat, rows, n_rows, out,
                               nthreads);
}

/* Attention output of the listed query rows of a whole prompt, given
 * khat/vhat from or_prefill_kv.  q_raw is [B][T][Hq][d]; rows lists query
 * positions (NULL = all T rows, n_rows = T); out is [B][n_rows][Hq][d]. */
void or_prefill_rows(const or_layer *L, int B, int T, const void *q_raw,
                     const void *wq, int dtype, int w_dtype,
                     const int *block_ids, const double *khat,
                     const double *vhat, const int *rows, int n_rows,
                     double *out, int nthreads) {
  or_prefill_chunk_rows(L, B, T, 0, q_raw, wq, dtype, w_dtype, block_ids, khat,
                        vhat, rows, n_rows, out, nthreads);
}

/* ------------------------------------------------------------------ */
/* decode                                                               */

/* One decode step for the listed sequences.
 *
 * The cache (cache_k, cache_v: [B][Hkv][C][d] in cache_dtype) holds the
 * post-prologue keys/values of positions 0..len[b]-1; a rolling cache keeps
 * position p at slot p % C.  If k_new is non-NULL the new token (raw K/V of
 * the layer that owns the cache, [B][Hkv][d]) is appended at position
 * P = len[b] through the key/value prologue of Lkv; otherwise (a KV-shared
 * layer reading a cache that already holds the new token) P = len[b] - 1.
 * The query (q_raw [B][Hq][d], prologue of Lq at position P) attends over
 * the interval of row P: decode is the last row of a prefill over P + 1
 * tokens.  keep, when given, is the padding mask of the prompt positions,
 * [B][mask_len] ("Gemma4ConditionalGenerate" arguments: attention_mask,
 * 1 = keep, 0 = padding): position p < mask_len is dropped when its entry
 * is 0; later positions (the generated tokens) are kept.  out is
 * [n_seqs][Hq][d].  Returns 0, or -1 if a key the query needs is not in the
 * cache. */
typedef struct {
  const or_layer *Lq, *Lkv;
  const void *q_raw, *wq;
  int dtype, w_dtype;
  const void *cache_k, *cache_v;
  int cache_dtype, C, rolling;
  const int *len;
  const void *k_new, *v_new, *wk;
  const unsigned char *keep; /* [B][mask_len] or NULL */
  int mask_len;
  const int *seqs;
  int n_seqs;
  double *out;
  int tid, nthreads;
  int err;
} or_decode_job;

static void *or_decode_worker(void *arg) {
  or_decode_job *J = (or_decode_job *)arg;
  const or_layer *Lq = J->Lq;
  int d = Lq->head_dim, Hq = Lq->num_heads, Hkv = Lq->num_kv_heads;
  int g = Hq / Hkv;
  long items = (long)J->n_seqs * Hq;
  double *q = (double *)malloc(sizeof(double) * d);
  double *kn = (double *)malloc(sizeof(double) * d);
  double *vn = (double *)malloc(sizeof(double) * d);
  for (long it = J->tid; it < items; it += J->nthreads) {
    int h = (int)(it % Hq);
    int si = (int)(it / Hq);
    int b = J->seqs ? J->seqs[si] : si;
    int kvh = h / g;
    int append = J->k_new != NULL;
    long P = append ? J->len[b] : (long)J->len[b] - 1;
    or_prologue_q(Lq, J->q_raw, ((long)b * Hq + h) * d, J->dtype, J->wq,
                  J->w_dtype, P, q);
    if (append)
      or_prologue_kv(J->Lkv, J->k_new, J->v_new, ((long)b * Hkv + kvh) * d,
                     J->dtype, J->wk, J->w_dtype, P, kn, vn);
    long lo = 0;
    if (Lq->layer_type == OR_SLIDING) {
      int w = Lq->window + (Lq->window_plus_one ? 1 : 0);
      lo = P - w + 1;
      if (lo < 0) lo = 0;
    }
    /* the keys must still be in the cache */
    long oldest = J->rolling ? P - J->C + 1 : 0;
    if (lo < oldest || (!J->rolling && P >= J->C)) {
      J->err = -1;
      continue;
    }
    long n = P - lo + 1;
    double *kk = (double *)malloc(sizeof(double) * n * d);
    double *vv = (double *)malloc(sizeof(double) * n * d);
    double *s = (double *)malloc(sizeof(double) * n);
    unsigned char *kp = (unsigned char *)malloc(n); /* padding mask of lo..P */
    for (long p = lo; p <= P; ++p) {
      double *kd = kk + (p - lo) * d, *vd = vv + (p - lo) * d;
      kp[p - lo] = (J->keep && p < J->mask_len)
                       ? (J->keep[(long)b * J->mask_len + p] != 0)
                       : 1;
      if (append && p == P) {
        memcpy(kd, kn, sizeof(double) * d);
        memcpy(vd, vn, sizeof(double) * d);
        continue;
      }
      long slot = J->rolling ? p % J->C : p;
      long base = (((long)b * Hkv + kvh) * J->C + slot) * d;
      for (int k = 0; k < d; ++k) {
        kd[k] = or_load(J->cache_k, base + k, J->cache_dtype);
        vd[k] = or_load(J->cache_v, base + k, J->cache_dtype);
      }
    }
    or_attend(q, kk, vv, d, 0, (int)(n - 1), d, Lq->softmax_scale,
              Lq->logit_softcap, kp, s, J->out + ((long)si * Hq + h) * d);
    free(kk);
    free(vv);
    free(s);
    free(kp);
  }
  free(q);
  free(kn);
  free(vn);
  return NULL;
}

int or_decode(const or_layer *Lq, const or_layer *Lkv, const void *q_raw,
              const void *wq, int dtype, int w_dtype, const void *cache_k,
              const void *cache_v, int cache_dtype, int C, int rolling,
              const int *len, const void *k_new, const void *v_new,
              const void *wk, const unsigned char *keep, int mask_len,
              const int *seqs, int n_seqs, double *out, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  or_decode_job *jobs =
      (or_decode_job *)calloc(nthreads, sizeof(or_decode_job));
  for (int t = 0; t < nthreads; ++t) {
    or_decode_job j = {Lq,      Lkv,     q_raw,       wq,    dtype,   w_dtype,
                       cache_k, cache_v, cache_dtype, C,     rolling, len,
                       k_new,   v_new,   wk,          keep,  mask_len, seqs,
                       n_seqs,  out,     t,           nthreads, 0};
    jobs[t] = j;
  }
  or_run(or_decode_worker, jobs, sizeof(or_decode_job), nthreads);
  int err = 0;
  for (int t = 0; t < nthreads; ++t)
    if (jobs[t].err) err = jobs[t].err;
  free(jobs);
  return err;
}

/* ------------------------------------------------------------------ */
/* split-KV partial softmax and its combine                             */

/* Partial softmax of one query over keys lo..hi (rows `stride` apart):
 * m = max_j s_j, l = sum_j e^{s_j - m}, o_tilde = sum_j e^{s_j - m} v_j. */
void or_partial(const double *q, const double *kbase, const double *vbase,
                long stride, int lo, int hi, int d, double scale, double *m,
                double *l, double *o_tilde) {
  double mm = -INFINITY;
  for (int j = lo; j <= hi; ++j) {
    double dot = 0.0;
    for (int k = 0; k < d; ++k) dot += q[k] * kbase[(long)j * stride + k];
    if (scale * dot > mm) mm = scale * dot;
  }
  double ll = 0.0;
  for (int k = 0; k < d; ++k) o_tilde[k] = 0.0;
  for (int j = lo; j <= hi; ++j) {
    double dot = 0.0;
    for (int k = 0; k < d; ++k) dot += q[k] * kbase[(long)j * stride + k];
    double p = exp(scale * dot - mm);
    ll += p;
    for (int k = 0; k < d; ++k) o_tilde[k] += p * vbase[(long)j * stride + k];
  }
  *m = mm;
  *l = ll;
}

/* Log-sum-exp merge of n partials:
 *   o = sum_c e^{m_c - M} o_tilde_c / sum_c e^{m_c - M} l_c,  M = max_c m_c.
 * o_tilde is [n][d]. */
void or_combine(int n, const double *m, const double *l,
                const double *o_tilde, int d, double *o) {
  double M = -INFINITY;
  for (int c = 0; c < n; ++c)
    if (m[c] > M) M = m[c];
  double den = 0.0;
  for (int k = 0; k < d; ++k) o[k] = 0.0;
  for (int c = 0; c < n; ++c) {
    double a = exp(m[c] - M);
    den += a * l[c];
    for (int k = 0; k < d; ++k) o[k] += a * o_tilde[(long)c * d + k];
  }
  for (int k = 0; k < d; ++k) o[k] /= den;
}
