/*
 * g4attn -- Gemma 4 decoder attention layer on NVIDIA B200 (sm_100a).
 *
 * C ABI of libg4attn.so.  Every pointer argument is a plain pointer: "device"
 * means memory the calling process allocated on the current CUDA device,
 * "host" means ordinary process memory.  All tensors are dense row-major
 * (last dimension contiguous).  The library never allocates, frees or
 * synchronises device memory except where a function says so; the caller
 * owns every buffer, the stream and the workspace.  Calls enqueue work on the
 * given stream (a cudaStream_t passed as void*, NULL = the legacy default
 * stream) and return without waiting.
 *
 * Page passages that define the operations (page title, section):
 *  [K1] "Gemma 4" (Keras port docs), "What changed from Gemma 3":
 *       plain-weight RMSNorm; zero-pad partial rope on partial_rotary_factor
 *       of each head; K=V global MQA at global_head_dim 512; image tokens
 *       attend bidirectionally within each image block on sliding layers,
 *       global layers stay causal; a tail of layers reuses an earlier
 *       layer's K/V.
 *  [K2] "Gemma 4" (Keras port docs), "Gemma4Model" argument table:
 *       num_heads, num_kv_heads, num_global_kv_heads, head_dim,
 *       global_head_dim, k_eq_v, sliding_window, partial_rotary_factor,
 *       num_kv_shared_layers.
 *  [K3] "Gemma 4" (Keras port docs), "Gemma4ConditionalGenerate": decoding
 *       is text-only over the per-layer KV cache.
 *  [P1] "gemma4-pt-claude" README, "Supported Models": every variant uses
 *       QK-norm and V-norm; "Attention Backend Notes": norms multiply by the
 *       weight (x_normed * weight).
 *  [P2] "gemma4-pt-claude" README, "KV Cache": the cache is sized for
 *       prompt + new tokens and a write past its end is an error;
 *       sliding-window layers may use a rolling cache of
 *       max(window, prompt) slots; global layers keep the full context.
 *  [V1] "Gemma 4" overview blog, "Sliding-window attention" and "Global
 *       attention layers": a sliding query sees a window of recent keys, a
 *       global query every earlier key.
 *  [V2] "Gemma 4" overview blog, "Dual RoPE configurations": standard RoPE
 *       on sliding layers, proportional/pruned RoPE on global layers, each
 *       two-dimensional subspace rotated by the 2x2 rotation matrix.
 *  [V3] "Gemma 4" overview blog, "Shared KV Cache": later layers reuse the
 *       K/V of the most recent earlier layer of the same type and compute
 *       only their own queries.
 *  [K4] "Gemma 4" (Keras port docs), "Gemma4ConditionalGenerate" argument
 *       table: attention_mask (batch, seq), 1 = keep, 0 = padding.
 *  [P3] "gemma4-pt-claude" README, "Attention Backend Notes": an attention
 *       logit soft-cap (attn_logits_soft_cap) exists as a layer option; the
 *       page prints no formula, the reading is the tanh cap the Keras docs'
 *       argument table names for the final logits.
 *  [P4] "gemma4-pt-claude" README, "Key architectural features": the vision
 *       encoder is ViT-style with bidirectional attention; "Attention
 *       Backend Notes": the vision tower runs its attention at scale 1.0.
 *  [V4] "Gemma 4" overview blog, "Shared KV Cache": the key and value
 *       projections produce the K/V a layer stores (and later layers reuse).
 *
 * Definitions used throughout (readings of the pages, stated once):
 *  - RMSNorm over the d values of one head: x / sqrt(mean(x^2) + eps) * w,
 *    with the weight vector w[d] used as it is (no 1 + w) and shared by all
 *    heads of the layer; V-norm is the same without a weight  [K1][P1].
 *  - RoPE at the 0-based token position p: pair k is (x[k], x[k + d/2]);
 *    for k < R = rotary_fraction * d / 2 it is rotated by the angle
 *    p * rope_theta^(-2k/d); the pairs k >= R pass through unchanged
 *    (a zero-padded frequency vector)  [K1][V2].
 *  - K=V (k_eq_v): K = RoPE(RMSNorm(k_raw) * w_k), V = RMSNorm(k_raw):
 *    one raw projection feeds both  [K1].
 *  - Query head h reads KV head h / (num_heads / num_kv_heads)  [K2].
 *  - Keys a query at position i sees: global layer [0, i]; sliding layer the
 *    `window` most recent positions [max(0, i - window + 1), i]; a sliding
 *    query inside an image block [s, e) sees the union of its window and the
 *    whole block, [min(max(0, i - window + 1), s), e - 1]  [K1][V1].
 *    An image block is a maximal run of equal non-negative ids in
 *    image_block_ids; -1 marks text.  A bidirectional (vision-tower) layer:
 *    every position of the sequence, [0, T - 1]  [P4].
 *  - o_i = sum_j softmax_j(s_ij) v_j over those keys, with the score
 *    s_ij = softmax_scale * q_i . k_j, or c * tanh(softmax_scale * q_i . k_j / c)
 *    with a logit soft-cap c > 0 [P3].  A padding key (mask entry 0) is never
 *    attended [K4]; a query left without any key outputs 0.
 */
#ifndef G4ATTN_H
#define G4ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes.  Host-checkable errors return before anything is enqueued. */
typedef enum {
  G4ATTN_OK = 0,
  G4ATTN_EINVAL = 1,          /* bad argument (NULL, shape, inconsistent desc) */
  G4ATTN_EUNSUPPORTED = 2,    /* valid layer the library has no kernel for */
  G4ATTN_ECACHE_OVERFLOW = 3, /* a write past the end of a non-rolling cache */
  G4ATTN_ECUDA = 4,           /* a CUDA runtime call failed */
  G4ATTN_EDEVICE = 5,         /* a kernel recorded an error (see status word) */
  G4ATTN_EWORKSPACE = 6,      /* workspace NULL or smaller than required */
  G4ATTN_ECACHE_EMPTY = 7     /* decode on a sequence whose cache holds nothing */
} g4attn_status;

/* G4ATTN_BIDIRECTIONAL: the vision tower's attention shape [P4]; prefill
 * (and g4attn_attend) only: append and decode return G4ATTN_EUNSUPPORTED. */
enum { G4ATTN_SLIDING = 0, G4ATTN_GLOBAL = 1, G4ATTN_BIDIRECTIONAL = 2 };
enum { G4ATTN_BF16 = 0, G4ATTN_FP32 = 1 };

/* One attention layer [K2].  Sliding layers: window > 0, typically
 * rotary_fraction 1.0 and rope_theta 1e4.  Global layers: window ignored,
 * typically rotary_fraction 0.25 and rope_theta 1e6, k_eq_v on the K=V
 * variants.  rotary_fraction * head_dim must be an even integer.
 * softmax_scale (> 0) multiplies q.k (1/sqrt(head_dim) or 1.0; the pages
 * print both); rms_eps is added to mean(x^2) (the pages do not state it; 1e-6 is
 * the usual value).  dtype is the element type of every raw input, weight,
 * output and cache tensor of the call. */
typedef struct {
  int layer_type;        /* G4ATTN_SLIDING, G4ATTN_GLOBAL or
                            G4ATTN_BIDIRECTIONAL */
  int window;            /* keys per sliding query, itself included */
  float rotary_fraction; /* fraction of each head that is rotated */
  double rope_theta;     /* RoPE base */
  int k_eq_v;            /* 1: V derives from the K projection (v_raw NULL) */
  int num_heads;         /* Hq, query heads */
  int num_kv_heads;      /* Hkv, divides Hq */
  int head_dim;          /* d: 64, 128, 256 or 512 (other even sizes:
                            G4ATTN_EUNSUPPORTED) */
  float softmax_scale;
  float rms_eps;
  int dtype;             /* G4ATTN_BF16 or G4ATTN_FP32 */
  float logit_softcap;   /* c > 0: scores become c * tanh(score / c) [P3];
                            0: no cap */
} g4attn_layer_desc;

/* A per-layer KV cache [P2], caller-owned device memory.  K and V are stored
 * separately, also on K=V layers, each [batch, num_kv_heads, capacity,
 * head_dim] in `dtype`, holding post-prologue values (K after RMSNorm * w_k
 * and RoPE, V after V-norm).  len[b] (device int32) counts the positions of
 * sequence b written so far.  A rolling cache keeps position p at slot
 * p % capacity and needs capacity >= window; it is only valid on sliding
 * layers.  A non-rolling cache keeps position p at slot p and rejects
 * p >= capacity.
 * key_mask (device uint8 [batch, mask_len], or NULL) is the padding mask of
 * the prompt the cache holds [K4]: position p < mask_len of sequence b is a
 * padding key when key_mask[b * mask_len + p] == 0; positions >= mask_len
 * (tokens appended later) are kept.  g4attn_decode reads it; the prefill
 * calls take their mask as an argument.  mask_len is ignored when key_mask
 * is NULL.
 *
 * Single-tensor cache of a K=V layer [K1]: v == NULL.  On a K=V layer both K
 * and V derive from one raw vector, V = RMSNorm(k_raw) and K =
 * RoPE(V * w_k), so the cache stores V alone in `k` (half the bytes of the
 * two-tensor cache the pages' KV-cache table counts [P2]) and k_norm_w
 * (device [head_dim], the owning layer's key-norm weight) lets a reader
 * rebuild K.  Non-rolling caches only.  Writers: g4attn_prefill (the cache
 * is then not the attention's source) and g4attn_cache_append.  Readers:
 * g4attn_decode / _noalloc on bf16 layers with at most 8 query heads per KV
 * head (also KV-shared); other readers return G4ATTN_EUNSUPPORTED.
 * k_norm_w is ignored when v != NULL. */
typedef struct {
  void *k;
  void *v;
  int32_t *len;
  int capacity;
  int rolling;
  int batch;
  int num_kv_heads;
  int head_dim;
  int dtype;
  const uint8_t *key_mask;
  int mask_len;
  const void *k_norm_w;
} g4attn_cache;

/* Bytes of device workspace g4attn_prefill needs for this layer and size.
 * Returns 0 if the arguments are invalid. */
size_t g4attn_prefill_workspace_size(const g4attn_layer_desc *desc, int B,
                                     int T);

/* Bytes of device workspace g4attn_decode needs for this layer and cache
 * (batch, capacity).  Returns 0 if the arguments are invalid. */
size_t g4attn_decode_workspace_size(const g4attn_layer_desc *desc,
                                    const g4attn_cache *cache);

/* Prefill of a whole prompt (positions 0..T-1) through one layer
 * [K1][V1][V2]: prologue on Q, K, V, then masked softmax attention.
 *
 *  q_raw           device [B, T, num_heads, d]: query projection output.
 *  k_raw           device [B, T, num_kv_heads, d], or NULL for a KV-shared
 *                  layer [V3], which then reads its keys/values from `cache`
 *                  (positions 0..T-1 must be present there) and writes none.
 *  v_raw           device [B, T, num_kv_heads, d]; must be NULL with k_eq_v
 *                  or with k_raw NULL, non-NULL otherwise.
 *  q_norm_w        device [d]: QK-norm weight of the queries, used as is.
 *  k_norm_w        device [d]: QK-norm weight of the keys (ignored if k_raw
 *                  is NULL).
 *  image_block_ids device int32 [B, T] or NULL: -1 text, a block is a maximal
 *                  run of one non-negative id.  Ignored on global and
 *                  bidirectional layers.
 *  attention_mask  device uint8 [B, T] or NULL [K4]: a key at a position
 *                  whose entry is 0 is padding and never attended (RoPE
 *                  positions stay the token indices); a row left without any
 *                  key outputs 0.  NULL: no padding.
 *  cache           NULL, or a cache of this layer: with k_raw the post-prologue
 *                  K/V of positions 0..T-1 are written to it (a rolling cache
 *                  keeps the last `capacity` of them) and len[b] is set to T;
 *                  a non-rolling cache needs capacity >= T.
 *  out             device [B, T, num_heads, d]: attention output.
 *  workspace       device scratch of g4attn_prefill_workspace_size bytes,
 *                  256-byte aligned; its contents are not preserved.
 *  stream          cudaStream_t.
 *
 * Errors: G4ATTN_EINVAL for bad shapes, NULLs, an odd or non-positive
 * head_dim, num_heads % num_kv_heads != 0, window <= 0 on a sliding layer,
 * rotary_fraction * d not an even integer, cache shape or dtype mismatch, a
 * rolling cache on a global layer; G4ATTN_EUNSUPPORTED for a head_dim other
 * than 64, 128, 256 or 512 or more than 32 KV heads; G4ATTN_ECACHE_OVERFLOW
 * for a non-rolling cache with capacity < T; G4ATTN_EWORKSPACE; G4ATTN_ECUDA
 * if a launch fails.  Nothing is written when an error is returned.
 * image_block_ids are not checked: every maximal run of one non-negative id
 * is a block, so an id that appears in two separate runs makes two blocks
 * (not an error). */
int g4attn_prefill(const g4attn_layer_desc *desc, int B, int T,
                   const void *q_raw, const void *k_raw, const void *v_raw,
                   const void *q_norm_w, const void *k_norm_w,
                   const int32_t *image_block_ids,
                   const uint8_t *attention_mask, g4attn_cache *cache,
                   void *out, void *workspace, size_t ws_bytes, void *stream);

/* Bytes of device workspace g4attn_prefill_chunk needs.  Returns 0 if the
 * arguments are invalid. */
size_t g4attn_prefill_chunk_workspace_size(const g4attn_layer_desc *desc,
                                           int B, int T, int p0);

/* Cached (chunked) prefill ("gemma4-pt-claude" README, "Tests": a cached
 * path reproduces the uncached forward pass, image spans included): a chunk
 * of T tokens per sequence at positions p0 .. p0+T-1 after the p0 tokens
 * `cache` already holds (len[b] == p0 for every sequence: the caller's
 * contract).  The chunk's keys/values go through the prologue into slots
 * p0 .. p0+T-1 and len[b] becomes p0 + T; each query row then attends over
 * the interval of its position in a prompt of p0 + T tokens (image blocks
 * seen up to position p0 + T - 1: cut chunks between blocks to reproduce a
 * whole prompt).
 *
 *  q_raw, k_raw, v_raw, q_norm_w, k_norm_w, out: as g4attn_prefill, [B, T,
 *                  ...] for the chunk; k_raw NULL: a KV-shared layer reading
 *                  `cache`, which must hold positions 0 .. p0+T-1.
 *  image_block_ids device int32 [B, p0 + T] or NULL (ignored on global layers).
 *  attention_mask  device uint8 [B, p0 + T] or NULL: the padding mask of every
 *                  position up to the chunk's last (as g4attn_prefill); the
 *                  cache's key_mask is not read.
 *  cache           required; capacity >= p0 + T (a rolling cache only before
 *                  it wraps).
 *  workspace       g4attn_prefill_chunk_workspace_size bytes, 256-byte aligned.
 *
 * Errors: as g4attn_prefill; G4ATTN_ECACHE_OVERFLOW for a non-rolling cache
 * with capacity < p0 + T; G4ATTN_EINVAL for a rolling or KV-shared one. */
int g4attn_prefill_chunk(const g4attn_layer_desc *desc, int B, int T, int p0,
                         const void *q_raw, const void *k_raw,
                         const void *v_raw, const void *q_norm_w,
                         const void *k_norm_w, const int32_t *image_block_ids,
                         const uint8_t *attention_mask, g4attn_cache *cache,
                         void *out, void *workspace, size_t ws_bytes,
                         void *stream);

/* The QKV projection with the prologue in its epilogue [V4][K1]: for every
 * token row of x, raw = x W^T on the tensor cores, then per output head
 * RMSNorm (* w_q / w_k) and RoPE at the token's position p0 + t for query and
 * key heads, weightless RMSNorm for value heads (and, with k_eq_v, for the
 * key heads' V); the raw projections are never written.  bf16 only.
 *
 *  x         device bf16 [B, T, hidden], hidden a multiple of 8, 16-byte
 *            aligned.
 *  w_qkv     device bf16 [n_heads * d, hidden], 16-byte aligned: the rows of
 *            the num_heads query heads, then (with a cache) the num_kv_heads
 *            key heads, then (without k_eq_v) the num_kv_heads value heads.
 *  q_norm_w, k_norm_w  device [d]; k_norm_w is needed with a cache.
 *  q_hat     device bf16 [B, T, num_heads, d], 16-byte aligned: the
 *            post-prologue queries (the input of g4attn_attend).
 *  cache     NULL: a KV-shared layer [V3] that projects its queries only.
 *            Otherwise K/V of positions p0 .. p0+T-1 go to their slots (a
 *            rolling cache keeps the last `capacity` of them; a single-tensor
 *            cache V alone) and len[b] becomes p0 + T.
 *
 * Errors: G4ATTN_EINVAL for NULLs, hidden < 8 or not a multiple of 8,
 * misaligned pointers, a cache shape mismatch; G4ATTN_EUNSUPPORTED for fp32;
 * G4ATTN_ECACHE_OVERFLOW for a non-rolling cache with capacity < p0 + T;
 * G4ATTN_ECUDA. */
int g4attn_qkv_prologue(const g4attn_layer_desc *desc, int B, int T, int p0,
                        const void *x, int hidden, const void *w_qkv,
                        const void *q_norm_w, const void *k_norm_w, void *q_hat,
                        g4attn_cache *cache, void *stream);

/* Bytes of device workspace g4attn_attend needs.  Returns 0 if the
 * arguments are invalid. */
size_t g4attn_attend_workspace_size(const g4attn_layer_desc *desc, int B, int T,
                                    int p0);

/* The attention of a prefill from post-prologue inputs [K1][V1][P4]: the
 * queries q_hat (RMSNorm * w_q and RoPE already applied, e.g. by
 * g4attn_qkv_prologue or by a vision tower's own 2-D rotary) of T tokens at
 * positions p0 .. p0+T-1 attend over the keys/values `cache` holds at
 * positions 0 .. p0+T-1 (slots 0 .. p0+T-1), with the intervals of
 * g4attn_prefill_chunk.  Nothing is written to the cache and len[] is not
 * read or changed.
 *
 *  q_hat           device [B, T, num_heads, d] in dtype.
 *  image_block_ids device int32 [B, p0 + T] or NULL (sliding layers only).
 *  attention_mask  device uint8 [B, p0 + T] or NULL, as g4attn_prefill_chunk.
 *  cache           a two-tensor cache (k and v), capacity >= p0 + T.
 *  out             device [B, T, num_heads, d].
 *  workspace       g4attn_attend_workspace_size bytes, 256-byte aligned.
 *
 * Errors: G4ATTN_EINVAL for NULLs, shape or dtype mismatch, capacity <
 * p0 + T; G4ATTN_EUNSUPPORTED for a single-tensor cache; G4ATTN_EWORKSPACE;
 * G4ATTN_ECUDA. */
int g4attn_attend(const g4attn_layer_desc *desc, int B, int T, int p0,
                  const void *q_hat, const int32_t *image_block_ids,
                  const uint8_t *attention_mask, const g4attn_cache *cache,
                  void *out, void *workspace, size_t ws_bytes, void *stream);

/* Append one token per sequence to a layer's cache [P2][K3]: the key/value
 * prologue of k_raw/v_raw (device [B, 1, num_kv_heads, d]; v_raw NULL with
 * k_eq_v) at position p = len[b], written at slot p (rolling: p % capacity),
 * then len[b] = p + 1.  k_norm_w is device [d].
 * If p >= capacity on a non-rolling cache nothing is written for that
 * sequence, len[b] is unchanged and the device status word records
 * G4ATTN_ECACHE_OVERFLOW (read it with g4attn_get_device_status).
 * A bidirectional layer has no cache append: G4ATTN_EUNSUPPORTED. */
int g4attn_cache_append(const g4attn_layer_desc *desc, g4attn_cache *cache,
                        const void *k_raw, const void *v_raw,
                        const void *k_norm_w, void *stream);

/* Single-token decode [K3][V1][V3]: for every sequence b the query of the
 * token at position P = len[b] - 1 (the last one appended) attends over the
 * keys of row P of a prefill -- [max(0, P - window + 1), P] on a sliding
 * layer, [0, P] on a global one -- read from `cache`, minus the padding keys
 * the cache's key_mask marks [K4].  A KV-shared layer passes the cache of
 * the layer it reads and skips the append.
 *
 *  q_raw     device [B, 1, num_heads, d];  q_norm_w device [d].
 *  out       device [B, 1, num_heads, d].
 *  workspace device scratch of g4attn_decode_workspace_size bytes (split-KV
 *            partials), 256-byte aligned.
 *
 * The keys are split into fixed-size chunks; each chunk yields a partial
 * softmax (max, sum, weighted values) and a combine kernel merges them.
 * A sequence with len[b] == 0 gets a zero output and the device status word
 * records G4ATTN_ECACHE_EMPTY.  A bidirectional layer has no decode step:
 * G4ATTN_EUNSUPPORTED. */
int g4attn_decode(const g4attn_layer_desc *desc, const g4attn_cache *cache,
                  const void *q_raw, const void *q_norm_w, void *out,
                  void *workspace, size_t ws_bytes, void *stream);

/* g4attn_decode without a workspace, for callers that cannot give the
 * library device memory per call (for example a serving runtime that has
 * handed all free device memory to its KV-cache pool, or a plugin host that
 * exposes no allocator).  The pages have no counterpart: this is a property
 * of the library, not of the layer.
 *
 * Same arguments, semantics and outputs as g4attn_decode, minus the
 * workspace.  The split-KV partials go to a fixed 16 MiB array of device
 * memory that the library holds on every GPU that loads it, until the process
 * exits; this call allocates and frees nothing.  If the partials of one chunk
 * per (sequence, query head) -- batch * num_heads * (head_dim + 2) * 4 bytes
 * -- exceed 16 MiB the call returns G4ATTN_EWORKSPACE and enqueues nothing;
 * when the usual number of chunks does not fit, the keys are split into fewer,
 * longer chunks.  All calls on a device share the array: calls whose kernels
 * may overlap on the GPU (other streams, other host threads) race on it and
 * must be serialised by the caller.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress); make that first call before
 * any stream capture. */
int g4attn_decode_noalloc(const g4attn_layer_desc *desc, const g4attn_cache *cache,
                          const void *q_raw, const void *q_norm_w, void *out,
                          void *stream);

/* Waits for `stream`, then returns and clears the device status word of the
 * current device: G4ATTN_OK, or the first error a kernel recorded since the
 * last call.  Returns G4ATTN_ECUDA if the wait or the copy fails. */
int g4attn_get_device_status(void *stream);

/* Optional timing hook: the next g4attn_prefill or g4attn_decode call on any
 * stream records start_event on the call's stream after enqueueing everything
 * that precedes its attention kernel (the dominant launch) and stop_event
 * right after enqueueing that kernel, then forgets both.  The interval holds
 * the attention kernel alone; when the stream has drained before the kernel
 * is enqueued it also holds the host's setup of that launch (tensor maps),
 * so time it behind preceding work.  The events are cudaEvent_t handles
 * owned by the caller.  Passing NULLs cancels a pending request. */
void g4attn_time_next_attention(void *start_event, void *stop_event);

/* Number of kernel launches the library has enqueued since it was loaded. */
uint64_t g4attn_launch_count(void);

/* Static text for a status code. */
const char *g4attn_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* G4ATTN_H */
