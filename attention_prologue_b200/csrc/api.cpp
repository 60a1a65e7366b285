// C-ABI entry points of libg4attn.so (declared in include/g4attn.h): host-side
// validation, workspace layout and kernel launches on the caller's stream.
// Nothing here allocates device memory or waits for the device, except
// g4attn_get_device_status.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "g4attn.h"
#include "g4attn_internal.h"

namespace g4 {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// An NVTX range over one entry point, so a profiler's timeline shows the
// library's calls around their kernels (a no-op unless a tool is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// The unique id of the calling thread's current CUDA context (cuCtxGetId:
// never reused within a process, unlike the context handle).  Device
// addresses of the library's __device__ variables are cached per context id,
// so a context destroyed and re-created (cudaDeviceReset) gets a fresh lookup.
bool current_context_id(unsigned long long* id) {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static std::once_flag once;
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return false;
  if (!ctx) {
    // a thread that has made no runtime call yet: let the runtime make the
    // device's primary context current (never reached while a stream of
    // this thread is being captured, which needs a current context)
    if (cudaFree(nullptr) != cudaSuccess || get_current(&ctx) != CUDA_SUCCESS || !ctx)
      return false;
  }
  return get_id(ctx, id) == CUDA_SUCCESS;
}

static std::mutex g_time_mu;
static cudaEvent_t g_time_ev0 = nullptr, g_time_ev1 = nullptr;

// Take (and forget) a pending timing request.
static void take_timing(cudaEvent_t* e0, cudaEvent_t* e1) {
  std::lock_guard<std::mutex> lock(g_time_mu);
  *e0 = g_time_ev0;
  *e1 = g_time_ev1;
  g_time_ev0 = g_time_ev1 = nullptr;
}

static size_t elem_size(int dtype) { return dtype == G4ATTN_FP32 ? 4 : 2; }
static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Validate a layer descriptor and derive the kernels' view of it.
static int make_cfg(const g4attn_layer_desc* d, LayerCfg* L) {
  if (!d) return G4ATTN_EINVAL;
  if (d->layer_type != G4ATTN_SLIDING && d->layer_type != G4ATTN_GLOBAL &&
      d->layer_type != G4ATTN_BIDIRECTIONAL)
    return G4ATTN_EINVAL;
  if (d->dtype != G4ATTN_BF16 && d->dtype != G4ATTN_FP32) return G4ATTN_EINVAL;
  if (d->head_dim < 2 || (d->head_dim & 1)) return G4ATTN_EINVAL;
  if (d->num_heads < 1 || d->num_kv_heads < 1) return G4ATTN_EINVAL;
  if (d->num_heads % d->num_kv_heads != 0) return G4ATTN_EINVAL;
  if (d->layer_type == G4ATTN_SLIDING && d->window < 1) return G4ATTN_EINVAL;
  if (!(d->rotary_fraction >= 0.f && d->rotary_fraction <= 1.f)) return G4ATTN_EINVAL;
  const double rd = (double)d->rotary_fraction * d->head_dim;  // rotated dims, even integer
  const long R2 = std::lround(rd);
  if (std::fabs(rd - (double)R2) > 1e-6 || (R2 & 1)) return G4ATTN_EINVAL;
  if (!(d->rope_theta > 0.0) || !std::isfinite(d->rope_theta)) return G4ATTN_EINVAL;
  if (!(d->softmax_scale > 0.f) || !std::isfinite(d->softmax_scale)) return G4ATTN_EINVAL;
  if (!(d->rms_eps >= 0.f) || !std::isfinite(d->rms_eps)) return G4ATTN_EINVAL;
  if (!(d->logit_softcap >= 0.f) || !std::isfinite(d->logit_softcap)) return G4ATTN_EINVAL;
  if (d->k_eq_v != 0 && d->k_eq_v != 1) return G4ATTN_EINVAL;
  // a valid layer without a kernel: head sizes other than 64/128/256/512, or
  // more than 32 KV heads (the cache append runs one warp per KV head in a
  // single block of at most 1024 threads)
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256 && d->head_dim != 512)
    return G4ATTN_EUNSUPPORTED;
  if (d->num_kv_heads > 32) return G4ATTN_EUNSUPPORTED;
  L->layer_type = d->layer_type;
  L->window = d->layer_type == G4ATTN_SLIDING ? d->window : 0;
  L->k_eq_v = d->k_eq_v;
  L->Hq = d->num_heads;
  L->Hkv = d->num_kv_heads;
  L->d = d->head_dim;
  L->dtype = d->dtype;
  L->scale = d->softmax_scale;
  L->eps = d->rms_eps;
  L->softcap = d->logit_softcap;
  std::memset(&L->rope, 0, sizeof(L->rope));
  L->rope.rotated_pairs = (int)(R2 / 2);
  for (int k = 0; k < L->rope.rotated_pairs; ++k) {
    L->rope.inv_freq[k] = std::pow(d->rope_theta, -2.0 * k / (double)d->head_dim);
    // < 1/(2 pi) turns per position (inv_freq <= 1): the fraction fits 64 bits
    L->rope.turns[k] = (unsigned long long)std::ldexp(L->rope.inv_freq[k] / 6.283185307179586476925, 64);
  }
  return G4ATTN_OK;
}

// A single-tensor cache (v == NULL) stores V = RMSNorm(k_raw) of a K=V layer
// in `k`; a reader rebuilds K with the owning layer's k_norm_w and RoPE.
static bool single_tensor(const g4attn_cache* c) { return c->v == nullptr; }

static int check_cache(const LayerCfg& L, const g4attn_cache* c, int B) {
  if (!c->k || !c->len) return G4ATTN_EINVAL;
  if (single_tensor(c) && (!L.k_eq_v || !c->k_norm_w || c->rolling)) return G4ATTN_EINVAL;
  if (c->batch != B || c->num_kv_heads != L.Hkv || c->head_dim != L.d || c->dtype != L.dtype)
    return G4ATTN_EINVAL;
  if (c->capacity < 1 || (c->rolling != 0 && c->rolling != 1)) return G4ATTN_EINVAL;
  if (c->rolling && (L.layer_type != G4ATTN_SLIDING || c->capacity < L.window))
    return G4ATTN_EINVAL;
  if (c->key_mask && c->mask_len < 0) return G4ATTN_EINVAL;
  return G4ATTN_OK;
}

static KeyMask cache_mask(const g4attn_cache* c) {
  return c->key_mask ? KeyMask{c->key_mask, c->mask_len} : KeyMask{nullptr, 0};
}

// Workspace of one prefill call.
struct PrefillWs {
  size_t q_hat, kv, intervals, bits, span, total;  // byte offsets / sizes
  bool need_kv;                              // keys go to scratch (no usable cache)
  int words;                                 // 64-key words of the padding bits
};

// Tk: key positions the call's rows may see (T, or p0 + T for a chunk).
static PrefillWs prefill_ws(const LayerCfg& L, int B, int T, bool need_kv, bool intervals,
                            bool mask, int Tk, bool with_q = true) {
  PrefillWs w;
  const size_t es = elem_size(L.dtype);
  size_t off = 0;
  w.q_hat = off;
  if (with_q) off += align256((size_t)B * T * L.Hq * L.d * es);
  w.kv = off;
  if (need_kv) off += 2 * align256((size_t)B * T * L.Hkv * L.d * es);
  w.intervals = off;
  if (intervals) off += 2 * align256((size_t)B * T * sizeof(int32_t));
  w.words = (Tk + 63) / 64;
  w.bits = off;
  if (mask) off += align256((size_t)B * w.words * sizeof(uint64_t));
  w.span = off;
  if (mask) off += align256((size_t)B * sizeof(int2));
  w.total = off;
  w.need_kv = need_kv;
  return w;
}

// The first and last kept position of every sequence (the row intervals are
// clamped to them: key tiles of padding alone are never visited), or none.
static cudaError_t padding_span(const PrefillWs& w, char* ws, int B, int Tk, const uint8_t* mask,
                                const int2** span, cudaStream_t s) {
  *span = nullptr;
  if (!mask) return cudaSuccess;
  int2* sp = reinterpret_cast<int2*>(ws + w.span);
  *span = sp;
  return launch_mask_span(B, Tk, mask, sp, s);
}

// The padding bits of a prefill call, or none.
static cudaError_t padding_bits(const PrefillWs& w, char* ws, int B, int Tk, const uint8_t* mask,
                                KeyBits* kb, cudaStream_t s) {
  *kb = KeyBits{nullptr, 0};
  if (!mask) return cudaSuccess;
  uint64_t* bits = reinterpret_cast<uint64_t*>(ws + w.bits);
  *kb = KeyBits{bits, w.words};
  return launch_mask_bits(B, Tk, mask, bits, w.words, s);
}

}  // namespace g4

using namespace g4;

extern "C" {

size_t g4attn_prefill_workspace_size(const g4attn_layer_desc* desc, int B, int T) {
  LayerCfg L;
  if (make_cfg(desc, &L) != G4ATTN_OK || B < 0 || T < 0) return 0;
  return prefill_ws(L, B, T, true, true, true, T).total;
}

size_t g4attn_decode_workspace_size(const g4attn_layer_desc* desc, const g4attn_cache* cache) {
  LayerCfg L;
  if (make_cfg(desc, &L) != G4ATTN_OK || !cache) return 0;
  if (check_cache(L, cache, cache->batch) != G4ATTN_OK) return 0;
  return align256(decode_partials_bytes(L, cache->batch, decode_plan(L, cache->capacity)));
}

int g4attn_prefill(const g4attn_layer_desc* desc, int B, int T, const void* q_raw,
                   const void* k_raw, const void* v_raw, const void* q_norm_w,
                   const void* k_norm_w, const int32_t* image_block_ids,
                   const uint8_t* attention_mask, g4attn_cache* cache, void* out,
                   void* workspace, size_t ws_bytes, void* stream) {
  g4::CallRange range("g4attn_prefill");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (B < 0 || T < 0) return G4ATTN_EINVAL;
  if (!q_raw || !q_norm_w || !out) return G4ATTN_EINVAL;
  const bool shared = k_raw == nullptr;  // KV-shared layer: keys come from the cache
  if (shared) {
    if (v_raw || !cache) return G4ATTN_EINVAL;
  } else {
    if (!k_norm_w) return G4ATTN_EINVAL;
    if ((v_raw == nullptr) != (L.k_eq_v == 1)) return G4ATTN_EINVAL;
  }
  if (cache) {
    if ((st = check_cache(L, cache, B)) != G4ATTN_OK) return st;
    if (!cache->rolling && cache->capacity < T) return G4ATTN_ECACHE_OVERFLOW;
    if (shared && cache->capacity < T) return G4ATTN_EINVAL;  // evicted keys cannot be read
    if (shared && single_tensor(cache)) return G4ATTN_EUNSUPPORTED;  // no K to read
  }
  if (B == 0 || T == 0) return G4ATTN_OK;

  // attention reads keys from the cache when it holds K and V of positions
  // 0..T-1 at slots 0..T-1, otherwise from scratch
  const bool cache_is_src = cache && cache->capacity >= T && !single_tensor(cache);
  const bool bidir = L.layer_type == G4ATTN_BIDIRECTIONAL;
  const bool intervals = (L.layer_type == G4ATTN_SLIDING && image_block_ids != nullptr) || bidir ||
                         attention_mask != nullptr;
  PrefillWs w = prefill_ws(L, B, T, !cache_is_src, intervals, attention_mask != nullptr, T);
  if (!workspace || ws_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return G4ATTN_EWORKSPACE;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t es = elem_size(L.dtype);

  KVSrc src;
  if (cache_is_src) {
    src = {cache->k, cache->v, cache->capacity, T};
  } else {
    char* kbuf = ws + w.kv;
    char* vbuf = kbuf + align256((size_t)B * T * L.Hkv * L.d * es);
    src = {kbuf, vbuf, T, T};
  }
  cudaError_t e = cudaSuccess;
  KVDst d0{nullptr, nullptr, 1, 0, 0}, d1{nullptr, nullptr, 1, 0, 0};
  if (!shared) {
    d0 = {const_cast<void*>(src.k), const_cast<void*>(src.v), src.cap, 0, 0};
    if (cache && single_tensor(cache))  // V alone (put_kv with v == nullptr)
      d1 = {cache->k, nullptr, cache->capacity, 0, 0};
    else if (cache && !cache_is_src)  // rolling cache smaller than the prompt: the last `cap`
      d1 = {cache->k, cache->v, cache->capacity, 1, T - cache->capacity};
  }
  void* q_hat = ws + w.q_hat;
  e = launch_token_prologue(L, B, T, 0, q_raw, q_norm_w, q_hat, shared ? nullptr : k_raw, v_raw,
                            k_norm_w, d0, d1, (cache && !shared) ? cache->len : nullptr, s);
  if (e != cudaSuccess) return G4ATTN_ECUDA;
  RowIntervals rows{nullptr, nullptr};
  if (intervals) {
    int32_t* lo = reinterpret_cast<int32_t*>(ws + w.intervals);
    int32_t* hi = reinterpret_cast<int32_t*>(ws + w.intervals +
                                             align256((size_t)B * T * sizeof(int32_t)));
    const int2* span;
    if (padding_span(w, ws, B, T, attention_mask, &span, s) != cudaSuccess) return G4ATTN_ECUDA;
    e = (bidir || span)
            ? launch_chunk_intervals(
                  L, B, T, 0, L.layer_type == G4ATTN_SLIDING ? image_block_ids : nullptr, span,
                  lo, hi, s)
            : launch_block_intervals(L, B, T, image_block_ids, lo, hi, s);
    if (e != cudaSuccess) return G4ATTN_ECUDA;
    rows = {lo, hi};
  }
  KeyBits kb;
  if (padding_bits(w, ws, B, T, attention_mask, &kb, s) != cudaSuccess) return G4ATTN_ECUDA;
  cudaEvent_t ev0, ev1;
  take_timing(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, s);
  e = attention_sm100_supported(L)
          ? launch_attention_sm100(L, B, T, q_hat, src, rows, kb, out, status_ptr(), s)
          : launch_attention_simt(L, B, T, q_hat, src, rows, kb, out, s);
  if (ev1) cudaEventRecord(ev1, s);
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

size_t g4attn_prefill_chunk_workspace_size(const g4attn_layer_desc* desc, int B, int T, int p0) {
  LayerCfg L;
  if (make_cfg(desc, &L) != G4ATTN_OK || B < 0 || T < 0 || p0 < 0) return 0;
  return prefill_ws(L, B, T, false, true, true, p0 + T).total;
}

int g4attn_prefill_chunk(const g4attn_layer_desc* desc, int B, int T, int p0, const void* q_raw,
                         const void* k_raw, const void* v_raw, const void* q_norm_w,
                         const void* k_norm_w, const int32_t* image_block_ids,
                         const uint8_t* attention_mask, g4attn_cache* cache, void* out,
                         void* workspace, size_t ws_bytes, void* stream) {
  g4::CallRange range("g4attn_prefill_chunk");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (B < 0 || T < 0 || p0 < 0) return G4ATTN_EINVAL;
  if (!q_raw || !q_norm_w || !out || !cache) return G4ATTN_EINVAL;
  const bool shared = k_raw == nullptr;  // KV-shared layer: the chunk's keys are in the cache
  if (shared) {
    if (v_raw) return G4ATTN_EINVAL;
  } else {
    if (!k_norm_w) return G4ATTN_EINVAL;
    if ((v_raw == nullptr) != (L.k_eq_v == 1)) return G4ATTN_EINVAL;
  }
  if ((st = check_cache(L, cache, B)) != G4ATTN_OK) return st;
  if (single_tensor(cache)) return G4ATTN_EUNSUPPORTED;  // the chunk reads K from the cache
  if ((long)p0 + T > cache->capacity)  // every position must stay readable
    return cache->rolling || shared ? G4ATTN_EINVAL : G4ATTN_ECACHE_OVERFLOW;
  if (B == 0 || T == 0) return G4ATTN_OK;

  PrefillWs w = prefill_ws(L, B, T, false, true, attention_mask != nullptr, p0 + T);
  if (!workspace || ws_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return G4ATTN_EWORKSPACE;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* q_hat = ws + w.q_hat;
  KVDst d0{nullptr, nullptr, 1, 0, 0}, d1{nullptr, nullptr, 1, 0, 0};
  if (!shared) d0 = {cache->k, cache->v, cache->capacity, cache->rolling, 0};
  cudaError_t e = launch_token_prologue(L, B, T, p0, q_raw, q_norm_w, q_hat,
                                        shared ? nullptr : k_raw, v_raw, k_norm_w, d0, d1,
                                        shared ? nullptr : cache->len, s);
  if (e != cudaSuccess) return G4ATTN_ECUDA;
  int32_t* lo = reinterpret_cast<int32_t*>(ws + w.intervals);
  int32_t* hi =
      reinterpret_cast<int32_t*>(ws + w.intervals + align256((size_t)B * T * sizeof(int32_t)));
  const int2* span;
  if (padding_span(w, ws, B, p0 + T, attention_mask, &span, s) != cudaSuccess)
    return G4ATTN_ECUDA;
  e = launch_chunk_intervals(L, B, T, p0,
                             L.layer_type == G4ATTN_SLIDING ? image_block_ids : nullptr, span, lo,
                             hi, s);
  if (e != cudaSuccess) return G4ATTN_ECUDA;
  const KVSrc src{cache->k, cache->v, cache->capacity, p0 + T};
  const RowIntervals rows{lo, hi};
  KeyBits kb;
  if (padding_bits(w, ws, B, p0 + T, attention_mask, &kb, s) != cudaSuccess)
    return G4ATTN_ECUDA;
  cudaEvent_t ev0, ev1;
  take_timing(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, s);
  e = attention_sm100_supported(L)
          ? launch_attention_sm100(L, B, T, q_hat, src, rows, kb, out, status_ptr(), s)
          : launch_attention_simt(L, B, T, q_hat, src, rows, kb, out, s);
  if (ev1) cudaEventRecord(ev1, s);
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

int g4attn_qkv_prologue(const g4attn_layer_desc* desc, int B, int T, int p0, const void* x,
                        int hidden, const void* w_qkv, const void* q_norm_w,
                        const void* k_norm_w, void* q_hat, g4attn_cache* cache, void* stream) {
  g4::CallRange range("g4attn_qkv_prologue");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (B < 0 || T < 0 || p0 < 0) return G4ATTN_EINVAL;
  if (!x || !w_qkv || !q_norm_w || !q_hat) return G4ATTN_EINVAL;
  if (hidden < 8 || hidden % 8 != 0) return G4ATTN_EINVAL;  // rows of 16-byte multiples
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w_qkv) |
       reinterpret_cast<uintptr_t>(q_hat)) & 15)
    return G4ATTN_EINVAL;
  if (L.dtype != G4ATTN_BF16) return G4ATTN_EUNSUPPORTED;  // the tensor-core path is bf16
  if ((long)B * T > INT32_MAX) return G4ATTN_EINVAL;
  KVDst kv{nullptr, nullptr, 1, 0, 0};
  int n_heads = L.Hq;
  if (cache) {
    if (!k_norm_w) return G4ATTN_EINVAL;
    if ((st = check_cache(L, cache, B)) != G4ATTN_OK) return st;
    if (!cache->rolling && (long)p0 + T > cache->capacity) return G4ATTN_ECACHE_OVERFLOW;
    // a rolling cache keeps the last `capacity` positions of the call
    const long first = cache->rolling ? (long)p0 + T - cache->capacity : 0;
    kv = {cache->k, cache->v, cache->capacity, cache->rolling, (int)std::max(0L, first)};
    n_heads += L.k_eq_v ? L.Hkv : 2 * L.Hkv;
  }
  if (B == 0 || T == 0) return G4ATTN_OK;
  cudaError_t e = launch_qkv_prologue(L, B, T, p0, x, hidden, w_qkv, n_heads, q_norm_w,
                                      cache ? k_norm_w : nullptr, q_hat, kv,
                                      cache ? cache->len : nullptr, status_ptr(),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

size_t g4attn_attend_workspace_size(const g4attn_layer_desc* desc, int B, int T, int p0) {
  LayerCfg L;
  if (make_cfg(desc, &L) != G4ATTN_OK || B < 0 || T < 0 || p0 < 0) return 0;
  return prefill_ws(L, B, T, false, true, true, p0 + T, false).total;
}

int g4attn_attend(const g4attn_layer_desc* desc, int B, int T, int p0, const void* q_hat,
                  const int32_t* image_block_ids, const uint8_t* attention_mask,
                  const g4attn_cache* cache, void* out, void* workspace, size_t ws_bytes,
                  void* stream) {
  g4::CallRange range("g4attn_attend");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (B < 0 || T < 0 || p0 < 0) return G4ATTN_EINVAL;
  if (!q_hat || !out || !cache) return G4ATTN_EINVAL;
  if ((st = check_cache(L, cache, B)) != G4ATTN_OK) return st;
  if (single_tensor(cache)) return G4ATTN_EUNSUPPORTED;  // reads K from the cache
  if ((long)p0 + T > cache->capacity) return G4ATTN_EINVAL;  // positions must be at slot = pos
  if (B == 0 || T == 0) return G4ATTN_OK;
  PrefillWs w = prefill_ws(L, B, T, false, true, attention_mask != nullptr, p0 + T, false);
  if (!workspace || ws_bytes < w.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return G4ATTN_EWORKSPACE;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* lo = reinterpret_cast<int32_t*>(ws + w.intervals);
  int32_t* hi =
      reinterpret_cast<int32_t*>(ws + w.intervals + align256((size_t)B * T * sizeof(int32_t)));
  const int2* span;
  if (padding_span(w, ws, B, p0 + T, attention_mask, &span, s) != cudaSuccess)
    return G4ATTN_ECUDA;
  cudaError_t e = launch_chunk_intervals(
      L, B, T, p0, L.layer_type == G4ATTN_SLIDING ? image_block_ids : nullptr, span, lo, hi, s);
  if (e != cudaSuccess) return G4ATTN_ECUDA;
  const KVSrc src{cache->k, cache->v, cache->capacity, p0 + T};
  const RowIntervals rows{lo, hi};
  KeyBits kb;
  if (padding_bits(w, ws, B, p0 + T, attention_mask, &kb, s) != cudaSuccess)
    return G4ATTN_ECUDA;
  cudaEvent_t ev0, ev1;
  take_timing(&ev0, &ev1);
  if (ev0) cudaEventRecord(ev0, s);
  e = attention_sm100_supported(L)
          ? launch_attention_sm100(L, B, T, q_hat, src, rows, kb, out, status_ptr(), s)
          : launch_attention_simt(L, B, T, q_hat, src, rows, kb, out, s);
  if (ev1) cudaEventRecord(ev1, s);
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

int g4attn_cache_append(const g4attn_layer_desc* desc, g4attn_cache* cache, const void* k_raw,
                        const void* v_raw, const void* k_norm_w, void* stream) {
  g4::CallRange range("g4attn_cache_append");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (L.layer_type == G4ATTN_BIDIRECTIONAL) return G4ATTN_EUNSUPPORTED;  // no decode step
  if (!cache || !k_raw || !k_norm_w) return G4ATTN_EINVAL;
  if ((v_raw == nullptr) != (L.k_eq_v == 1)) return G4ATTN_EINVAL;
  if ((st = check_cache(L, cache, cache->batch)) != G4ATTN_OK) return st;
  if (cache->batch == 0) return G4ATTN_OK;
  cudaError_t e = launch_append(L, cache->batch, k_raw, v_raw, k_norm_w, cache->k, cache->v,
                                cache->len, cache->capacity, cache->rolling, status_ptr(),
                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

int g4attn_decode(const g4attn_layer_desc* desc, const g4attn_cache* cache, const void* q_raw,
                  const void* q_norm_w, void* out, void* workspace, size_t ws_bytes,
                  void* stream) {
  g4::CallRange range("g4attn_decode");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (L.layer_type == G4ATTN_BIDIRECTIONAL) return G4ATTN_EUNSUPPORTED;  // no decode step
  if (!cache || !q_raw || !q_norm_w || !out) return G4ATTN_EINVAL;
  if ((st = check_cache(L, cache, cache->batch)) != G4ATTN_OK) return st;
  if (single_tensor(cache) && !decode_mma_supported(L, cache->capacity, 0))
    return G4ATTN_EUNSUPPORTED;  // K is rebuilt only by the tensor-core split kernel
  if (cache->batch == 0) return G4ATTN_OK;
  const DecodePlan plan = decode_plan(L, cache->capacity);
  const size_t need = decode_partials_bytes(L, cache->batch, plan);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return G4ATTN_EWORKSPACE;
  cudaEvent_t ev0, ev1;
  take_timing(&ev0, &ev1);
  cudaError_t e = launch_decode(L, cache->batch, q_raw, q_norm_w, cache->k, cache->v,
                                single_tensor(cache) ? cache->k_norm_w : nullptr, cache->len,
                                cache->capacity, cache->rolling, cache_mask(cache), plan,
                                static_cast<float*>(workspace), out, status_ptr(),
                                static_cast<cudaStream_t>(stream), ev0, ev1);
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

int g4attn_decode_noalloc(const g4attn_layer_desc* desc, const g4attn_cache* cache,
                          const void* q_raw, const void* q_norm_w, void* out, void* stream) {
  g4::CallRange range("g4attn_decode_noalloc");
  LayerCfg L;
  int st = make_cfg(desc, &L);
  if (st != G4ATTN_OK) return st;
  if (L.layer_type == G4ATTN_BIDIRECTIONAL) return G4ATTN_EUNSUPPORTED;  // no decode step
  if (!cache || !q_raw || !q_norm_w || !out) return G4ATTN_EINVAL;
  if ((st = check_cache(L, cache, cache->batch)) != G4ATTN_OK) return st;
  if (single_tensor(cache) && !decode_mma_supported(L, cache->capacity, 0))
    return G4ATTN_EUNSUPPORTED;
  if (cache->batch == 0) return G4ATTN_OK;
  return launch_decode_noalloc(L, cache->batch, q_raw, q_norm_w, cache->k, cache->v,
                               single_tensor(cache) ? cache->k_norm_w : nullptr, cache->len,
                               cache->capacity, cache->rolling, cache_mask(cache), out,
                               status_ptr(), static_cast<cudaStream_t>(stream));
}

int g4attn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return G4ATTN_ECUDA;
  int* p = status_ptr();
  if (!p) return G4ATTN_ECUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return G4ATTN_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess)
      return G4ATTN_ECUDA;
  }
  return v;
}

void g4attn_time_next_attention(void* start_event, void* stop_event) {
  std::lock_guard<std::mutex> lock(g_time_mu);
  g_time_ev0 = static_cast<cudaEvent_t>(start_event);
  g_time_ev1 = static_cast<cudaEvent_t>(stop_event);
}

uint64_t g4attn_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* g4attn_status_string(int status) {
  switch (status) {
    case G4ATTN_OK: return "ok";
    case G4ATTN_EINVAL: return "invalid argument";
    case G4ATTN_EUNSUPPORTED: return "unsupported layer";
    case G4ATTN_ECACHE_OVERFLOW: return "write past the end of a non-rolling KV cache";
    case G4ATTN_ECUDA: return "CUDA runtime error";
    case G4ATTN_EDEVICE: return "a kernel recorded an error";
    case G4ATTN_EWORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case G4ATTN_ECACHE_EMPTY: return "decode on a sequence with an empty cache";
  }
  return "unknown status";
}

}  // extern "C"
