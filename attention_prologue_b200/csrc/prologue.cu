// Prologue kernels of the Gemma 4 attention layer ("Gemma 4" Keras docs,
// "What changed from Gemma 3": plain-weight RMSNorm, zero-pad partial rope,
// K=V; "gemma4-pt-claude" README, "Supported Models": QK-norm and V-norm),
// the per-row interval pre-pass of image blocks, and the cache append
// ("gemma4-pt-claude" README, "KV Cache").
//
// Memory-bound: one warp per token (prompt) or per KV head (append), 16-byte
// accesses where the head size allows, fp32 arithmetic, fp64 RoPE angle
// reduction computed once per token and shared by all of its heads.
#include <mutex>

#include "common.cuh"
#include "g4attn.h"

namespace g4 {

__device__ int g_status;  // first error recorded by a kernel, 0 = none

// Device address of g_status in the current context, looked up once per
// context (the host-side name of a __device__ variable is only a stand-in).
int* status_ptr() {
  static std::mutex mu;
  static unsigned long long ids[64] = {0};
  static int* ptrs[64] = {nullptr};
  int dev = 0;
  unsigned long long id = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!current_context_id(&id)) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev] || ids[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess || !p) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
    ids[dev] = id;
  }
  return ptrs[dev];
}

constexpr int kWarps = 4;  // warps per block of the per-vector kernels

template <typename T, int D>
__device__ __forceinline__ void put_kv(const KVDst& d, int Hkv, long b, int h, long t,
                                       const float* k0, const float* k1, const float* v0,
                                       const float* v1) {
  if (!d.k || t < d.first) return;
  const long slot = d.rolling ? t % d.cap : t;
  const long off = (((long)b * Hkv + h) * d.cap + slot) * D;
  if (!d.v) {  // single-tensor cache of a K=V layer: V alone
    store_vec<T, D>(static_cast<T*>(d.k) + off, v0, v1);
    return;
  }
  store_vec<T, D>(static_cast<T*>(d.k) + off, k0, k1);
  store_vec<T, D>(static_cast<T*>(d.v) + off, v0, v1);
}

// Prologue of a whole prompt, one warp per token: the RoPE factors of the
// token (position t) are computed once and applied to its Hq query heads and
// Hkv key heads; the value heads are normalised without weight or rotation
// (from the key projection with K=V).  Heads are processed NB = 4 at a time
// with all their loads issued first (four at a time and four warps a block
// leave ~95 registers a thread: 20 warps per SM, against 16 with eight heads
// a batch; the prologue is bound by memory latency).  k_raw == nullptr:
// queries only.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
    token_prologue_kernel(const T* __restrict__ q_raw, const T* __restrict__ wq,
                          T* __restrict__ q_hat, const T* __restrict__ k_raw,
                          const T* __restrict__ v_raw, const T* __restrict__ wk, int B, int T_,
                          int p0, int Hq, int Hkv, KVDst d0, KVDst d1,
                          int32_t* __restrict__ len_out, const __grid_constant__ RopeParams rope,
                          float eps) {
  constexpr int E = D / 64, NB = 4;
  __shared__ double inv_freq[D / 2];
  for (int k = threadIdx.x; k < D / 2; k += blockDim.x) inv_freq[k] = rope.inv_freq[k];
  __syncthreads();
  const long tok = (long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tok >= (long)B * T_) return;
  const int lane = threadIdx.x & 31;
  const long b = tok / T_;
  const long t = p0 + tok % T_;  // position of the token
  // the loads of the first batch of query heads and of the first K/V head
  // go out together, and the RoPE factors (fp64 angle reduction) are
  // computed while they are in flight
  float x0[NB][E], x1[NB][E];
  auto load_q = [&](int h0) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int h = min(h0 + j, Hq - 1);  // tail: recompute the last head, store once
      const T* src = q_raw + (tok * Hq + h) * D;
      Vec<T, E>::load(src + lane * E, x0[j]);
      Vec<T, E>::load(src + D / 2 + lane * E, x1[j]);
    }
  };
  load_q(0);
  const T* vsrc = v_raw ? v_raw : k_raw;
  float kv0[2][E], kv1[2][E];
  if (k_raw) {
    const long off = tok * Hkv * D;
    Vec<T, E>::load(k_raw + off + lane * E, kv0[0]);
    Vec<T, E>::load(k_raw + off + D / 2 + lane * E, kv1[0]);
    Vec<T, E>::load(vsrc + off + lane * E, kv0[1]);
    Vec<T, E>::load(vsrc + off + D / 2 + lane * E, kv1[1]);
  }
  float w0[E], w1[E];
  Vec<T, E>::load(wq + lane * E, w0);
  Vec<T, E>::load(wq + D / 2 + lane * E, w1);
  float c[E], s[E];
  bool rot[E];
  rope_factors<D>(t, inv_freq, rope.rotated_pairs, c, s, rot);
  for (int h0 = 0; h0 < Hq; h0 += NB) {
    if (h0 > 0) load_q(h0);
    norm_rope<D, NB>(x0, x1, w0, w1, c, s, rot, true, eps);
#pragma unroll
    for (int j = 0; j < NB; ++j)
      if (h0 + j < Hq) store_vec<T, D>(q_hat + (tok * Hq + h0 + j) * D, x0[j], x1[j]);
  }
  if (!k_raw) return;
  Vec<T, E>::load(wk + lane * E, w0);
  Vec<T, E>::load(wk + D / 2 + lane * E, w1);
  for (int h = 0; h < Hkv; ++h) {
    float x0[2][E], x1[2][E];
    const long off = (tok * Hkv + h) * D;
    if (h == 0) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x0[0][e] = kv0[0][e];
        x1[0][e] = kv1[0][e];
        x0[1][e] = kv0[1][e];
        x1[1][e] = kv1[1][e];
      }
    } else {
      Vec<T, E>::load(k_raw + off + lane * E, x0[0]);
      Vec<T, E>::load(k_raw + off + D / 2 + lane * E, x1[0]);
      Vec<T, E>::load(vsrc + off + lane * E, x0[1]);
      Vec<T, E>::load(vsrc + off + D / 2 + lane * E, x1[1]);
    }
    norm_rope<D, 1>(x0, x1, w0, w1, c, s, rot, true, eps);
    norm_rope<D, 1>(x0 + 1, x1 + 1, nullptr, nullptr, c, s, rot, false, eps);
    put_kv<T, D>(d0, Hkv, b, h, t, x0[0], x1[0], x0[1], x1[1]);
    put_kv<T, D>(d1, Hkv, b, h, t, x0[0], x1[0], x0[1], x1[1]);
  }
  if (len_out && t == p0 && lane == 0) len_out[b] = p0 + T_;
}

// Raw bf16 values kept packed (two per 32-bit word) between their load and
// their use: the E = D/64 elements a lane holds of one half of a head.
template <int E>
struct PackedHalf {
  static constexpr int W = E / 2;
  uint32_t w[W];
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    if constexpr (W == 4) {
      const uint4 v = *reinterpret_cast<const uint4*>(p);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (W == 2) {
      const uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x; w[1] = v.y;
    } else {
      w[0] = *reinterpret_cast<const uint32_t*>(p);
    }
  }
  // bf16 -> fp32 is exact: the bits move into the high half of the word
  __device__ __forceinline__ void unpack(float* x) const {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// Prologue of a whole prompt for bf16 heads of 128/256/512: as
// token_prologue_kernel, but the raw vectors of up to NQ query heads and NKV
// key/value heads are loaded together, kept packed, before any arithmetic,
// so a warp has ~2-5 KB of loads in flight at once (the kernel is bound by
// memory latency: bytes in flight per SM set its rate).  Heads are then
// normalised and rotated two at a time (the two norms' shuffles interleave).
template <int D, int NQ, int NKV>
__global__ void __launch_bounds__(kWarps * 32)
    token_prologue_packed_kernel(const __nv_bfloat16* __restrict__ q_raw,
                                 const __nv_bfloat16* __restrict__ wq,
                                 __nv_bfloat16* __restrict__ q_hat,
                                 const __nv_bfloat16* __restrict__ k_raw,
                                 const __nv_bfloat16* __restrict__ v_raw,
                                 const __nv_bfloat16* __restrict__ wk, int B, int T_, int p0,
                                 int Hq, int Hkv, KVDst d0, KVDst d1,
                                 int32_t* __restrict__ len_out,
                                 const __grid_constant__ RopeParams rope, float eps) {
  using bf16 = __nv_bfloat16;
  constexpr int E = D / 64;
  static_assert(E % 2 == 0 && NQ % 2 == 0, "packed pairs, heads two at a time");
  __shared__ double inv_freq[D / 2];
  for (int k = threadIdx.x; k < D / 2; k += blockDim.x) inv_freq[k] = rope.inv_freq[k];
  __syncthreads();
  const long tok = (long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tok >= (long)B * T_) return;
  const int lane = threadIdx.x & 31;
  const long b = tok / T_;
  const long t = p0 + tok % T_;  // position of the token
  PackedHalf<E> q[NQ][2];
  auto load_q = [&](int h0) {
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
      const int h = min(h0 + j, Hq - 1);  // tail: reload the last head, store it once
      const bf16* src = q_raw + (tok * Hq + h) * D + lane * E;
      q[j][0].load(src);
      q[j][1].load(src + D / 2);
    }
  };
  PackedHalf<E> kv[NKV][2][2];  // [head][K or V][half]
  const bf16* vsrc = v_raw ? v_raw : k_raw;
  auto load_kv = [&](int h0) {
#pragma unroll
    for (int j = 0; j < NKV; ++j) {
      const long off = (tok * Hkv + min(h0 + j, Hkv - 1)) * D + lane * E;
      kv[j][0][0].load(k_raw + off);
      kv[j][0][1].load(k_raw + off + D / 2);
      kv[j][1][0].load(vsrc + off);
      kv[j][1][1].load(vsrc + off + D / 2);
    }
  };
  load_q(0);
  if (k_raw) load_kv(0);
  float w0[E], w1[E];
  Vec<bf16, E>::load(wq + lane * E, w0);
  Vec<bf16, E>::load(wq + D / 2 + lane * E, w1);
  float c[E], s[E];
  bool rot[E];
  rope_factors<D>(t, inv_freq, rope.rotated_pairs, c, s, rot);
  for (int h0 = 0; h0 < Hq; h0 += NQ) {
    if (h0 > 0) load_q(h0);
#pragma unroll
    for (int j = 0; j < NQ; j += 2) {
      float x0[2][E], x1[2][E];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        q[j + u][0].unpack(x0[u]);
        q[j + u][1].unpack(x1[u]);
      }
      norm_rope<D, 2>(x0, x1, w0, w1, c, s, rot, true, eps);
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (h0 + j + u < Hq) store_vec<bf16, D>(q_hat + (tok * Hq + h0 + j + u) * D, x0[u], x1[u]);
    }
  }
  if (!k_raw) return;
  Vec<bf16, E>::load(wk + lane * E, w0);
  Vec<bf16, E>::load(wk + D / 2 + lane * E, w1);
  for (int h0 = 0; h0 < Hkv; h0 += NKV) {
    if (h0 > 0) load_kv(h0);
#pragma unroll
    for (int j = 0; j < NKV; ++j) {
      if (h0 + j >= Hkv) break;
      float x0[2][E], x1[2][E];  // [K, V]
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        kv[j][u][0].unpack(x0[u]);
        kv[j][u][1].unpack(x1[u]);
      }
      norm_rope<D, 1>(x0, x1, w0, w1, c, s, rot, true, eps);
      norm_rope<D, 1>(x0 + 1, x1 + 1, nullptr, nullptr, c, s, rot, false, eps);
      put_kv<bf16, D>(d0, Hkv, b, h0 + j, t, x0[0], x1[0], x0[1], x1[1]);
      put_kv<bf16, D>(d1, Hkv, b, h0 + j, t, x0[0], x1[0], x0[1], x1[1]);
    }
  }
  if (len_out && t == p0 && lane == 0) len_out[b] = p0 + T_;
}

// lo/hi of every row of a sliding layer with image blocks: the window
// [max(0, i-w+1), i] united with the maximal run of equal non-negative ids
// that contains i.
__global__ void block_interval_kernel(const int32_t* __restrict__ ids, int B, int T_, int window,
                                      int32_t* __restrict__ lo, int32_t* __restrict__ hi) {
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)B * T_) return;
  const int i = (int)(idx % T_);
  const int32_t* row = ids + (idx - i);
  int a = i - window + 1;
  if (a < 0) a = 0;
  int e = i;
  const int id = row[i];
  if (id >= 0) {
    int s = i;
    while (s > 0 && row[s - 1] == id) --s;
    while (e + 1 < T_ && row[e + 1] == id) ++e;
    if (s < a) a = s;
  }
  lo[idx] = a;
  hi[idx] = e;
}

// One token per sequence into the cache: CTA b, warp h = KV head.
template <typename T, int D>
__global__ void append_kernel(const T* __restrict__ k_raw, const T* __restrict__ v_raw,
                              const T* __restrict__ wk, T* __restrict__ cache_k,
                              T* __restrict__ cache_v, int32_t* __restrict__ len, int Hkv, int cap,
                              int rolling, int* status, const __grid_constant__ RopeParams rope,
                              float eps) {
  const int b = blockIdx.x;
  const int h = threadIdx.x >> 5;
  const int pos = len[b];
  if (!rolling && pos >= cap) {  // whole block takes this branch
    if (threadIdx.x == 0) record_status(status, G4ATTN_ECACHE_OVERFLOW);
    return;
  }
  const long slot = rolling ? pos % cap : pos;
  const long src = ((long)b * Hkv + h) * D;
  const long dst = (((long)b * Hkv + h) * cap + slot) * D;
  float y0[D / 64], y1[D / 64];
  if (cache_v) {
    prologue_vec<T, D>(k_raw + src, wk, pos, &rope, eps, y0, y1);
    store_vec<T, D>(cache_k + dst, y0, y1);
  }
  // V; a single-tensor cache (cache_v == nullptr, K=V layer) keeps V alone
  prologue_vec<T, D>((v_raw ? v_raw : k_raw) + src, nullptr, pos, nullptr, eps, y0, y1);
  store_vec<T, D>(cache_v ? cache_v + dst : cache_k + dst, y0, y1);
  __syncthreads();  // every warp has read len[b]
  if (threadIdx.x == 0) len[b] = pos + 1;
}

// ---------------------------------------------------------------------------

template <typename F>
static cudaError_t dispatch(const LayerCfg& L, F&& f) {
  // f.template operator()<T, D>() for the layer's dtype and head size
  switch (L.d) {
    case 64: return L.dtype ? f.template operator()<float, 64>() : f.template operator()<__nv_bfloat16, 64>();
    case 128: return L.dtype ? f.template operator()<float, 128>() : f.template operator()<__nv_bfloat16, 128>();
    case 256: return L.dtype ? f.template operator()<float, 256>() : f.template operator()<__nv_bfloat16, 256>();
    case 512: return L.dtype ? f.template operator()<float, 512>() : f.template operator()<__nv_bfloat16, 512>();
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_token_prologue(const LayerCfg& L, int B, int T, int p0, const void* q_raw,
                                  const void* wq, void* q_hat, const void* k_raw,
                                  const void* v_raw, const void* wk, KVDst d0, KVDst d1,
                                  int32_t* len_out, cudaStream_t s) {
  const long n_tok = (long)B * T;
  const unsigned grid = (unsigned)((n_tok + kWarps - 1) / kWarps);
  using bf16 = __nv_bfloat16;
  if (L.dtype == 0 && L.d >= 128) {  // bf16: the packed-load kernel
    auto go = [&](auto kern) {
      kern<<<grid, kWarps * 32, 0, s>>>(
          static_cast<const bf16*>(q_raw), static_cast<const bf16*>(wq),
          static_cast<bf16*>(q_hat), static_cast<const bf16*>(k_raw),
          static_cast<const bf16*>(v_raw), static_cast<const bf16*>(wk), B, T, p0, L.Hq, L.Hkv,
          d0, d1, len_out, L.rope, L.eps);
      count_launch();
      return cudaGetLastError();
    };
    switch (L.d) {
      case 128: return go(token_prologue_packed_kernel<128, 8, 2>);
      case 256: return go(token_prologue_packed_kernel<256, 8, 1>);
      case 512: return go(token_prologue_packed_kernel<512, 4, 1>);
    }
  }
  return dispatch(L, [&]<typename E, int D>() {
    token_prologue_kernel<E, D><<<grid, kWarps * 32, 0, s>>>(
        static_cast<const E*>(q_raw), static_cast<const E*>(wq), static_cast<E*>(q_hat),
        static_cast<const E*>(k_raw), static_cast<const E*>(v_raw), static_cast<const E*>(wk), B,
        T, p0, L.Hq, L.Hkv, d0, d1, len_out, L.rope, L.eps);
    count_launch();
    return cudaGetLastError();
  });
}

cudaError_t launch_block_intervals(const LayerCfg& L, int B, int T, const int32_t* ids,
                                   int32_t* lo, int32_t* hi, cudaStream_t s) {
  const long n = (long)B * T;
  block_interval_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(ids, B, T, L.window, lo, hi);
  count_launch();
  return cudaGetLastError();
}

// lo/hi of every row of a chunk at positions p0 .. p0+T-1 of a prompt of
// p0 + T tokens (cached prefill): a global row sees [0, pos], a bidirectional
// one [0, p0 + T - 1]; a sliding row
// its window [max(0, pos-w+1), pos] united with the maximal run of equal
// non-negative ids (ids [B][p0 + T], or nullptr) that contains pos, seen up
// to the chunk's last position.
__global__ void chunk_interval_kernel(const int32_t* __restrict__ ids, int B, int T_, int p0,
                                      int layer_type, int window, const int2* __restrict__ span,
                                      int32_t* __restrict__ lo, int32_t* __restrict__ hi) {
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)B * T_) return;
  const int i = (int)(idx % T_);
  const long b = idx / T_;
  const int Tk = p0 + T_;
  const int pos = p0 + i;
  int a = 0, e = pos;
  if (layer_type == 2) {  // bidirectional: every position of the sequence
    e = Tk - 1;
  } else if (layer_type != 1) {
    a = pos - window + 1;
    if (a < 0) a = 0;
    if (ids) {
      const int32_t* row = ids + b * Tk;
      const int id = row[pos];
      if (id >= 0) {
        int s = pos;
        while (s > 0 && row[s - 1] == id) --s;
        while (e + 1 < Tk && row[e + 1] == id) ++e;
        if (s < a) a = s;
      }
    }
  }
  if (span) {  // keys outside [first kept, last kept] are padding: not visited
    a = max(a, span[b].x);
    e = min(e, span[b].y);  // a > e: the row has no key
  }
  lo[idx] = a;
  hi[idx] = e;
}

cudaError_t launch_chunk_intervals(const LayerCfg& L, int B, int T, int p0, const int32_t* ids,
                                   const int2* span, int32_t* lo, int32_t* hi, cudaStream_t s) {
  const long n = (long)B * T;
  chunk_interval_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
      ids, B, T, p0, L.layer_type, L.window, span, lo, hi);
  count_launch();
  return cudaGetLastError();
}

// First and last kept position of each sequence's padding mask (uint8
// [B][Tk], non-zero = keep): span[b] = (first, last), or (Tk, -1) when the
// whole sequence is padding.  One block per sequence.
__global__ void mask_span_kernel(const uint8_t* __restrict__ mask, int Tk,
                                 int2* __restrict__ span) {
  __shared__ int s_first, s_last;
  if (threadIdx.x == 0) {
    s_first = Tk;
    s_last = -1;
  }
  __syncthreads();
  const uint8_t* row = mask + (long)blockIdx.x * Tk;
  int f = Tk, l = -1;
  for (int t = threadIdx.x; t < Tk; t += blockDim.x)
    if (row[t]) {
      f = min(f, t);
      l = max(l, t);
    }
  f = __reduce_min_sync(0xffffffffu, f);
  l = __reduce_max_sync(0xffffffffu, l);
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&s_first, f);
    atomicMax(&s_last, l);
  }
  __syncthreads();
  if (threadIdx.x == 0) span[blockIdx.x] = make_int2(s_first, s_last);
}

cudaError_t launch_mask_span(int B, int Tk, const uint8_t* mask, int2* span, cudaStream_t s) {
  mask_span_kernel<<<B, 256, 0, s>>>(mask, Tk, span);
  count_launch();
  return cudaGetLastError();
}

// Padding mask as bits, one thread per 64-key word: bit k of word t of
// sequence b is 1 when key 64 t + k is kept (mask byte non-zero); keys past
// the mask's end (the last word's tail) read as kept, and no row sees them.
__global__ void mask_bits_kernel(const uint8_t* __restrict__ mask, int B, int Tk, int words,
                                 uint64_t* __restrict__ bits) {
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)B * words) return;
  const long b = idx / words;
  const int t = (int)(idx % words);
  const uint8_t* row = mask + b * Tk;
  const int k0 = t * 64;
  const int n = min(64, Tk - k0);
  uint64_t v = ~0ull;
  for (int k = 0; k < n; ++k)
    if (row[k0 + k] == 0) v &= ~(1ull << k);
  bits[idx] = v;
}

cudaError_t launch_mask_bits(int B, int Tk, const uint8_t* mask, uint64_t* bits, int words,
                             cudaStream_t s) {
  const long n = (long)B * words;
  if (n == 0) return cudaSuccess;
  mask_bits_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(mask, B, Tk, words, bits);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_append(const LayerCfg& L, int B, const void* k_raw, const void* v_raw,
                          const void* wk, void* cache_k, void* cache_v, int32_t* len, int cap,
                          int rolling, int* status, cudaStream_t s) {
  return dispatch(L, [&]<typename E, int D>() {
    append_kernel<E, D><<<B, 32 * L.Hkv, 0, s>>>(
        static_cast<const E*>(k_raw), static_cast<const E*>(v_raw), static_cast<const E*>(wk),
        static_cast<E*>(cache_k), static_cast<E*>(cache_v), len, L.Hkv, cap, rolling, status,
        L.rope, L.eps);
    count_launch();
    return cudaGetLastError();
  });
}

}  // namespace g4
