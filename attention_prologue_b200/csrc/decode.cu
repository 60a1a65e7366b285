// Single-token decode over a per-layer KV cache ("Gemma 4" Keras docs,
// "Gemma4ConditionalGenerate": decoding runs over the per-layer cache;
// "gemma4-pt-claude" README, "KV Cache": rolling sliding-window caches;
// "Gemma 4" overview blog, "Shared KV Cache": a later layer reads an earlier
// layer's cache and computes only its queries).
//
// Split-KV: the keys of sequence b, [lo, P] with P = len[b] - 1, are cut into
// fixed-size chunks on a grid aligned to 16 positions (chunk c covers
// [base + c*chunk, base + (c+1)*chunk) with base = lo rounded down to a
// multiple of 16, clipped to [lo, P]); CTA (chunk, KV head, sequence) computes for the query
// heads of that KV head the partial softmax of the chunk
//   m = max_j s_j,  l = sum_j e^{s_j - m},  o~ = sum_j e^{s_j - m} v_j,
// and the combine kernel merges the chunks with
//   o = sum_c e^{m_c - M} o~_c / sum_c e^{m_c - M} l_c,  M = max_c m_c.
// The query prologue (RMSNorm * w_q, RoPE at P) runs inside the split kernel.
// Padding keys of the prompt ("Gemma 4" Keras docs, "Gemma4ConditionalGenerate":
// attention_mask) are skipped, and scores take the optional logit soft-cap
// s -> c tanh(s / c) ("gemma4-pt-claude" README, "Attention Backend Notes");
// a chunk without a kept key yields m = -inf, l = 0, which the combine ignores.
#include "common.cuh"
#include "g4attn.h"

namespace g4 {

constexpr int kDecWarps = 4;
constexpr int kDecHeads = 4;  // query heads handled per pass over the chunk

DecodePlan decode_plan(const LayerCfg& L, int cap) {
  DecodePlan p;
  const long span = L.layer_type == 0 ? (long)(L.window < cap ? L.window : cap) : (long)cap;
  p.chunk = span <= 4096 ? 256 : 2048;  // a multiple of 16
  p.n_chunks = (int)((span + 15 + p.chunk - 1) / p.chunk);  // the aligned grid adds <= 15
  return p;
}

size_t decode_partials_bytes(const LayerCfg& L, int B, const DecodePlan& p) {
  return sizeof(float) * (size_t)B * L.Hq * p.n_chunks * (size_t)(L.d + 2);
}

__device__ __forceinline__ int decode_lo(int P, int layer_type, int window) {
  return layer_type == 0 ? max(0, P - window + 1) : 0;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecWarps * 32)
    decode_split_kernel(const T* __restrict__ q_raw, const T* __restrict__ wq,
                        const T* __restrict__ ck, const T* __restrict__ cv,
                        const int32_t* __restrict__ len, int cap, int rolling, int Hq, int Hkv,
                        int layer_type, int window, float scale, float softcap, KeyMask km,
                        float eps, int chunk, int nc, float* __restrict__ part_ml,
                        float* __restrict__ part_o, int* status,
                        const __grid_constant__ RopeParams rope) {
  constexpr int E = D / 32;  // contiguous elements per lane
  __shared__ float sq[kDecHeads][D];
  __shared__ float red_ml[kDecWarps][kDecHeads][2];
  __shared__ float red_o[kDecWarps][kDecHeads][D];

  const int c = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = Hq / Hkv;
  const int L = len[b];
  if (L <= 0 || (!rolling && L > cap)) {  // nothing to read / len past the end: no access
    if (c == 0 && kvh == 0 && threadIdx.x == 0)
      record_status(status, L <= 0 ? G4ATTN_ECACHE_EMPTY : G4ATTN_ECACHE_OVERFLOW);
    return;
  }
  const int P = L - 1;
  const int lo = decode_lo(P, layer_type, window);
  const int c0 = (lo & ~15) + c * chunk;
  if (c0 > P) return;
  const int k_begin = max(lo, c0);
  const int k_end = min(P + 1, c0 + chunk);
  const long kv_base = ((long)b * Hkv + kvh) * cap;

  for (int hg = 0; hg < g; hg += kDecHeads) {
    const int nh = min(kDecHeads, g - hg);
    if (warp < nh) {
      const int h = kvh * g + hg + warp;
      float y0[D / 64], y1[D / 64];
      prologue_vec<T, D>(q_raw + ((long)b * Hq + h) * D, wq, P, &rope, eps, y0, y1);
#pragma unroll
      for (int e = 0; e < D / 64; ++e) {
        sq[warp][lane * (D / 64) + e] = y0[e];
        sq[warp][D / 2 + lane * (D / 64) + e] = y1[e];
      }
    }
    __syncthreads();
    float q[kDecHeads][E], o[kDecHeads][E], m[kDecHeads], l[kDecHeads];
#pragma unroll
    for (int hh = 0; hh < kDecHeads; ++hh) {
      m[hh] = -INFINITY;
      l[hh] = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        q[hh][e] = hh < nh ? sq[hh][lane * E + e] : 0.f;
        o[hh][e] = 0.f;
      }
    }
    for (int key = k_begin + warp; key < k_end; key += kDecWarps) {
      if (km.keep && key < km.len && km.keep[(long)b * km.len + key] == 0) continue;  // padding
      const long slot = rolling ? key % cap : key;
      float kf[E], vf[E];
      Vec<T, E>::load(ck + (kv_base + slot) * D + lane * E, kf);
      Vec<T, E>::load(cv + (kv_base + slot) * D + lane * E, vf);
#pragma unroll
      for (int hh = 0; hh < kDecHeads; ++hh) {
        if (hh >= nh) break;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) dot = fmaf(q[hh][e], kf[e], dot);
        float s = warp_sum(dot) * scale;
        if (softcap > 0.f) s = softcap * tanhf(s / softcap);
        const float mn = fmaxf(m[hh], s);
        const float corr = expf(m[hh] - mn);
        const float p = expf(s - mn);
        l[hh] = l[hh] * corr + p;
        m[hh] = mn;
#pragma unroll
        for (int e = 0; e < E; ++e) o[hh][e] = fmaf(p, vf[e], o[hh][e] * corr);
      }
    }
#pragma unroll
    for (int hh = 0; hh < kDecHeads; ++hh) {
      if (lane == 0) {
        red_ml[warp][hh][0] = m[hh];
        red_ml[warp][hh][1] = l[hh];
      }
#pragma unroll
      for (int e = 0; e < E; ++e) red_o[warp][hh][lane * E + e] = o[hh][e];
    }
    __syncthreads();
    for (int hh = 0; hh < nh; ++hh) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, red_ml[w][hh][0]);
      float a[kDecWarps], den = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        a[w] = red_ml[w][hh][0] == -INFINITY ? 0.f : expf(red_ml[w][hh][0] - M);
        den += a[w] * red_ml[w][hh][1];
      }
      const long pidx = ((long)b * Hq + kvh * g + hg + hh) * nc + c;
      if (threadIdx.x == 0) {
        part_ml[2 * pidx] = M;
        part_ml[2 * pidx + 1] = den;
      }
      for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) acc += a[w] * red_o[w][hh][dim];
        part_o[pidx * D + dim] = acc;
      }
    }
    __syncthreads();
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float* __restrict__ part_ml, const float* __restrict__ part_o,
                          const int32_t* __restrict__ len, int Hq, int layer_type, int window,
                          int chunk, int nc, int cap, int rolling, T* __restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y;
  T* dst = out + ((long)b * Hq + h) * D;
  const int L = len[b];
  if (L <= 0 || (!rolling && L > cap)) {
    for (int dim = threadIdx.x; dim < D; dim += blockDim.x) dst[dim] = from_f<T>(0.f);
    return;
  }
  const int P = L - 1;
  const int n = P + 1 - (decode_lo(P, layer_type, window) & ~15);
  const int cnt = (n + chunk - 1) / chunk;
  const long base = ((long)b * Hq + h) * nc;
  float M = -INFINITY;
  for (int c = 0; c < cnt; ++c) M = fmaxf(M, part_ml[2 * (base + c)]);
  // a chunk with m = -inf (no key, or a split CTA that gave up) weighs 0
  auto weight = [&](int c) {
    const float m = part_ml[2 * (base + c)];
    return m == -INFINITY ? 0.f : expf(m - M);
  };
  float den = 0.f;
  for (int c = 0; c < cnt; ++c) den += weight(c) * part_ml[2 * (base + c) + 1];
  const float inv = den > 0.f ? 1.f / den : 0.f;  // no key at all: a zero output
  for (int dim = threadIdx.x; dim < D; dim += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < cnt; ++c) acc += weight(c) * part_o[(base + c) * D + dim];
    dst[dim] = from_f<T>(acc * inv);
  }
}

template <typename T, int D>
static cudaError_t run_decode(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                              const void* cache_k, const void* cache_v, const void* wk_single,
                              const int32_t* len, int cap, int rolling, KeyMask km,
                              const DecodePlan& plan, float* partials, void* out, int* status,
                              cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1) {
  float* part_ml = partials;
  float* part_o = partials + 2 * (size_t)B * L.Hq * plan.n_chunks;
  dim3 grid(plan.n_chunks, L.Hkv, B);
  if (ev0) cudaEventRecord(ev0, s);
  cudaError_t e;
  if (decode_mma_supported(L, cap, rolling)) {
    e = launch_decode_mma(L, B, q_raw, wq, cache_k, cache_v, wk_single, len, cap, rolling, km,
                          plan, part_ml, part_o, status, s);
  } else if (!cache_v) {  // a single-tensor cache needs the tensor-core kernel (host-checked)
    return cudaErrorInvalidValue;
  } else {
    decode_split_kernel<T, D><<<grid, kDecWarps * 32, 0, s>>>(
        static_cast<const T*>(q_raw), static_cast<const T*>(wq), static_cast<const T*>(cache_k),
        static_cast<const T*>(cache_v), len, cap, rolling, L.Hq, L.Hkv, L.layer_type, L.window,
        L.scale, L.softcap, km, L.eps, plan.chunk, plan.n_chunks, part_ml, part_o, status,
        L.rope);
    count_launch();
    e = cudaGetLastError();
  }
  if (ev1) cudaEventRecord(ev1, s);
  if (e != cudaSuccess) return e;
  decode_combine_kernel<T, D><<<dim3(L.Hq, B), 128, 0, s>>>(part_ml, part_o, len, L.Hq,
                                                            L.layer_type, L.window, plan.chunk,
                                                            plan.n_chunks, cap, rolling,
                                                            static_cast<T*>(out));
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                          const void* cache_k, const void* cache_v, const void* wk_single,
                          const int32_t* len, int cap, int rolling, KeyMask km,
                          const DecodePlan& plan, float* partials, void* out, int* status,
                          cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1) {
  const bool f32 = L.dtype == 1;
#define G4_DEC(D)                                                                             \
  return f32 ? run_decode<float, D>(L, B, q_raw, wq, cache_k, cache_v, wk_single, len, cap,  \
                                    rolling, km, plan, partials, out, status, s, ev0, ev1)     \
             : run_decode<__nv_bfloat16, D>(L, B, q_raw, wq, cache_k, cache_v, wk_single, len, \
                                            cap, rolling, km, plan, partials, out, status, s, \
                                            ev0, ev1)
  switch (L.d) {
    case 64: G4_DEC(64);
    case 128: G4_DEC(128);
    case 256: G4_DEC(256);
    case 512: G4_DEC(512);
  }
#undef G4_DEC
  return cudaErrorInvalidValue;
}

}  // namespace g4
