// Shared device helpers of the g4attn CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "g4attn_internal.h"

namespace g4 {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Load / store N consecutive elements (N * sizeof(T) bytes, naturally
// aligned) as fp32, using the widest vector access the size allows.
template <typename T, int N> struct Vec;
template <int N> struct Vec<float, N> {
  __device__ __forceinline__ static void load(const float* p, float* x) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 4) {
        float4 v = *reinterpret_cast<const float4*>(p + i);
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
      }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 2) {
        float2 v = *reinterpret_cast<const float2*>(p + i);
        x[i] = v.x; x[i + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) x[i] = p[i];
    }
  }
  __device__ __forceinline__ static void store(float* p, const float* x) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 4)
        *reinterpret_cast<float4*>(p + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
    } else if constexpr (N % 2 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 2) *reinterpret_cast<float2*>(p + i) = make_float2(x[i], x[i + 1]);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) p[i] = x[i];
    }
  }
};
template <int N> struct Vec<__nv_bfloat16, N> {
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* x) {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 8) {
        uint4 v = *reinterpret_cast<const uint4*>(p + i);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 f = __bfloat1622float2(h[j]);
          x[i + 2 * j] = f.x; x[i + 2 * j + 1] = f.y;
        }
      }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 2) {
        float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p + i));
        x[i] = f.x; x[i + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) x[i] = __bfloat162float(p[i]);
    }
  }
  __device__ __forceinline__ static void store(__nv_bfloat16* p, const float* x) {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 8) {
        uint4 v;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(x[i + 2 * j], x[i + 2 * j + 1]);
        *reinterpret_cast<uint4*>(p + i) = v;
      }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
      for (int i = 0; i < N; i += 2)
        *reinterpret_cast<__nv_bfloat162*>(p + i) = __floats2bfloat162_rn(x[i], x[i + 1]);
    } else {
#pragma unroll
      for (int i = 0; i < N; ++i) p[i] = __float2bfloat16_rn(x[i]);
    }
  }
};

// sin/cos of the RoPE angle pos * f from the frequency in turns as a 64-bit
// binary fraction, F = f / (2 pi) * 2^64: the fractional turns of pos * f
// are bits 32..63 of the wrapping integer product pos * F (two integer
// multiplies, no fp64), read as a signed fraction in [-1/2, 1/2) turn and
// handed to the hardware approximation on [-pi, pi).  F carries f to 2^-53
// relative, as the fp64 product in rope_sincos does; the 32-bit turn rounds
// to 24 bits in the float conversion (2e-7 rad).
__device__ __forceinline__ void rope_sincos_turns(uint32_t pos, unsigned long long F, float* s,
                                                  float* c) {
  const uint32_t lo = (uint32_t)F, hi = (uint32_t)(F >> 32);
  const uint32_t top = __umulhi(lo, pos) + hi * pos;
  const float turns = (float)(int32_t)top * 2.3283064365386963e-10f;  // 2^-32
  __sincosf(turns * 6.283185307179586f, s, c);
}

// Angle pos * inv_freq reduced to [-pi, pi] in fp64, then sin/cos in fp32.
// (pos * inv_freq in fp32 would err by up to ~1e-2 rad at pos ~ 1.3e5.)
__device__ __forceinline__ void rope_sincos(long pos, double inv_freq, float* s, float* c) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = (double)pos * inv_freq;
  double n = rint(a * (1.0 / two_pi));
  double r = fma(-n, two_pi, a);
  // |r| <= pi: the hardware approximation's absolute error there (~4e-7) is
  // far below the fp32 and bf16 tolerances
  __sincosf((float)r, s, c);
}

// Prologue of one head vector by one warp:
//   y = x / sqrt(mean(x^2) + eps) * w      (w == nullptr: weightless)
//   then RoPE at `pos` on the pairs (k, k + D/2), k < rope.rotated_pairs
//   (rope == nullptr: no rotation).
// Lane l holds elements [l*E, l*E+E) of each half, E = D/64, so every RoPE
// pair lives in one lane and the loads are contiguous across the warp.
template <typename T, int D>
__device__ __forceinline__ void prologue_vec(const T* __restrict__ src, const T* __restrict__ w,
                                             long pos, const RopeParams* rope, float eps,
                                             float* y0, float* y1) {
  constexpr int E = D / 64;
  const int lane = threadIdx.x & 31;
  float x0[E], x1[E];
  Vec<T, E>::load(src + lane * E, x0);
  Vec<T, E>::load(src + D / 2 + lane * E, x1);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) ss += x0[e] * x0[e] + x1[e] * x1[e];
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)D + eps);
  float w0[E], w1[E];
  if (w) {
    Vec<T, E>::load(w + lane * E, w0);
    Vec<T, E>::load(w + D / 2 + lane * E, w1);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) w0[e] = w1[e] = 1.f;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    y0[e] = x0[e] * r * w0[e];
    y1[e] = x1[e] * r * w1[e];
  }
  if (rope) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int k = lane * E + e;
      if (k < rope->rotated_pairs) {
        float s, c;
        rope_sincos(pos, rope->inv_freq[k], &s, &c);
        const float a = y0[e], b = y1[e];
        y0[e] = a * c - b * s;
        y1[e] = a * s + b * c;
      }
    }
  }
}

// RoPE factors of one token for the pairs a lane holds (k = lane*E + e,
// E = D/64): rot[e] = 0 marks a pass-through pair.  inv_freq: the layer's
// frequencies in shared memory (a per-lane index into the kernel's parameter
// space would serialise the warp's 32 reads).
template <int D>
__device__ __forceinline__ void rope_factors(long pos, const double* inv_freq, int rotated_pairs,
                                             float* c, float* s, bool* rot) {
  constexpr int E = D / 64;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int k = lane * E + e;
    rot[e] = k < rotated_pairs;
    c[e] = 1.f;
    s[e] = 0.f;
    if (rot[e]) rope_sincos(pos, inv_freq[k], &s[e], &c[e]);
  }
}

// RMSNorm (x * rsqrt(mean(x^2) + eps) * w) and optional RoPE of NH head
// vectors of one token already loaded into registers (x0/x1: the two halves,
// E = D/64 values per lane each), in place.  w0/w1 == nullptr: no weight.
template <int D, int NH>
__device__ __forceinline__ void norm_rope(float (*x0)[D / 64], float (*x1)[D / 64], const float* w0,
                                          const float* w1, const float* c, const float* s,
                                          const bool* rot, bool rope, float eps) {
  constexpr int E = D / 64;
  float ss[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    ss[h] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ss[h] += x0[h][e] * x0[h][e] + x1[h][e] * x1[h][e];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int h = 0; h < NH; ++h) ss[h] += __shfl_xor_sync(0xffffffffu, ss[h], o);
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    const float r = rsqrtf(ss[h] / (float)D + eps);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float a = x0[h][e] * r, b = x1[h][e] * r;
      if (w0) {
        a *= w0[e];
        b *= w1[e];
      }
      if (rope && rot[e]) {
        const float a2 = a * c[e] - b * s[e];
        b = a * s[e] + b * c[e];
        a = a2;
      }
      x0[h][e] = a;
      x1[h][e] = b;
    }
  }
}

template <typename T, int D>
__device__ __forceinline__ void store_vec(T* __restrict__ dst, const float* y0, const float* y1) {
  constexpr int E = D / 64;
  const int lane = threadIdx.x & 31;
  Vec<T, E>::store(dst + lane * E, y0);
  Vec<T, E>::store(dst + D / 2 + lane * E, y1);
}

__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace g4
