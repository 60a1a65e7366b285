// Masked softmax attention on CUDA cores in fp32 (any head size, bf16 or
// fp32 data).  This is the exact path of the library: it is the only one that
// meets the fp32 tolerance (tensor-core operands are bf16), and it serves
// every mask the layer has:
//   sliding rows  [max(0, i-w+1), i]   ("Gemma 4" overview blog,
//                                       "Sliding-window attention")
//   image blocks  window U block        ("Gemma 4" Keras docs, "What changed")
//   global rows   [0, i]                (overview blog, "Global attention layers")
//   padding keys  dropped               ("Gemma 4" Keras docs,
//                                        "Gemma4ConditionalGenerate": attention_mask)
// with an optional logit soft-cap s -> c tanh(s / c) ("gemma4-pt-claude"
// README, "Attention Backend Notes").  A row left without any key outputs 0.
// Key tiles outside the union of a CTA's row intervals are never visited.
//
// CTA = (32 query rows, one query head, one sequence); 8 warps x 4 rows.
// Keys stream through shared memory 32 at a time; lane j scores key j, then
// the warp accumulates o += p_j v_j with p_j broadcast by shuffles.
#include "common.cuh"

namespace g4 {

constexpr int kSimtRows = 32;
constexpr int kSimtKeys = 32;
constexpr int kSimtRowsPerWarp = 4;

template <int D>
constexpr size_t simt_smem_bytes() {
  return sizeof(float) * (size_t)(kSimtRows * D + kSimtKeys * (D + 1) + kSimtKeys * D);
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
    attn_simt_kernel(const T* __restrict__ q_hat, KVSrc kv, RowIntervals rows, KeyBits kb,
                     T* __restrict__ out, int T_, int Hq, int Hkv, int layer_type, int window,
                     float scale, float cap) {
  extern __shared__ float smem[];
  float* sq = smem;                      // [rows][D]
  float* sk = sq + kSimtRows * D;        // [keys][D + 1] (padded: lane j reads row j)
  float* sv = sk + kSimtKeys * (D + 1);  // [keys][D]
  __shared__ int s_lo[kSimtRows], s_hi[kSimtRows];
  __shared__ int s_range[2];

  const int b = blockIdx.z, h = blockIdx.y, r0 = blockIdx.x * kSimtRows;
  const int kvh = h / (Hq / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int idx = threadIdx.x; idx < kSimtRows * D; idx += blockDim.x) {
    const int r = idx / D, c = idx % D, i = r0 + r;
    sq[idx] = i < T_ ? to_f(q_hat[(((long)b * T_ + i) * Hq + h) * D + c]) : 0.f;
  }
  if (threadIdx.x < kSimtRows) {
    const int i = r0 + threadIdx.x;
    int lo = 1, hi = 0;  // empty
    if (i < T_) {
      if (rows.lo) {
        lo = rows.lo[(long)b * T_ + i];
        hi = rows.hi[(long)b * T_ + i];
      } else if (layer_type == 1) {
        lo = 0;
        hi = i;
      } else {
        lo = max(0, i - window + 1);
        hi = i;
      }
    }
    s_lo[threadIdx.x] = lo;
    s_hi[threadIdx.x] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0x7fffffff, e = -1;
    for (int r = 0; r < kSimtRows; ++r)
      if (s_lo[r] <= s_hi[r]) {
        a = min(a, s_lo[r]);
        e = max(e, s_hi[r]);
      }
    s_range[0] = a;
    s_range[1] = e;
  }
  __syncthreads();
  const int klo = s_range[0], khi = s_range[1];

  constexpr int C = D / 32;
  float m[kSimtRowsPerWarp], l[kSimtRowsPerWarp], o[kSimtRowsPerWarp][C];
#pragma unroll
  for (int rr = 0; rr < kSimtRowsPerWarp; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) o[rr][c] = 0.f;
  }

  const long kv_base = ((long)b * Hkv + kvh) * kv.cap * D;
  const T* K = static_cast<const T*>(kv.k) + kv_base;
  const T* V = static_cast<const T*>(kv.v) + kv_base;

  for (int t0 = klo; t0 <= khi; t0 += kSimtKeys) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < kSimtKeys * D; idx += blockDim.x) {
      const int j = idx / D, c = idx % D, key = t0 + j;
      const bool ok = key <= khi;
      sk[j * (D + 1) + c] = ok ? to_f(K[(long)key * D + c]) : 0.f;
      sv[j * D + c] = ok ? to_f(V[(long)key * D + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kSimtRowsPerWarp; ++rr) {
      const int r = warp * kSimtRowsPerWarp + rr;
      const int lo = s_lo[r], hi = s_hi[r];
      if (lo > hi || hi < t0 || lo >= t0 + kSimtKeys) continue;  // warp-uniform
      const int key = t0 + lane;
      const bool ok = key >= lo && key <= hi &&
                      (!kb.bits || ((kb.bits[(long)b * kb.words + (key >> 6)] >> (key & 63)) & 1));
      float s = -INFINITY;
      if (ok) {
        const float* qr = sq + r * D;
        const float* kr = sk + lane * (D + 1);
        float dot = 0.f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) dot = fmaf(qr[c], kr[c], dot);
        s = dot * scale;
        if (cap > 0.f) s = cap * tanhf(s / cap);
      }
      const float mn = fmaxf(m[rr], warp_max(s));
      if (mn == -INFINITY) continue;  // no key of this row so far (warp-uniform)
      const float p = ok ? expf(s - mn) : 0.f;
      const float corr = m[rr] == -INFINITY ? 0.f : expf(m[rr] - mn);
      l[rr] = l[rr] * corr + warp_sum(p);
      m[rr] = mn;
#pragma unroll
      for (int c = 0; c < C; ++c) o[rr][c] *= corr;
      for (int j = 0; j < kSimtKeys; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p, j);
        const float* vr = sv + j * D + lane;
#pragma unroll
        for (int c = 0; c < C; ++c) o[rr][c] = fmaf(pj, vr[32 * c], o[rr][c]);
      }
    }
  }

#pragma unroll
  for (int rr = 0; rr < kSimtRowsPerWarp; ++rr) {
    const int r = warp * kSimtRowsPerWarp + rr, i = r0 + r;
    if (i >= T_) continue;
    const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;  // no key: a zero row
    T* dst = out + (((long)b * T_ + i) * Hq + h) * D;
#pragma unroll
    for (int c = 0; c < C; ++c) dst[lane + 32 * c] = from_f<T>(o[rr][c] * inv);
  }
}

template <typename E, int D>
static cudaError_t run_simt(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                            RowIntervals rows, KeyBits kb, void* out, cudaStream_t s) {
  constexpr size_t smem = simt_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<E, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((T + kSimtRows - 1) / kSimtRows, L.Hq, B);
  attn_simt_kernel<E, D><<<grid, 256, smem, s>>>(static_cast<const E*>(q_hat), kv, rows, kb,
                                                  static_cast<E*>(out), T, L.Hq, L.Hkv,
                                                  L.layer_type, L.window, L.scale, L.softcap);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_attention_simt(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                  RowIntervals rows, KeyBits kb, void* out, cudaStream_t s) {
  const bool f32 = L.dtype == 1;
  switch (L.d) {
    case 64: return f32 ? run_simt<float, 64>(L, B, T, q_hat, kv, rows, kb, out, s)
                        : run_simt<__nv_bfloat16, 64>(L, B, T, q_hat, kv, rows, kb, out, s);
    case 128: return f32 ? run_simt<float, 128>(L, B, T, q_hat, kv, rows, kb, out, s)
                         : run_simt<__nv_bfloat16, 128>(L, B, T, q_hat, kv, rows, kb, out, s);
    case 256: return f32 ? run_simt<float, 256>(L, B, T, q_hat, kv, rows, kb, out, s)
                         : run_simt<__nv_bfloat16, 256>(L, B, T, q_hat, kv, rows, kb, out, s);
    case 512: return f32 ? run_simt<float, 512>(L, B, T, q_hat, kv, rows, kb, out, s)
                         : run_simt<__nv_bfloat16, 512>(L, B, T, q_hat, kv, rows, kb, out, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g4
