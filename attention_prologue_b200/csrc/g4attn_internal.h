// Internal interface between the C-ABI layer (api.cpp) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace g4 {

constexpr int kMaxHalf = 256;  // head_dim <= 512

// RoPE of one layer: pair k (k < rotated_pairs) turns by pos * inv_freq[k];
// inv_freq[k] = theta^(-2k/d) computed on the host in fp64.
struct RopeParams {
  double inv_freq[kMaxHalf];
  // the same frequencies in turns per position as 64-bit binary fractions,
  // F = inv_freq / (2 pi) * 2^64 (rope_sincos_turns)
  unsigned long long turns[kMaxHalf];
  int rotated_pairs;
};

// Validated copy of g4attn_layer_desc.
struct LayerCfg {
  int layer_type;  // 0 sliding, 1 global
  int window;
  int k_eq_v;
  int Hq, Hkv, d;
  int dtype;  // 0 bf16, 1 fp32
  float scale, eps;
  float softcap;  // logit soft-cap c (0: none)
  RopeParams rope;
};

// Soft-cap of a score already in log2 units: with C2 = c * log2(e),
// x -> C2 * tanh(x / C2) (the cap c * tanh(s / c) of the natural-log score
// s = x / log2(e)).  C2 == 0: no cap.
inline float softcap_log2(const LayerCfg& L) {
  return L.softcap > 0.f ? L.softcap * 1.4426950408889634f : 0.f;
}

// Where the key/value prologue writes: [B, Hkv, cap, d]; positions t >= first
// go to slot (rolling ? t % cap : t).  k == nullptr: no destination;
// v == nullptr: a single-tensor cache of a K=V layer, V alone goes to k.
struct KVDst {
  void* k;
  void* v;
  int cap;
  int rolling;
  int first;
};

// Keys of one attention source: [B, Hkv, cap, d], position t at slot t;
// positions 0 .. len-1 exist (a cached prefill reads len = p0 + T of them).
struct KVSrc {
  const void* k;
  const void* v;
  int cap;
  int len;
};

// Per-row key interval [lo[b*T+i], hi[b*T+i]] (image blocks), or nullptr
// when the interval follows from the layer type and window alone.
struct RowIntervals {
  const int32_t* lo;
  const int32_t* hi;
};

// Padding mask of the keys as bits: bit k of bits[b * words + t] is 1 when
// key position 64 t + k of sequence b is kept.  bits == nullptr: every key.
struct KeyBits {
  const uint64_t* bits;
  int words;
};

// bits [B][words] of a byte mask [B][Tk] (non-zero = keep); words = ceil(Tk / 64).
cudaError_t launch_mask_bits(int B, int Tk, const uint8_t* mask, uint64_t* bits, int words,
                             cudaStream_t s);

// Q, K and V prologue of T tokens at positions p0 .. p0+T-1 in one launch
// (one warp per token); k_raw == nullptr: queries only (KV-shared layer).
cudaError_t launch_token_prologue(const LayerCfg& L, int B, int T, int p0, const void* q_raw,
                                  const void* wq, void* q_hat, const void* k_raw,
                                  const void* v_raw, const void* wk, KVDst d0, KVDst d1,
                                  int32_t* len_out, cudaStream_t s);
cudaError_t launch_block_intervals(const LayerCfg& L, int B, int T, const int32_t* ids,
                                   int32_t* lo, int32_t* hi, cudaStream_t s);
// Per-row key intervals of a cached-prefill chunk (positions p0 .. p0+T-1);
// ids [B][p0 + T] or nullptr.
cudaError_t launch_chunk_intervals(const LayerCfg& L, int B, int T, int p0, const int32_t* ids,
                                   const int2* span, int32_t* lo, int32_t* hi, cudaStream_t s);
// span[b] = (first, last) kept position of sequence b's padding mask [B][Tk]
cudaError_t launch_mask_span(int B, int Tk, const uint8_t* mask, int2* span, cudaStream_t s);
cudaError_t launch_attention_simt(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                  RowIntervals rows, KeyBits kb, void* out, cudaStream_t s);
// tcgen05 prefill attention (bf16, head_dim 64/128/256/512); q_hat [B, T, Hq, d].
bool attention_sm100_supported(const LayerCfg& L);
cudaError_t launch_attention_sm100(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                   RowIntervals rows, KeyBits kb, void* out, int* status,
                                   cudaStream_t s);
// head_dim 512 on 2-CTA clusters (called by launch_attention_sm100).
cudaError_t launch_attention_pair(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                  RowIntervals rows, KeyBits kb, void* out, int* status,
                                  cudaStream_t s);

// Query heads packed into one 128-row prefill tile, as a power of two: the
// largest 2^g <= 8 dividing Hq / Hkv (every head of a tile reads the same KV
// head, so a tile spans 128 / 2^g positions).
inline int gqa_pack_log2(int Hq, int Hkv) {
  const int g = Hq / Hkv;
  int lg = 0;
  while (lg < 3 && g % (2 << lg) == 0) ++lg;
  return lg;
}
cudaError_t launch_append(const LayerCfg& L, int B, const void* k_raw, const void* v_raw,
                          const void* wk, void* cache_k, void* cache_v, int32_t* len, int cap,
                          int rolling, int* status, cudaStream_t s);

// Split-KV decode.  Partials: m, l [B, Hq, n_chunks] and o~ [B, Hq, n_chunks, d], fp32.
struct DecodePlan {
  int chunk;     // keys per chunk
  int n_chunks;  // chunks per (sequence, head), upper bound
};
DecodePlan decode_plan(const LayerCfg& L, int cap);
size_t decode_partials_bytes(const LayerCfg& L, int B, const DecodePlan& p);
// Padding mask of a cache's prompt positions: position p < len of sequence
// b is a padding key when keep[b * len + p] == 0 (keep == nullptr: none).
struct KeyMask {
  const uint8_t* keep;
  int len;
};

// cache_v == nullptr: a single-tensor cache (cache_k holds V of a K=V layer;
// wk_single, the owning layer's key-norm weight, rebuilds K).
cudaError_t launch_decode(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                          const void* cache_k, const void* cache_v, const void* wk_single,
                          const int32_t* len, int cap, int rolling, KeyMask km,
                          const DecodePlan& plan, float* partials, void* out, int* status,
                          cudaStream_t s, cudaEvent_t ev0, cudaEvent_t ev1);

// Tensor-core split kernel of g4attn_decode (bf16, <= 8 query heads per KV
// head, rolling caches with capacity % 16 == 0); writes the same partials
// as the CUDA-core split kernel.
// QKV projection x W^T with the prologue in the epilogue (bf16): q_hat
// [B, T, Hq, d]; K/V of the Hkv key (and value) heads into kv; len[b] =
// p0 + T when len is given.  W holds n_heads * d rows.
cudaError_t launch_qkv_prologue(const LayerCfg& L, int B, int T, int p0, const void* x,
                                int hidden, const void* w_qkv, int n_heads, const void* wq,
                                const void* wk, void* q_hat, KVDst kv, int32_t* len, int* status,
                                cudaStream_t s);

bool decode_mma_supported(const LayerCfg& L, int cap, int rolling);
cudaError_t launch_decode_mma(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                              const void* cache_k, const void* cache_v, const void* wk_single,
                              const int32_t* len, int cap, int rolling, KeyMask km,
                              const DecodePlan& plan, float* part_ml, float* part_o,
                              int* status, cudaStream_t s);

// g4attn_decode with the split-KV partials in the library's fixed device
// array instead of a workspace; returns a g4attn_status code.
int launch_decode_noalloc(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                          const void* cache_k, const void* cache_v, const void* wk_single,
                          const int32_t* len, int cap, int rolling, KeyMask km, void* out,
                          int* status, cudaStream_t s);

// Tensor map of a bf16 tensor with a 128-byte-swizzled box (dims[0]
// contiguous, strides in bytes for dims 1..rank-1); false on failure.
}  // namespace g4
struct CUtensorMap_st;
namespace g4 {
bool make_bf16_map(CUtensorMap_st* m, const void* ptr, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box);

// Device status word of the current device (nullptr if it cannot be found).
int* status_ptr();

// Unique id of the current CUDA context (false if there is none or the
// driver cannot say); caches of device addresses are keyed on it.
bool current_context_id(unsigned long long* id);

// Kernel launches counter (incremented by every launcher).
void count_launch(int n = 1);

}  // namespace g4
