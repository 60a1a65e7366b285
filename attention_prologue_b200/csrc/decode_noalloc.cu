// Allocation-free decode: the split-KV partials of g4attn_decode_noalloc live
// in a fixed array compiled into the library instead of a caller-supplied
// workspace.  Some callers cannot hand the library device memory per call:
// a serving runtime that has already given all free device memory to its
// KV-cache pool, or a plugin host that exposes no allocator.  This variant
// needs nothing beyond its inputs and outputs.
//
// The array is kDecodeScratchBytes (16 MiB) of device memory on every GPU
// that loads the library, held until the process exits.  All calls on a
// device share it and it keeps whatever the last call left there; every
// split CTA writes its partials before the combine reads them (a CTA that
// gives up on a bounded wait writes an empty partial, which the combine
// ignores), so nothing has to start at zero.  Calls whose kernels overlap on
// the GPU (two streams, or two host threads) race on the array and must be
// serialised by the caller.
#include <mutex>

#include "g4attn.h"
#include "g4attn_internal.h"

namespace g4 {

constexpr size_t kDecodeScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

// Device address of g_decode_scratch on the current device.  The host-side
// name of the array is only a stand-in, so the address is looked up once per
// device (with that device current) and cached, keyed on the id of the
// device's current context: after the context is destroyed and re-created
// (cudaDeviceReset) the array lives elsewhere and is looked up again.
// nullptr if the lookup fails.
static float* decode_scratch_ptr() {
  static std::mutex mu;
  static unsigned long long ids[64] = {0};
  static void* ptrs[64] = {nullptr};
  int dev = 0;
  unsigned long long id = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!current_context_id(&id)) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev] || ids[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
    ptrs[dev] = p;
    ids[dev] = id;
  }
  return static_cast<float*>(ptrs[dev]);
}

int launch_decode_noalloc(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                          const void* cache_k, const void* cache_v, const void* wk_single,
                          const int32_t* len, int cap, int rolling, KeyMask km, void* out,
                          int* status, cudaStream_t s) {
  DecodePlan plan = decode_plan(L, cap);
  const size_t per_chunk = decode_partials_bytes(L, B, DecodePlan{plan.chunk, 1});
  const size_t max_chunks = kDecodeScratchBytes / per_chunk;
  if (max_chunks == 0) return G4ATTN_EWORKSPACE;  // one chunk's partials exceed the array
  if ((size_t)plan.n_chunks > max_chunks) {
    // fewer, longer chunks (still multiples of 16) covering at least the same span
    const long span = (long)plan.chunk * plan.n_chunks;
    plan.n_chunks = (int)max_chunks;
    plan.chunk = (int)(((span + plan.n_chunks - 1) / plan.n_chunks + 15) & ~15L);
  }
  float* scratch = decode_scratch_ptr();
  if (!scratch) return G4ATTN_ECUDA;
  cudaError_t e = launch_decode(L, B, q_raw, wq, cache_k, cache_v, wk_single, len, cap, rolling,
                                km, plan, scratch, out, status, s, nullptr, nullptr);
  return e == cudaSuccess ? G4ATTN_OK : G4ATTN_ECUDA;
}

}  // namespace g4
