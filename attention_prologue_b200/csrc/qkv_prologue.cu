// The QKV projection with the layer's prologue in its epilogue: the step in
// front of the attention ("Gemma 4" overview blog, "Shared KV Cache": the key
// and value projections produce what a layer stores; "Gemma 4" Keras docs,
// "What changed from Gemma 3": plain-weight QK-RMSNorm, weightless V-norm,
// zero-pad partial rope, K=V from one projection).
//
//   raw = x W^T                       5th-generation tensor cores, fp32 in TMEM
//   q_hat = RoPE(RMSNorm(raw_q) w_q)  per query head, bf16 to q_hat
//   K = RoPE(RMSNorm(raw_k) w_k), V = RMSNorm(raw_v or raw_k)  into the cache
//
// The raw projections never leave the SM: the fp32 accumulator is normalised,
// weighted and rotated where it lies and only the bf16 results are written.
//
// A work tile is 128 tokens x one output head (N = head_dim), so the thread
// that owns TMEM lane r holds token r's whole head: the mean square over the
// head and the RoPE pairs (k, k + d/2) need no exchange between threads.
// Tiles are taken in groups of up to 32 token tiles per head sweep, so a group
// of x rows and the heads' weight rows both stay in L2 while they are reused.
// The kernel is persistent (one CTA per SM), with two accumulators in TMEM
// up to head_dim 256 so the epilogue of one tile runs under the MMAs of the
// next.
//   warp 0      TMA producer: x (128 x 64) and W (d x 64) per stage
//   warp 1      owns TMEM; one thread issues raw (+)= x W^T, M 128, N <= 256, K 16
//   warps 2..9  epilogue: TMEM lane quarter warp % 4, two warps per quarter;
//               each of the two threads of a row sums the squares of the
//               whole head and rotates, weights and stores half of its pairs
//               (one warp per quarter left the epilogue slower than the MMAs
//               of a tile at the E2B shape: the RoPE factors of 128 pairs a
//               row are a long dependent chain per thread)
// Every wait is bounded; on a timeout the CTA records G4ATTN_EDEVICE, lets
// its copies and MMAs finish, frees TMEM and exits.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "g4attn.h"
#include "g4attn_internal.h"
#include "sm100.cuh"

namespace g4 {

using namespace sm100;

namespace {

constexpr int kQM = 128;  // tokens per tile (TMEM lanes)
constexpr int kQK = 64;   // hidden dims per stage (one 128-byte swizzled row)
constexpr int kQkvThreads = 320;
constexpr int kEpiWarps = 8;  // warps 2 .. 9
constexpr int kMaxGroupM = 32;

template <int D>
struct QkvLayout {
  static constexpr int kAcc = D <= 256 ? 2 : 1;  // accumulators in TMEM
  static constexpr uint32_t kCols = D * kAcc;    // 128, 256, 512, 512
  static constexpr uint32_t kA = kQM * 128;      // x tile of a stage
  static constexpr uint32_t kB = D * 128;        // W tile of a stage
  static constexpr uint32_t kStage = kA + kB;
  static constexpr int kFit = (192 * 1024) / kStage;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;  // 8, 6, 4, 2
  static constexpr uint32_t kBars = kStages * kStage;
  static constexpr uint32_t kW = kBars + 256;          // float w_q [D], w_k [D]
  static constexpr uint32_t kFreq = kW + 2 * D * 4;    // the pairs' frequencies in turns [D / 2]
  static constexpr uint32_t kAlloc = kFreq + (D / 2) * 8;
  static_assert(kAlloc + 1024 <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static_assert(2 * kStages + 5 <= 32, "barriers fit their 256 bytes");
};

struct QkvArgs {
  int M, T, p0, hidden, B;
  int Hq, Hkv, k_eq_v, n_heads;  // output heads of W: Hq query, then Hkv key (then Hkv value)
  int m_tiles, group_m, n_tiles;
  const __nv_bfloat16* wq;
  const __nv_bfloat16* wk;
  __nv_bfloat16* q_hat;
  KVDst kv;  // the cache (k == nullptr: none); v == nullptr: single-tensor
  int32_t* len;
  float eps;
  int* status;
};

// Tile t -> (token tile, head): groups of group_m token tiles, each group
// swept head by head.
__device__ __forceinline__ void qkv_tile(const QkvArgs& a, int t, int* mt, int* head) {
  const int per_group = a.group_m * a.n_heads;
  const int grp = t / per_group, r = t - grp * per_group;
  const int gm = min(a.group_m, a.m_tiles - grp * a.group_m);
  *head = r / gm;
  *mt = grp * a.group_m + (r - *head * gm);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---- CTA pairs (cta_group::2): one MMA spans the two SMs of a cluster --------

// Tile of a CTA pair: 256 tokens (128 in each CTA's shared memory and TMEM)
// x one head; each CTA loads its own 128 x rows and half of the head's W
// rows (the N columns of an M256 MMA are split between the two CTAs), so an
// SM moves 0.0078 bytes per FLOP (d 256) instead of 0.0117.
template <int D>
struct QkvPairLayout {
  static constexpr int kAcc = D <= 256 ? 2 : 1;
  static constexpr uint32_t kCols = D * kAcc;
  static constexpr int kN = D > 256 ? 256 : D;        // N of one MMA
  static constexpr int kChunksN = D / kN;             // MMAs per 16-wide k step
  static constexpr uint32_t kA = kQM * 128;           // this CTA's 128 x rows
  static constexpr uint32_t kBHalf = (kN / 2) * 128;  // this CTA's half of one N chunk
  static constexpr uint32_t kB = kChunksN * kBHalf;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr int kFit = (192 * 1024) / kStage;
  static constexpr int kStages = kFit > 8 ? 8 : kFit;  // 8, 8, 6, 4
  static constexpr uint32_t kBars = kStages * kStage;
  static constexpr uint32_t kW = kBars + 256;
  static constexpr uint32_t kFreq = kW + 2 * D * 4;
  static constexpr uint32_t kAlloc = kFreq + (D / 2) * 8;
  static_assert(kAlloc + 1024 <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static_assert(2 * kStages + 5 <= 32, "barriers fit their 256 bytes");
  static_assert(kBHalf % 1024 == 0, "swizzle atoms of 8 rows");
};

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A B^T over the pair: M 256 (A's rows and D's lanes: 128 in each
// CTA, at the same shared-memory offset / TMEM address), B's N rows split
// between the two CTAs' shared memory at the same offset.
__device__ __forceinline__ void mma_pair_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// One arrival on the mbarrier at `bar_cluster` (a shared::cluster address:
// this CTA's own barrier or the peer's) once the issuing thread's earlier
// pair MMAs are complete.
__device__ __forceinline__ void mma_commit_pair_to(uint32_t bar_cluster) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          bar_cluster)
      : "memory");
}
// ... on the barrier at the same offset in both CTAs of the pair (two commits)
__device__ __forceinline__ void mma_commit_pair_both(uint32_t bar) {
  mma_commit_pair_to(bar);
  mma_commit_pair_to(map_peer(bar, 1));
}
// A tile into this CTA's shared memory whose bytes are counted on an
// mbarrier of the pair's even CTA (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}

}  // namespace

// The epilogue of one tile for the thread that owns token row m (TMEM lane
// address tacc): RMSNorm over the head from the fp32 accumulator, the
// weight and RoPE for query and key heads, bf16 stores of the rotated and /
// or the weightless vectors.  Warp-collective (the TMEM loads).
// half: which half of the rotation pairs (k, k + D/2) this thread takes
// (the two threads of a row each read the whole head for the mean square).
template <int D>
__device__ __forceinline__ void qkv_epilogue_tile(const QkvArgs& a, uint32_t tacc, int m,
                                                  int head, const float* wsm,
                                                  const unsigned long long* fq, int R,
                                                  int half) {
  // pass 1: the head's mean square, from the fp32 accumulator
  float ss = 0.f;
#pragma unroll 1
  for (int c = 0; c < D; c += 32) {
    uint32_t v[32];
    tmem_ld32(tacc + c, v);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), ss);
  }
  const float rs = rsqrtf(ss / (float)D + a.eps);
  const bool row = m < a.M;
  const long b = row ? m / a.T : 0;
  const long pos = a.p0 + (row ? m % a.T : 0);
  const bool is_q = head < a.Hq;
  const bool is_k = !is_q && head < a.Hq + a.Hkv;
  const int kvh = is_q ? 0 : (is_k ? head - a.Hq : head - a.Hq - a.Hkv);
  const float* w = wsm + (is_q ? 0 : D);
  // destinations: the rotated vector (q_hat, or K) and the weightless
  // normalised one (V: a value head, or a key head of a K=V layer)
  uint32_t* rot_dst = nullptr;
  uint32_t* val_dst = nullptr;
  if (row) {
    if (is_q) {
      rot_dst = reinterpret_cast<uint32_t*>(a.q_hat + ((long)m * a.Hq + head) * D);
    } else if (a.kv.k && pos >= a.kv.first) {
      const long slot = a.kv.rolling ? pos % a.kv.cap : pos;
      const long off = ((b * a.Hkv + kvh) * a.kv.cap + slot) * D;
      const bool single = a.kv.v == nullptr;  // a single-tensor cache keeps V alone
      if (is_k && !single)
        rot_dst = reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(a.kv.k) + off);
      if (!is_k || a.k_eq_v)
        val_dst = reinterpret_cast<uint32_t*>(
            static_cast<__nv_bfloat16*>(single ? a.kv.k : a.kv.v) + off);
    }
  }
  const bool rotate = is_q || is_k;  // warp-uniform: one head per tile
  // pass 2: pairs (k, k + D/2), 32 at a time; head_dim 64 has one chunk of
  // 32 pairs, which the first thread of the row takes alone
  constexpr int kPer = D / 2 >= 64 ? D / 4 : D / 2;  // pairs a thread takes
  if (kPer * half >= D / 2) return;
#pragma unroll 1
  for (int c = kPer * half; c < kPer * (half + 1); c += 32) {
    uint32_t lo[32], hi[32];
    tmem_ld32(tacc + c, lo);
    tmem_ld32(tacc + D / 2 + c, hi);
    tmem_wait_ld();
    uint32_t r0[16], r1[16], v0[16], v1[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      float x0[2], x1[2], y0[2], y1[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kp = c + e + u;
        x0[u] = __uint_as_float(lo[e + u]) * rs;  // normalised, no weight
        x1[u] = __uint_as_float(hi[e + u]) * rs;
        y0[u] = x0[u];
        y1[u] = x1[u];
        if (rotate) {
          y0[u] *= w[kp];
          y1[u] *= w[kp + D / 2];
          if (kp < R) {
            float sn, cs;
            rope_sincos_turns((uint32_t)pos, fq[kp], &sn, &cs);
            const float t0 = y0[u] * cs - y1[u] * sn;
            y1[u] = y0[u] * sn + y1[u] * cs;
            y0[u] = t0;
          }
        }
      }
      r0[e / 2] = pack2_bf16(y0[0], y0[1]);
      r1[e / 2] = pack2_bf16(y1[0], y1[1]);
      v0[e / 2] = pack2_bf16(x0[0], x0[1]);
      v1[e / 2] = pack2_bf16(x1[0], x1[1]);
    }
    if (rot_dst) {
      st_global_v8(rot_dst + c / 2, r0);
      st_global_v8(rot_dst + c / 2 + 8, r0 + 8);
      st_global_v8(rot_dst + (D / 2 + c) / 2, r1);
      st_global_v8(rot_dst + (D / 2 + c) / 2 + 8, r1 + 8);
    }
    if (val_dst) {
      st_global_v8(val_dst + c / 2, v0);
      st_global_v8(val_dst + c / 2 + 8, v0 + 8);
      st_global_v8(val_dst + (D / 2 + c) / 2, v1);
      st_global_v8(val_dst + (D / 2 + c) / 2 + 8, v1 + 8);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kQkvThreads, 1)
    qkv_prologue_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w, const QkvArgs a,
                        const __grid_constant__ RopeParams rope) {
  using Ly = QkvLayout<D>;
  constexpr int NS = Ly::kStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  if (smem_u32(smem) & 1023u) {  // the swizzled tiles assume a 1024-byte aligned base
    if (threadIdx.x == 0) record_status(a.status, G4ATTN_EDEVICE);
    return;
  }
  volatile int* abort = &s_abort;
  const uint32_t base = smem_u32(smem), bars = base + Ly::kBars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full = [&](int s) { return bars + 8u * (uint32_t)s; };
  auto empty = [&](int s) { return bars + 8u * (uint32_t)(NS + s); };
  auto acc_full = [&](int i) { return bars + 8u * (uint32_t)(2 * NS + i); };
  auto acc_empty = [&](int i) { return bars + 8u * (uint32_t)(2 * NS + 2 + i); };
  const uint32_t drain = bars + 8u * (uint32_t)(2 * NS + 4);

  float* wsm = reinterpret_cast<float*>(smem + Ly::kW);  // w_q [D], w_k [D]
  unsigned long long* fq = reinterpret_cast<unsigned long long*>(smem + Ly::kFreq);
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    wsm[k] = __bfloat162float(a.wq[k]);
    wsm[D + k] = a.wk ? __bfloat162float(a.wk[k]) : 1.f;
  }
  // the frequencies in shared memory: lane-indexed reads of the parameter
  // space would serialise
  for (int k = threadIdx.x; k < rope.rotated_pairs; k += blockDim.x) fq[k] = rope.turns[k];
  if (blockIdx.x == 0 && a.len)
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) a.len[b] = a.p0 + a.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), Ly::kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_k = (a.hidden + kQK - 1) / kQK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      int g = 0;  // stages issued
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x) {
        int mt, head;
        qkv_tile(a, t, &mt, &head);
        // the k loop starts at a tile-dependent offset: the CTAs that sweep
        // one head (or one token tile) at the same time then read different
        // lines of its W rows (of its x rows); many SMs reading the same
        // lines at once serialise in L2.  The MMA side counts iterations, so
        // only the order of the fp32 accumulation changes.
        const int kb0 = (mt + 5 * head) % n_k;
        for (int i = 0; i < n_k; ++i) {
          const int kb = kb0 + i < n_k ? kb0 + i : kb0 + i - n_k;
          const int s = g % NS;
          if (!(ok = mbar_wait(empty(s), ((g / NS) & 1) ^ 1, abort))) break;
          const uint32_t st = base + s * Ly::kStage;
          mbar_arrive_expect_tx(full(s), Ly::kStage);
          tma_load_2d(st, &tm_x, full(s), kb * kQK, mt * kQM);
#pragma unroll
          for (int h = 0; h < D; h += 256)  // a box holds at most 256 rows
            tma_load_2d(st + Ly::kA + h * 128, &tm_w, full(s), kb * kQK, head * D + h);
          ++g;
        }
      }
      if (*abort)  // the copies already issued land before the CTA exits
        for (int j = max(0, g - NS); j < g; ++j) mbar_wait(full(j % NS), (j / NS) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr int kN = D > 256 ? 256 : D;
      constexpr uint32_t idesc = idesc_bf16(kQM, kN, 0, 0);
      const uint64_t da0 = desc_sw128(base, 16, 1024);
      const uint64_t db0 = desc_sw128(base + Ly::kA, 16, 1024);
      int g = 0, k = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int ai = Ly::kAcc == 2 ? (k & 1) : 0;  // accumulator of this tile
        const int use = Ly::kAcc == 2 ? (k >> 1) : k;
        // the epilogue has read this accumulator's previous tile
        if (use > 0 && !(ok = mbar_wait(acc_empty(ai), (use - 1) & 1, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + ai * D;
        for (int kb = 0; kb < n_k; ++kb) {
          const int s = g % NS;
          if (!(ok = mbar_wait(full(s), (g / NS) & 1, abort))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kQK / 16; ++kk) {
            const uint32_t off = s * Ly::kStage + kk * 32;
#pragma unroll
            for (int h = 0; h < D; h += kN)
              mma_ss(d + h, desc_add(da0, off), desc_add(db0, off + h * 128), idesc,
                     (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty(s));  // the stage is free once these MMAs have read it
          ++g;
        }
        if (ok) mma_commit(acc_full(ai));
      }
      if (*abort) {  // every MMA issued so far completes before TMEM is freed
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;  // TMEM lanes 32 q4 .. 32 q4 + 31
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    int k = 0;
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++k) {
      const int ai = Ly::kAcc == 2 ? (k & 1) : 0;
      const int use = Ly::kAcc == 2 ? (k >> 1) : k;
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full(ai), use & 1, abort))) break;
      tc_fence_after();
      int mt, head;
      qkv_tile(a, t, &mt, &head);
      qkv_epilogue_tile<D>(a, tmem + lane_off + ai * D, mt * kQM + r, head, wsm, fq,
                           rope.rotated_pairs, (warp - 2) >> 2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(ai));  // the accumulator may take a new tile
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) record_status(a.status, G4ATTN_EDEVICE);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Ly::kCols);
  }
}

// The same projection on CTA pairs: a cluster of two CTAs takes 256 tokens
// x one head; the even CTA issues M256 MMAs (cta_group::2) that read each
// CTA's 128 x rows and the two halves of the head's W rows from the two
// CTAs' shared memory and accumulate each CTA's 128 rows in its own TMEM.
// No load or commit uses cluster multicast: each CTA loads its own tiles and
// the even CTA commits once to each CTA's barrier.
//   warp 0      (both) TMA of this CTA's x rows and W half; the bytes of both
//               CTAs are counted on the even CTA's full barrier
//   warp 1      (both) TMEM allocation; (even) the MMA issuer, whose commits
//               arrive on the barriers of both CTAs
//   warps 2..9  (both) epilogue of this CTA's 128 rows; the odd CTA's warps
//               free an accumulator on the even CTA's barrier
template <int D>
__global__ void __launch_bounds__(kQkvThreads, 1)
    qkv_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_w, const QkvArgs a,
                    const __grid_constant__ RopeParams rope) {
  using Ly = QkvPairLayout<D>;
  constexpr int NS = Ly::kStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  // the swizzled tiles assume a 1024-byte aligned base (the same in both
  // CTAs of the pair, so both return here together)
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(a.status, G4ATTN_EDEVICE);
    return;
  }
  volatile int* abort = &s_abort;
  const uint32_t base = smem_u32(smem), bars = base + Ly::kBars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0: the even CTA, which issues the MMAs
  const bool even = rank == 0;
  auto full = [&](int s) { return bars + 8u * (uint32_t)s; };             // even CTA's counts
  auto empty = [&](int s) { return bars + 8u * (uint32_t)(NS + s); };     // each CTA
  auto acc_full = [&](int i) { return bars + 8u * (uint32_t)(2 * NS + i); };       // each CTA
  auto acc_empty = [&](int i) { return bars + 8u * (uint32_t)(2 * NS + 2 + i); };  // even CTA
  const uint32_t drain = bars + 8u * (uint32_t)(2 * NS + 4);
  const int pair = (int)blockIdx.x >> 1, n_pairs = (int)gridDim.x >> 1;

  float* wsm = reinterpret_cast<float*>(smem + Ly::kW);
  unsigned long long* fq = reinterpret_cast<unsigned long long*>(smem + Ly::kFreq);
  for (int k = threadIdx.x; k < D; k += blockDim.x) {
    wsm[k] = __bfloat162float(a.wq[k]);
    wsm[D + k] = a.wk ? __bfloat162float(a.wk[k]) : 1.f;
  }
  for (int k = threadIdx.x; k < rope.rotated_pairs; k += blockDim.x) fq[k] = rope.turns[k];
  if (blockIdx.x == 0 && a.len)
    for (int b = threadIdx.x; b < a.B; b += blockDim.x) a.len[b] = a.p0 + a.T;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 2 * kEpiWarps);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {  // with the peer CTA's warp 1: the same columns in both CTAs
    tmem_alloc_pair(smem_u32(&s_tmem), Ly::kCols);
    tmem_relinquish_pair();
  }
  // barriers initialised and TMEM allocated in both CTAs before any
  // cross-CTA arrival, copy or MMA
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_k = (a.hidden + kQK - 1) / kQK;

  if (warp == 0) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
      int g = 0;  // stages issued
      bool ok = true;
      for (int t = pair; ok && t < a.n_tiles; t += n_pairs) {
        int pt, head;
        qkv_tile(a, t, &pt, &head);
        const int kb0 = (pt + 5 * head) % n_k;  // as in the single-CTA kernel
        for (int i = 0; i < n_k; ++i) {
          const int kb = kb0 + i < n_k ? kb0 + i : kb0 + i - n_k;
          const int s = g % NS;
          // the stage is free once the pair MMAs that read it (in both CTAs) are done
          if (!(ok = mbar_wait_cluster(empty(s), ((g / NS) & 1) ^ 1, abort))) break;
          // the even CTA expects both CTAs' bytes; the odd CTA's may land
          // first (the phase still waits for this arrival)
          if (even) mbar_arrive_expect_tx(full(s), 2 * Ly::kStage);
          const uint32_t fb = map_peer(full(s), 0);
          const uint32_t st = base + s * Ly::kStage;
          tma_load_2d_pair(st, &tm_x, fb, kb * kQK, pt * (2 * kQM) + (int)rank * kQM);
#pragma unroll
          for (int h = 0; h < Ly::kChunksN; ++h)
            tma_load_2d_pair(st + Ly::kA + h * Ly::kBHalf, &tm_w, fb, kb * kQK,
                             head * D + h * Ly::kN + (int)rank * (Ly::kN / 2));
          ++g;
        }
      }
      // the odd CTA's copies count on the even CTA's barriers, which that
      // CTA waits for; the even CTA lets its own issued copies land
      if (*abort && even)
        for (int j = max(0, g - NS); j < g; ++j)
          mbar_wait_cluster(full(j % NS), (j / NS) & 1, nullptr, 200000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && even) {
      constexpr uint32_t idesc = idesc_bf16(2 * kQM, Ly::kN, 0, 0);
      const uint64_t da0 = desc_sw128(base, 16, 1024);
      const uint64_t db0 = desc_sw128(base + Ly::kA, 16, 1024);
      int g = 0, k = 0;
      bool ok = true;
      for (int t = pair; ok && t < a.n_tiles; t += n_pairs, ++k) {
        const int ai = Ly::kAcc == 2 ? (k & 1) : 0;
        const int use = Ly::kAcc == 2 ? (k >> 1) : k;
        // both CTAs' epilogues have read this accumulator's previous tile
        if (use > 0 && !(ok = mbar_wait_cluster(acc_empty(ai), (use - 1) & 1, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + ai * D;
        for (int i = 0; i < n_k; ++i) {
          const int s = g % NS;
          if (!(ok = mbar_wait_cluster(full(s), (g / NS) & 1, abort))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kQK / 16; ++kk) {
            const uint32_t off = s * Ly::kStage + kk * 32;
#pragma unroll
            for (int h = 0; h < Ly::kChunksN; ++h)
              mma_pair_ss(d + h * Ly::kN, desc_add(da0, off),
                          desc_add(db0, off + h * Ly::kBHalf), idesc,
                          (i > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair_both(empty(s));  // frees the stage in both CTAs
          ++g;
        }
        if (ok) mma_commit_pair_both(acc_full(ai));
      }
      if (*abort) {  // every pair MMA issued so far completes before TMEM is freed
        mma_commit_pair_to(drain);
        mbar_wait(drain, 0, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t ae = map_peer(acc_empty(0), 0);  // the even CTA's acc_empty[0]
    int k = 0;
    for (int t = pair; t < a.n_tiles; t += n_pairs, ++k) {
      const int ai = Ly::kAcc == 2 ? (k & 1) : 0;
      const int use = Ly::kAcc == 2 ? (k >> 1) : k;
      if (!__all_sync(0xffffffffu, mbar_wait_cluster(acc_full(ai), use & 1, abort))) break;
      tc_fence_after();
      int pt, head;
      qkv_tile(a, t, &pt, &head);
      qkv_epilogue_tile<D>(a, tmem + lane_off + ai * D, pt * (2 * kQM) + (int)rank * kQM + r,
                           head, wsm, fq, rope.rotated_pairs, (warp - 2) >> 2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(ae + 8u * (uint32_t)ai);
    }
  }

  // both CTAs are done with every copy, MMA and arrival before either frees
  // TMEM or exits
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (threadIdx.x == 0 && *abort) record_status(a.status, G4ATTN_EDEVICE);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Ly::kCols);
  }
}

template <int D>
static cudaError_t run_qkv(const LayerCfg& L, int B, int T, int p0, const void* x, int hidden,
                           const void* w_qkv, int n_heads, const void* wq, const void* wk,
                           void* q_hat, KVDst kv, int32_t* len, int* status, cudaStream_t s) {
  const long M = (long)B * T;
  // CTA pairs (256-token tiles) unless one 128-token tile covers the call
  const bool pairs = M > kQM;
  const int tile_m = pairs ? 2 * kQM : kQM;
  CUtensorMap tx, tw;
  {
    const uint64_t dims[2] = {(uint64_t)hidden, (uint64_t)M};
    const uint64_t str[1] = {(uint64_t)hidden * 2};
    const uint32_t box[2] = {kQK, kQM};
    if (!make_bf16_map(&tx, x, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)hidden, (uint64_t)n_heads * D};
    const uint32_t rows = (uint32_t)std::min(D, 256) / (pairs ? 2 : 1);  // W rows a CTA loads
    const uint64_t str[1] = {(uint64_t)hidden * 2};
    const uint32_t box[2] = {kQK, rows};
    if (!make_bf16_map(&tw, w_qkv, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  QkvArgs a{};
  a.M = (int)M;
  a.T = T;
  a.p0 = p0;
  a.hidden = hidden;
  a.B = B;
  a.Hq = L.Hq;
  a.Hkv = L.Hkv;
  a.k_eq_v = L.k_eq_v;
  a.n_heads = n_heads;
  a.m_tiles = (int)((M + tile_m - 1) / tile_m);
  a.group_m = std::min(a.m_tiles, pairs ? kMaxGroupM / 2 : kMaxGroupM);
  a.n_tiles = a.m_tiles * n_heads;
  a.wq = static_cast<const __nv_bfloat16*>(wq);
  a.wk = static_cast<const __nv_bfloat16*>(wk);
  a.q_hat = static_cast<__nv_bfloat16*>(q_hat);
  a.kv = kv;
  a.len = len;
  a.eps = L.eps;
  a.status = status;
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (!pairs) {
    using Ly = QkvLayout<D>;
    e = cudaFuncSetAttribute(qkv_prologue_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
    if (e != cudaSuccess) return e;
    const int grid = std::min(a.n_tiles, n_sm);
    qkv_prologue_kernel<D><<<grid, kQkvThreads, Ly::kAlloc, s>>>(tx, tw, a, L.rope);
  } else {
    using Ly = QkvPairLayout<D>;
    e = cudaFuncSetAttribute(qkv_pair_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Ly::kAlloc);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * std::min(a.n_tiles, n_sm / 2));
    cfg.blockDim = dim3(kQkvThreads);
    cfg.dynamicSmemBytes = Ly::kAlloc;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, qkv_pair_kernel<D>, tx, tw, a, L.rope);
    if (e != cudaSuccess) return e;
  }
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_qkv_prologue(const LayerCfg& L, int B, int T, int p0, const void* x,
                                int hidden, const void* w_qkv, int n_heads, const void* wq,
                                const void* wk, void* q_hat, KVDst kv, int32_t* len, int* status,
                                cudaStream_t s) {
  switch (L.d) {
    case 64: return run_qkv<64>(L, B, T, p0, x, hidden, w_qkv, n_heads, wq, wk, q_hat, kv, len,
                                status, s);
    case 128: return run_qkv<128>(L, B, T, p0, x, hidden, w_qkv, n_heads, wq, wk, q_hat, kv, len,
                                  status, s);
    case 256: return run_qkv<256>(L, B, T, p0, x, hidden, w_qkv, n_heads, wq, wk, q_hat, kv, len,
                                  status, s);
    case 512: return run_qkv<512>(L, B, T, p0, x, hidden, w_qkv, n_heads, wq, wk, q_hat, kv, len,
                                  status, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g4
