// Prefill attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA)
// for head_dim 64 / 128 / 256 (512 lives in attn_pair.cu): the sliding-window layers with image blocks
// ("Gemma 4" overview blog, "Sliding-window attention"; "Gemma 4" Keras docs,
// "What changed": bidirectional image blocks on sliding layers) and causal
// global layers ("Global attention layers").
//
// One CTA computes 128 query rows: gp query heads that share one KV head
// (GQA) x 128/gp consecutive positions, row r = (position r / gp, head
// r % gp), so a tile spans fewer positions and meets fewer masked keys:
//   warps 0, 2  TMA producers: Q tile once and K tiles (warp 0), V tiles
//               (warp 2), 64 keys each, two-stage rings (128-byte swizzle,
//               no multicast); a K slot is refilled as soon as S_j is done,
//               a V slot as soon as PV_j is done
//   warp 1      owns TMEM; one thread issues S_j = Q K_j^T (M 128, N 64,
//               K = d; B K-major in smem, A in smem or TMEM) once PV_{j-NS}
//               is done
//   warp 3      one thread issues O += P_j V_j (M 128, N = d, K 64; P from
//               TMEM, V MN-major in smem)
//   warps 4..7  softmax: thread r owns query row r (TMEM lane r); reads S_j,
//               masks it with the row's key interval [lo, hi], writes
//               P_j = exp2(S_j - m) as bf16 into swizzled shared memory, and
//               at the end normalises O and stores it.
// TMEM columns: NS S buffers of 64 (NS = 4 for d = 256, else 2), O after
// them (at 256, resp. 128; d columns).
// Key tiles outside the union of the 128 rows' intervals are never loaded.
//
// The online softmax rescales O lazily: a row keeps the max it exponentiates
// against until a new tile raises it by more than 8 (in log2 units), so P
// stays below 2^8 and O is read and written back only on those rare tiles.
//
// Every mbarrier wait is bounded (sm100.cuh); on a timeout the CTA records
// G4ATTN_EDEVICE, drains its in-flight copies and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <mutex>

#include "common.cuh"
#include "g4attn.h"
#include "g4attn_internal.h"
#include "sm100.cuh"

namespace g4 {

using namespace sm100;

namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 64;   // keys per tile
constexpr int kStagesV = 2;
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;

template <int D>
struct Layout {
  // d = 256: the first 128 dims of Q live in tensor memory (the QK^T MMA
  // reads that half of A from TMEM), which takes 32 KB of operand reads per
  // tile off shared memory and leaves room for four K stages; they are staged
  // through the V ring at the start.  Three S buffers: S runs up to two tiles
  // ahead of PV.  Smaller heads: Q in shared memory, two S buffers (two CTAs
  // per SM fit the tensor memory).
  static constexpr int kQTmemChunks = D == 256 ? 2 : 0;
  static constexpr bool kQT = kQTmemChunks > 0;
  static constexpr int kStagesK = kQT ? 4 : 3;            // K is needed one S before V
  static constexpr int kChunks = D / 64;                  // 64-element (128-byte) columns
  static constexpr uint32_t kQChunk = BM * 128;           // bytes of one Q chunk
  static constexpr uint32_t kKVChunk = BN * 128;          // bytes of one K or V chunk
  static constexpr uint32_t kQ = 0;                       // Q chunks kQTmemChunks.. in smem
  static constexpr uint32_t kK = kQ + (kChunks - kQTmemChunks) * kQChunk;
  static constexpr uint32_t kV = kK + kStagesK * kChunks * kKVChunk;
  static constexpr uint32_t kBars = kV + kStagesV * kChunks * kKVChunk;
  static constexpr uint32_t kAlloc = kBars + 256;  // + barriers and scalars
  static_assert(kAlloc <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static_assert(kQTmemChunks * kQChunk <= kStagesV * kChunks * kKVChunk,
                "Q staging fits the V ring");
  static constexpr int kNS = kQT ? 3 : 2;
  static constexpr uint32_t kColQ = kNS * BN;             // Q (bf16 pairs) when kQT
  static constexpr uint32_t kColO = kQT ? 256 : kNS * BN;
  static constexpr uint32_t kTmemCols = (kColO + D) <= 256 ? 256 : 512;
  static_assert(!kQT || kColQ + kQTmemChunks * 32 <= kColO, "TMEM columns overlap");
  static_assert(kChunks * kQChunk <= kStagesK * kChunks * kKVChunk, "O staging fits the K ring");
};

// Offsets (in 8-byte words) of the mbarriers from Layout::kBars.
template <int NS>
struct BarsT {
  enum {
    q_full = 0,
    q_tmem = 1,           // Q is in TMEM (the staging area in the V ring is free)
    k_full = 2,           // [4]
    k_empty = 6,          // [4]
    v_full = 10,          // [2]
    v_empty = 12,         // [2]
    drain = 14,           // (S issuer)
    drain2 = 15,          // (PV issuer)
    o_last = 16,          // single phase: the last PV (the epilogue may lag several PVs)
    s_full = 17,          // [NS]
    p_full = s_full + NS,  // [NS]
    o_done = p_full + NS,  // [NS] PV_j done (one per S buffer: rescale waits stay in one phase)
    count = o_done + NS
  };
};

struct Scalars {  // ints after the barriers
  uint32_t tmem_base;
  int abort;
  int klo, khi;
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, RowIntervals rows,
                      __nv_bfloat16* __restrict__ out, int T_, int Hq, int Hkv, int layer_type,
                      int window, float scale_log2, int gp_log2, int* status) {
  using Ly = Layout<D>;
  using Bars = BarsT<Ly::kNS>;
  constexpr int kStagesK = Ly::kStagesK;
  constexpr int kNS = Ly::kNS;
  static_assert(8 * Bars::count + 16 <= 256, "barriers and scalars overflow their area");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128-byte-swizzle atoms assume a 1024-byte aligned base
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) record_status(status, G4ATTN_EDEVICE);
    return;
  }
  const uint32_t base = smem_u32(smem_raw);
  uint8_t* gbase = smem_raw;
  const uint32_t bars = base + Ly::kBars;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  Scalars* sc = reinterpret_cast<Scalars*>(gbase + Ly::kBars + 8 * Bars::count);
  volatile int* abort = &sc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = (int)gridDim.x - 1 - (int)blockIdx.x;  // latest rows first
  const int b = blockIdx.z;
  const int h0 = blockIdx.y << gp_log2;    // first query head of the tile
  const int p0 = tile * (BM >> gp_log2);   // first position of the tile
  const int kvh = h0 / (Hq / Hkv);

  if (threadIdx.x == 0) {
    mbar_init(bar(Bars::q_full), 1);
    mbar_init(bar(Bars::q_tmem), 4 * 32);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(bar(Bars::k_full + s), 1);
      mbar_init(bar(Bars::k_empty + s), 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(bar(Bars::v_full + s), 1);
      mbar_init(bar(Bars::v_empty + s), 1);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(Bars::s_full + s), 1);
      mbar_init(bar(Bars::p_full + s), 4 * 32);
      mbar_init(bar(Bars::o_done + s), 1);
    }
    mbar_init(bar(Bars::drain), 1);
    mbar_init(bar(Bars::drain2), 1);
    mbar_init(bar(Bars::o_last), 1);
    sc->abort = 0;
    sc->klo = 0x7fffffff;
    sc->khi = -1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(base + Ly::kBars + 8 * Bars::count, Ly::kTmemCols);
    tmem_relinquish();
  }
  // row intervals of the softmax threads, reduced to the CTA's key range
  int lo = 1, hi = 0;
  const int r = threadIdx.x - kSoftmaxWarp0 * 32;  // row of a softmax thread
  __syncthreads();
  const int i = p0 + (r >> gp_log2);             // position of a softmax thread's row
  const int hrow = h0 + (r & ((1 << gp_log2) - 1));  // and its query head
  if (warp >= kSoftmaxWarp0) {
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
      atomicMin(&sc->klo, lo);
      atomicMax(&sc->khi, hi);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sc->tmem_base;
  const int kt0 = sc->klo / BN;
  const int n_tiles = sc->khi / BN - kt0 + 1;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0 loads Q and the K tiles, warp 2 the V tiles: each ring is
    // refilled as soon as its own consumer (S_j for K, PV_j for V) is done.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      const uint32_t ring = base + (is_k ? Ly::kK : Ly::kV);
      const int full = is_k ? Bars::k_full : Bars::v_full;
      const int empty = is_k ? Bars::k_empty : Bars::v_empty;
      const int nst = is_k ? kStagesK : kStagesV;
      int n_load = n_tiles;
      if (is_k) {  // Q, into the V ring when it is staged for TMEM
        mbar_arrive_expect_tx(bar(Bars::q_full), BM * D * 2);
        for (int c = 0; c < Ly::kChunks; ++c)
          tma_load_4d(c < Ly::kQTmemChunks ? base + Ly::kV + c * Ly::kQChunk
                                           : base + Ly::kQ + (c - Ly::kQTmemChunks) * Ly::kQChunk,
                      &tm_q, bar(Bars::q_full), c * 64, h0, p0, b);
      } else if (Ly::kQT && !mbar_wait(bar(Bars::q_tmem), 0, abort)) {
        n_load = 0;  // the staged Q is still being read
      }
      int issued = 0;
      for (int j = 0; j < n_load; ++j) {
        const int s = j % nst;
        if (!mbar_wait(bar(empty + s), ((j / nst) & 1) ^ 1, abort)) break;
        const int key0 = (kt0 + j) * BN;
        mbar_arrive_expect_tx(bar(full + s), BN * D * 2);
        for (int c = 0; c < Ly::kChunks; ++c)
          tma_load_3d(ring + (s * Ly::kChunks + c) * Ly::kKVChunk, tm, bar(full + s), c * 64,
                      key0, b * Hkv + kvh);
        issued = j + 1;
      }
      if (*abort) {  // let the copies already issued land before the CTA exits
        if (is_k) mbar_wait(bar(Bars::q_full), 0, nullptr);
        for (int j = max(0, issued - nst); j < issued; ++j)
          mbar_wait(bar(full + j % nst), (j / nst) & 1, nullptr);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads feed the tensor core: warp 1 issues S_j = Q K_j^T, warp 3
    // issues O += P_j V_j.  The tensor core's issue queue is short and a
    // tcgen05.mma blocks while it is full, so with a single issuer a ready PV
    // waited behind the whole next S (~1000 cycles).  A commit tracks only
    // its own thread's MMAs: S_j, which overwrites the buffer P_{j-NS} lives
    // in, waits until PV_{j-NS} has completed (o_done), not just been issued.
    // No progress for 2 s sets the abort flag.
    if (lane == 0) {
      bool ok = mbar_wait(bar(Bars::q_full), 0, abort) &&
                (!Ly::kQT || mbar_wait(bar(Bars::q_tmem), 0, abort));
      if (ok) tc_fence_after();
      if (warp == 1) {
        constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0, 0);
        // descriptors: per-MMA ones are constant offsets from these bases
        const uint64_t dq0 = desc_sw128(base + Ly::kQ, 16, 1024);
        const uint64_t dk0 = desc_sw128(base + Ly::kK, 16, 1024);
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int s = j % kStagesK;
          if (j >= kNS && !(ok = mbar_wait(bar(Bars::o_done + (j - kNS) % kNS),
                                           ((j - kNS) / kNS) & 1, abort)))
            break;
          if (!(ok = mbar_wait(bar(Bars::k_full + s), (j / kStagesK) & 1, abort))) break;
          tc_fence_after();
          const uint64_t dk = desc_add(dk0, s * Ly::kChunks * Ly::kKVChunk);
          const uint32_t d = tmem + (j % kNS) * BN;
#pragma unroll
          for (int kc = 0; kc < D / 16; ++kc) {
            const int c = kc >> 2, sub = kc & 3;
            const uint64_t bd = desc_add(dk, c * Ly::kKVChunk + sub * 32);
            if (c < Ly::kQTmemChunks) {  // A from TMEM: 16 dims = 8 packed columns per step
              mma_ts(d, tmem + Ly::kColQ + kc * 8, bd, idesc_s, kc > 0 ? 1u : 0u);
            } else {
              mma_ss(d, desc_add(dq0, (c - Ly::kQTmemChunks) * Ly::kQChunk + sub * 32), bd,
                     idesc_s, kc > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar(Bars::s_full + j % kNS));
          mma_commit(bar(Bars::k_empty + s));
        }
      } else {
        constexpr uint32_t idesc_o = idesc_bf16(BM, D, 0, 1);
        const uint64_t dv0 = desc_sw128(base + Ly::kV, Ly::kKVChunk, 1024);
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int s = j % kStagesV;
          if (!(ok = mbar_wait(bar(Bars::p_full + j % kNS), (j / kNS) & 1, abort))) break;
          if (!(ok = mbar_wait(bar(Bars::v_full + s), (j / kStagesV) & 1, abort))) break;
          tc_fence_after();
          const uint64_t dv = desc_add(dv0, s * Ly::kChunks * Ly::kKVChunk);
          const uint32_t pa = tmem + (j % kNS) * BN;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // A = P_j in TMEM: row m in lane m, 16 keys = 8 packed columns per step
            mma_ts(tmem + Ly::kColO, pa + kk * 8, desc_add(dv, kk * 16 * 128), idesc_o,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(Bars::v_empty + s));
          mma_commit(bar(Bars::o_done + j % kNS));
        }
        if (ok && n_tiles > 0) mma_commit(bar(Bars::o_last));
      }
      if (*abort) {  // this thread's MMAs complete before TMEM is freed
        const int dr = warp == 1 ? Bars::drain : Bars::drain2;
        mma_commit(bar(dr));
        mbar_wait(bar(dr), 0, nullptr);
      }
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax
    const uint32_t lane_off = (uint32_t)((warp - kSoftmaxWarp0) * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    if constexpr (Ly::kQT) {
      // row r of the staged half of Q (128-byte swizzle) -> TMEM as bf16 pairs
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::q_full), 0, abort));
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < Ly::kQTmemChunks; ++c) {
          const uint4* row = reinterpret_cast<const uint4*>(gbase + Ly::kV + c * Ly::kQChunk + r * 128);
          uint32_t qw[32];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const uint4 v = row[g ^ (r & 7)];
            qw[4 * g] = v.x;
            qw[4 * g + 1] = v.y;
            qw[4 * g + 2] = v.z;
            qw[4 * g + 3] = v.w;
          }
          tmem_st32(tmem + lane_off + Ly::kColQ + 32 * c, qw);
        }
        tmem_wait_st();
        fence_proxy_async_smem();  // the V loads may now overwrite the staging area
        tc_fence_before();
        mbar_arrive(bar(Bars::q_tmem));
      }
    }
    for (int j = 0; ok && j < n_tiles; ++j) {
      const int sb = j % kNS;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + sb), (j / kNS) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[BN];
      tmem_ld32(tmem + lane_off + sb * BN, sr);
      tmem_ld32(tmem + lane_off + sb * BN + 32, sr + 32);
      tmem_wait_ld();
      const int key0 = (kt0 + j) * BN;
      float x[BN];
      float mt = -INFINITY;
      if (key0 >= lo && key0 + BN - 1 <= hi) {  // interior tile: no mask
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] = __uint_as_float(sr[c]);
          mt = fmaxf(mt, x[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] = (key0 + c >= lo && key0 + c <= hi) ? __uint_as_float(sr[c]) : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      }
      mt *= scale_log2;  // scale > 0: the max of the scaled scores
      // lazy rescale: only when the row max grows by more than 2^8
      const bool first = m_used == -INFINITY;
      const bool grow = !first && mt > m_used + 8.f;
      if (__any_sync(0xffffffffu, grow)) {
        // PV_{j-1} must be done; S_j done implies PV_{j-NS} is, so o_done
        // of that buffer is at most one phase behind
        const int pj = j - 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar(Bars::o_done + pj % kNS), (pj / kNS) & 1, abort));
        if (!ok) break;
        tc_fence_after();
        const float alpha = grow ? exp2f(m_used - mt) : 1.f;
        if (grow) {
          l *= alpha;
          m_used = mt;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + Ly::kColO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(tmem + lane_off + Ly::kColO + c0, o);
        }
        tmem_wait_st();
      }
      if (first && mt != -INFINITY) m_used = mt;
      // P = exp2(x - m_used) as packed bf16 pairs, stored over the first 32
      // columns of this tile's S buffer (the PV MMA reads A from TMEM; the
      // next S MMA into this buffer is issued after that PV)
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;  // row with no key yet: P = 0
      float rs = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int e = 0; e < BN / 2; ++e) {
        const float p0 = ex2_approx(fmaf(x[2 * e], scale_log2, neg_m));
        const float p1 = ex2_approx(fmaf(x[2 * e + 1], scale_log2, neg_m));
        rs += p0 + p1;
        __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
        pk[e] = *reinterpret_cast<uint32_t*>(&bb);
      }
      tmem_st32(tmem + lane_off + sb * BN, pk);
      tmem_wait_st();
      l += rs;
      tc_fence_before();
      mbar_arrive(bar(Bars::p_full + sb));
    }
    // ------------------------------------------------------------ epilogue
    if (ok)  // warp-uniform: the tcgen05 loads below are warp-collective
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::o_last), 0, abort));
    // O / l as bf16 into the (now idle) K ring in the 128-byte-swizzled
    // layout of the output tile, then four TMA tile stores: each row of a
    // thread would otherwise go out as 16-byte pieces 512 bytes apart
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < Ly::kChunks; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + Ly::kColO + 64 * c + 32 * h, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                      __uint_as_float(o[2 * e + 1]) * inv);
            pk[16 * h + e] = *reinterpret_cast<uint32_t*>(&bb);
          }
        }
        uint4* row = reinterpret_cast<uint4*>(gbase + Ly::kK + c * Ly::kQChunk + r * 128);
#pragma unroll
        for (int g = 0; g < 8; ++g)
          row[g ^ (r & 7)] = make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
      }
      fence_proxy_async_smem();
    }
    // (ok is uniform over the 128 softmax threads: all rows see the same waits)
    named_sync(1, 4 * 32);
    if (ok && r == 0) {
      for (int c = 0; c < Ly::kChunks; ++c)
        tma_store_4d(&tm_o, base + Ly::kK + c * Ly::kQChunk, c * 64, h0, p0, b);
      bulk_commit();
      bulk_wait_read();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) record_status(status, G4ATTN_EDEVICE);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Ly::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// bf16 tensor map with a 128-byte-swizzled box; dims[0] is the contiguous one.
bool make_bf16_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

namespace {

bool make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  return make_bf16_map(m, ptr, rank, dims, strides_bytes, box);
}

template <int D>
cudaError_t run_sm100(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                      RowIntervals rows, void* out, int* status, cudaStream_t s) {
  CUtensorMap tq, tk, tv, to;
  const int gp_log2 = gqa_pack_log2(L.Hq, L.Hkv);
  constexpr int DF = D;
  const uint64_t es = 2;
  {  // q_hat [B, T, Hq, D]: dims (D, Hq, T, B)
    const uint64_t dims[4] = {(uint64_t)DF, (uint64_t)L.Hq, (uint64_t)T, (uint64_t)B};
    const uint64_t str[3] = {DF * es, (uint64_t)L.Hq * DF * es, (uint64_t)T * L.Hq * DF * es};
    const uint32_t box[4] = {64, (uint32_t)(1 << gp_log2), (uint32_t)(BM >> gp_log2), 1};
    if (!make_map(&tq, q_hat, 4, dims, str, box)) return cudaErrorInvalidValue;
    // out [B, T, Hq, D]: the same geometry (the epilogue stores its tile)
    if (!make_map(&to, out, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // K, V [B * Hkv, cap, D]; only positions < T exist (rows past T read as 0)
    const uint64_t dims[3] = {(uint64_t)DF, (uint64_t)T, (uint64_t)B * L.Hkv};
    const uint64_t str[2] = {DF * es, (uint64_t)kv.cap * DF * es};
    const uint32_t box[3] = {64, BN, 1};
    if (!make_map(&tk, kv.k, 3, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tv, kv.v, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  using Ly = Layout<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
  if (e != cudaSuccess) return e;
  const float scale_log2 = L.scale * 1.4426950408889634f;
  const int bp = BM >> gp_log2;  // positions per tile
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((T + bp - 1) / bp, L.Hq >> gp_log2, B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Ly::kAlloc;
  cfg.stream = s;
  e = cudaLaunchKernelEx(&cfg, attn_sm100_kernel<D>, tq, tk, tv, to, rows,
                         static_cast<__nv_bfloat16*>(out), T, L.Hq, L.Hkv, L.layer_type, L.window,
                         scale_log2, gp_log2, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool attention_sm100_supported(const LayerCfg& L) {
  return L.dtype == 0 && (L.d == 64 || L.d == 128 || L.d == 256 || L.d == 512);
}

cudaError_t launch_attention_sm100(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                   RowIntervals rows, void* out, int* status, cudaStream_t s) {
  switch (L.d) {
    case 64: return run_sm100<64>(L, B, T, q_hat, kv, rows, out, status, s);
    case 128: return run_sm100<128>(L, B, T, q_hat, kv, rows, out, status, s);
    case 256: return run_sm100<256>(L, B, T, q_hat, kv, rows, out, status, s);
    case 512: return launch_attention_pair(L, B, T, q_hat, kv, rows, out, status, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g4
