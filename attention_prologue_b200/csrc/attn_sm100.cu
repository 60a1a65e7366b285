// Prefill attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA)
// for head_dim 64 / 128 / 256 (512 lives in attn_pair.cu): the sliding-window
// layers ("Gemma 4" overview blog, "Sliding-window attention"; "Gemma 4" Keras
// docs, "What changed": bidirectional image blocks on sliding layers) and
// causal global layers ("Global attention layers").
//
// A work tile is 128 query rows: gp query heads that share one KV head (GQA)
// x 128/gp consecutive positions, row r = (position r / gp, head r % gp), so
// K/V tiles serve all packed heads and a tile meets fewer masked keys.  Key
// tiles (64 keys) outside the union of the rows' key intervals are skipped.
//
// The kernel is persistent: one CTA per SM walks work tiles round-robin
// (latest rows first), and every ring and barrier runs on counters that
// continue across tiles, so one tile's tail (last softmax tiles, last PV,
// epilogue) overlaps the next tile's Q load and first S products.
//   warp 0      TMA producer of K tiles (all work tiles in sequence)
//   warp 2      TMA producer of V tiles
//   warp 1      owns TMEM; one thread issues S_j = Q K_j^T (M 128, N 64,
//               K = d; A and B K-major in smem), S_j only once PV_{j-NS}
//               is done (a commit tracks its own thread's MMAs)
//   warp 3      one thread issues O += P_j V_j (M 128, N = d, K 64; P from
//               TMEM, V MN-major); the first PV of a tile waits until the
//               epilogue warps have read the previous tile's O
//   warps 4..7  softmax: thread r owns row r (TMEM lane r); reads S_j, masks
//               edge tiles, lazy O rescale, P_j = exp2(S_j - m) as bf16 into
//               TMEM over S_j; hands the row sums to the epilogue warps
//   warps 8..11 Q and epilogue: after the last S of a tile, load the next
//               tile's Q by TMA; then normalise the previous tile's O and
//               write it out (each thread its row) while the next tile runs
// TMEM columns: NS = 4 S buffers of 64, O at 256.
//
// The tensor core's issue queue is short and a tcgen05.mma blocks while it
// is full; two issuing threads keep a ready PV from waiting behind an S.
// The online softmax rescales O lazily: a row keeps the max it exponentiates
// against until a tile raises it by more than 16 (log2 units), so P < 2^16
// (exact in bf16 up to its relative rounding; O and l stay far inside fp32).
// A rescale waits for the previous PV, and the first PV of a tile waits for
// the previous tile's O to be read out, so rescales must stay rare: with a
// threshold of 8 the rows whose first key tile was mostly masked rescaled at
// the second tile and stalled every tile boundary.
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

constexpr int BM = 128;  // query rows per work tile
constexpr int BN = 64;   // keys per key tile
constexpr int kMaxStages = 8;  // K or V ring slots (barrier area)
constexpr int kNS = 4;   // S buffers in TMEM
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kEpiWarp0 = 8;

template <int D>
struct Layout {
  // Q lives in shared memory (TMEM holds NS = 4 S buffers and O: 512
  // columns at d = 256); d = 256 then leaves room for three K stages and two
  // V stages.  Smaller heads take deeper rings: a tile's copy takes a few
  // thousand cycles to land, and with two V slots the PV of key tile j waited
  // for the copy that the PV of tile j - 2 released (the period was half
  // that latency at d = 64).
  static constexpr int kStagesK = D == 256 ? 3 : (D == 128 ? 6 : 8);
  static constexpr int kStagesV = D == 256 ? 2 : (D == 128 ? 6 : 8);
  static_assert(kStagesK <= kMaxStages && kStagesV <= kMaxStages, "ring barriers");
  static constexpr int kChunks = D / 64;                  // 64-element (128-byte) columns
  static constexpr uint32_t kQChunk = BM * 128;           // bytes of one 128-row chunk
  static constexpr uint32_t kKVChunk = BN * 128;          // bytes of one K or V chunk
  static constexpr uint32_t kQ = 0;                       // Q chunks
  static constexpr uint32_t kK = kQ + kChunks * kQChunk;
  static constexpr uint32_t kV = kK + kStagesK * kChunks * kKVChunk;
  static constexpr uint32_t kL = kV + kStagesV * kChunks * kKVChunk;  // row sums [2][128]
  static constexpr uint32_t kBars = kL + 2 * BM * 4;
  static constexpr uint32_t kAlloc = kBars + 512;  // + barriers and scalars
  static_assert(kAlloc <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static constexpr uint32_t kColO = kNS * BN;
  static constexpr uint32_t kTmemCols = (kColO + D) <= 256 ? 256 : 512;
};

struct Bars {  // offsets (in 8-byte words) of the mbarriers from Layout::kBars
  enum {
    q_full = 0,    // Q of the current tile in smem
    q_empty = 1,   // the last S of a tile is done: Q may be replaced
    o_last = 2,    // the last PV of a tile is done
    o_free = 3,    // the epilogue warps have read O out of TMEM (128 arrivals)
    l_ready = 4,   // [2] row sums of tiles k with k % 2 = i written (128 arrivals)
    l_free = 6,    // [2] the epilogue warps have read those row sums (128 arrivals)
    drain = 8,     // (S issuer)
    drain2 = 9,    // (PV issuer)
    k_full = 10,                   // [kStagesK]
    k_empty = k_full + kMaxStages,  // [kStagesK]
    v_full = k_empty + kMaxStages,  // [kStagesV]
    v_empty = v_full + kMaxStages,  // [kStagesV]
    s_full = v_empty + kMaxStages,  // [NS]
    p_full = s_full + kNS,          // [NS]
    o_done = p_full + kNS,  // [NS] PV_j done (one per S buffer: rescale waits stay in one phase)
    count = o_done + kNS
  };
};

struct Scalars {  // after the barriers
  uint32_t tmem_base;
  int abort;
};

// Work tile t: sequence b, first query head h0, first position p0 (row
// tiles latest first) and key-tile range [kt0, kt0 + n), walked from
// kt0 + rot and wrapping around.  Warp-collective: with image blocks the
// range is a min/max over the tile's positions.
struct TileInfo {
  int b, h0, p0, kt0, n, rot;
};

// Key tile of step j of a work tile.
__device__ __forceinline__ int key_tile(const TileInfo& ti, int j) {
  const int jj = j + ti.rot;
  return ti.kt0 + (jj < ti.n ? jj : jj - ti.n);
}

__device__ __forceinline__ TileInfo tile_info(int t, int n_rt, int n_hg, int gp_log2, int T_,
                                              const RowIntervals& rows, int layer_type,
                                              int window) {
  TileInfo ti;
  const int rt = n_rt - 1 - t % n_rt;
  const int rest = t / n_rt;
  ti.h0 = (rest % n_hg) << gp_log2;
  ti.b = rest / n_hg;
  const int bp = BM >> gp_log2;
  ti.p0 = rt * bp;
  const int p1 = min(ti.p0 + bp, T_) - 1;
  int lo, hi;
  if (rows.lo) {
    lo = 0x7fffffff;
    hi = -1;
    for (int i = ti.p0 + (int)(threadIdx.x & 31); i <= p1; i += 32) {
      const int a = rows.lo[(long)ti.b * T_ + i], e = rows.hi[(long)ti.b * T_ + i];
      if (a <= e) {  // a row left without keys (padding) widens nothing
        lo = min(lo, a);
        hi = max(hi, e);
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (hi < lo) lo = hi = 0;  // no row has a key: one key tile, all of it masked
  } else {
    lo = layer_type == 1 ? 0 : max(0, ti.p0 - window + 1);
    hi = p1;
  }
  ti.kt0 = lo / BN;
  ti.n = hi < lo ? 0 : hi / BN - ti.kt0 + 1;
  // The row tiles of one (sequence, head group) run side by side on the SMs
  // (consecutive tiles).  Where they share a key range that starts at the
  // same tile (global and bidirectional layers), each starts its walk at its
  // own offset: otherwise all of them ask for the same K and V tiles at
  // once, and the copies of those tiles were several times slower than
  // those of staggered readers.  Sliding windows are staggered already.
  // The order of the key tiles changes only the rounding of the online
  // softmax.
  ti.rot = layer_type == 0 || ti.n <= 1 ? 0 : (int)(((long)rt * ti.n) / n_rt) % ti.n;
  return ti;
}

}  // namespace

// kExtras: the padding mask and the logit soft-cap are compiled in (the
// plain instantiation carries none of their code in the softmax loop).
template <int D, bool kExtras>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      RowIntervals rows, KeyBits kb, __nv_bfloat16* __restrict__ out, int T_,
                      int Hq, int Hkv, int layer_type, int window, float scale_log2,
                      float cap2, int gp_log2, int n_work, int* status) {
  using Ly = Layout<D>;
  constexpr int kStagesK = Ly::kStagesK;
  constexpr int kStagesV = Ly::kStagesV;
  static_assert(8 * Bars::count + (int)sizeof(Scalars) <= 512, "barrier area");
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
  float* lbuf = reinterpret_cast<float*>(gbase + Ly::kL);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bp = BM >> gp_log2;
  const int n_rt = (T_ + bp - 1) / bp;
  const int n_hg = Hq >> gp_log2;
  const int grp = Hq / Hkv;
  auto tile_of = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
  auto info = [&](int t) {  // warp-collective
    return tile_info(t, n_rt, n_hg, gp_log2, T_, rows, layer_type, window);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(Bars::q_full), 1);
    mbar_init(bar(Bars::q_empty), 1);
    mbar_init(bar(Bars::o_last), 1);
    mbar_init(bar(Bars::o_free), 4 * 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Bars::l_ready + i), 4 * 32);
      mbar_init(bar(Bars::l_free + i), 4 * 32);
    }
    mbar_init(bar(Bars::drain), 1);
    mbar_init(bar(Bars::drain2), 1);
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
    sc->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(base + Ly::kBars + 8 * Bars::count, Ly::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sc->tmem_base;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0 the K tiles, warp 2 the V tiles of all work tiles in sequence;
    // a slot is refilled as soon as its consumer (S_j for K, PV_j for V) is done
    const bool is_k = warp == 0;
    const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
    const uint32_t ring = base + (is_k ? Ly::kK : Ly::kV);
    const int full = is_k ? Bars::k_full : Bars::v_full;
    const int empty = is_k ? Bars::k_empty : Bars::v_empty;
    const int nst = is_k ? kStagesK : kStagesV;
    int g = 0;  // key tiles issued so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int t = tile_of(k);
      if (t >= n_work) break;
      const TileInfo ti = info(t);
      if (lane == 0) {
        const int kv_row = ti.b * Hkv + ti.h0 / grp;
        for (int j = 0; j < ti.n; ++j, ++g) {
          const int s = g % nst;
          if (!mbar_wait(bar(empty + s), ((g / nst) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(full + s), BN * D * 2);
          for (int c = 0; c < Ly::kChunks; ++c)
            tma_load_3d(ring + (s * Ly::kChunks + c) * Ly::kKVChunk, tm, bar(full + s), c * 64,
                        key_tile(ti, j) * BN, kv_row);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0 && *abort) {  // let the copies already issued land before the CTA exits
      for (int j = max(0, g - nst); j < g; ++j)
        mbar_wait(bar(full + j % nst), (j / nst) & 1, nullptr);
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1 issues S, warp 3 issues PV (two threads: a tcgen05.mma blocks
    // while the tensor core's issue queue is full, and a ready PV should not
    // wait behind a whole S).  A commit tracks only its own thread's MMAs:
    // S_g, which overwrites the buffer of P_{g-NS}, waits until PV_{g-NS}
    // has completed.
    int g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int t = tile_of(k);
      if (t >= n_work) break;
      const TileInfo ti = info(t);
      if (lane == 0) {
        if (warp == 1) {
          constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0, 0);
          const uint64_t dq0 = desc_sw128(base + Ly::kQ, 16, 1024);
          const uint64_t dk0 = desc_sw128(base + Ly::kK, 16, 1024);
          ok = mbar_wait(bar(Bars::q_full), k & 1, abort);
          for (int j = 0; ok && j < ti.n; ++j, ++g) {
            const int s = g % kStagesK;
            // the K tile first: it lands well ahead, so the wait that gates
            // the issue is the last one (each wait costs a poll round trip)
            if (!(ok = mbar_wait(bar(Bars::k_full + s), (g / kStagesK) & 1, abort))) break;
            if (g >= kNS && !(ok = mbar_wait(bar(Bars::o_done + (g - kNS) % kNS),
                                             ((g - kNS) / kNS) & 1, abort)))
              break;
            tc_fence_after();
            const uint64_t dk = desc_add(dk0, s * Ly::kChunks * Ly::kKVChunk);
            const uint32_t d = tmem + (g % kNS) * BN;
#pragma unroll
            for (int kc = 0; kc < D / 16; ++kc) {
              const int c = kc >> 2, sub = kc & 3;
              mma_ss(d, desc_add(dq0, c * Ly::kQChunk + sub * 32),
                     desc_add(dk, c * Ly::kKVChunk + sub * 32), idesc_s, kc > 0 ? 1u : 0u);
            }
            mma_commit(bar(Bars::s_full + g % kNS));
            mma_commit(bar(Bars::k_empty + s));
          }
          if (ok) mma_commit(bar(Bars::q_empty));  // this tile's Q may now be replaced
        } else {
          constexpr uint32_t idesc_o = idesc_bf16(BM, D, 0, 1);
          const uint64_t dv0 = desc_sw128(base + Ly::kV, Ly::kKVChunk, 1024);
          for (int j = 0; ok && j < ti.n; ++j, ++g) {
            const int s = g % kStagesV;
            if (!(ok = mbar_wait(bar(Bars::v_full + s), (g / kStagesV) & 1, abort))) break;
            if (!(ok = mbar_wait(bar(Bars::p_full + g % kNS), (g / kNS) & 1, abort))) break;
            // the first PV of a tile overwrites O: the previous tile's O is read out
            if (j == 0 && k > 0 && !(ok = mbar_wait(bar(Bars::o_free), (k - 1) & 1, abort)))
              break;
            tc_fence_after();
            const uint64_t dv = desc_add(dv0, s * Ly::kChunks * Ly::kKVChunk);
            const uint32_t pa = tmem + (g % kNS) * BN;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              // A = P in TMEM: row m in lane m, 16 keys = 8 packed columns per step
              mma_ts(tmem + Ly::kColO, pa + kk * 8, desc_add(dv, kk * 16 * 128), idesc_o,
                     (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar(Bars::v_empty + s));
            mma_commit(bar(Bars::o_done + g % kNS));
          }
          if (ok) mma_commit(bar(Bars::o_last));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0 && *abort) {  // this thread's MMAs complete before TMEM is freed
      const int dr = warp == 1 ? Bars::drain : Bars::drain2;
      mma_commit(bar(dr));
      mbar_wait(bar(dr), 0, nullptr);
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x - kSoftmaxWarp0 * 32;  // row (TMEM lane) of this thread
    const uint32_t lane_off = (uint32_t)((warp - kSoftmaxWarp0) * 32) << 16;
    int g = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int t = tile_of(k);
      if (t >= n_work) break;
      const TileInfo ti = info(t);
      const int i = ti.p0 + (r >> gp_log2);  // position of this row
      int lo = 1, hi = 0;                     // key interval (empty past the prompt)
      if (i < T_) {
        if (rows.lo) {
          lo = rows.lo[(long)ti.b * T_ + i];
          hi = rows.hi[(long)ti.b * T_ + i];
        } else if (layer_type == 1) {
          lo = 0;
          hi = i;
        } else {
          lo = max(0, i - window + 1);
          hi = i;
        }
      }
      float m_used = -INFINITY, l = 0.f;
      // with a soft-cap the scores are capped in log2 units first, then the
      // scale is 1
      const float sl2 = (kExtras && cap2 > 0.f) ? 1.f : scale_log2;
      for (int j = 0; j < ti.n; ++j, ++g) {
        const int sb = g % kNS;
        // the padding bits of this key tile (all kept without a mask), read
        // before the wait so the load overlaps it
        const uint64_t keep =
            (kExtras && kb.bits) ? kb.bits[(long)ti.b * kb.words + key_tile(ti, j)] : ~0ull;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + sb), (g / kNS) & 1, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[BN];
        tmem_ld32(tmem + lane_off + sb * BN, sr);
        tmem_ld32(tmem + lane_off + sb * BN + 32, sr + 32);
        tmem_wait_ld();
        const int key0 = key_tile(ti, j) * BN;
        float x[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) x[c] = __uint_as_float(sr[c]);
        if (kExtras && cap2 > 0.f) {
          const float k = scale_log2 / cap2;
#pragma unroll
          for (int c = 0; c < BN; ++c) x[c] = cap2 * tanh_fast(x[c] * k);
        }
        float mt = -INFINITY;
        if (key0 >= lo && key0 + BN - 1 <= hi && (!kExtras || keep == ~0ull)) {  // no mask
#pragma unroll
          for (int c = 0; c < BN; ++c) mt = fmaxf(mt, x[c]);
        } else {
#pragma unroll
          for (int c = 0; c < BN; ++c) {
            const bool in =
                key0 + c >= lo && key0 + c <= hi && (!kExtras || ((keep >> c) & 1));
            x[c] = in ? x[c] : -INFINITY;
            mt = fmaxf(mt, x[c]);
          }
        }
        mt *= sl2;  // sl2 > 0: the max of the scaled scores
        // lazy rescale: only when the row max grows by more than 2^16
        const bool first = m_used == -INFINITY;
        const bool grow = !first && mt > m_used + 16.f;
        if (__any_sync(0xffffffffu, grow)) {
          // PV of the previous key tile must be done (j >= 1 here); S_g done
          // implies PV_{g-NS} is, so o_done of that buffer is one phase behind
          const int pg = g - 1;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar(Bars::o_done + pg % kNS), (pg / kNS) & 1, abort));
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
        // P = exp2(x - m_used) as packed bf16 pairs over the first 32 columns
        // of this S buffer (the PV MMA reads A from TMEM)
        const float neg_m = m_used == -INFINITY ? 0.f : -m_used;  // no key yet: P = 0
        float rs = 0.f;
        uint32_t pk[BN / 2];
#pragma unroll
        for (int e = 0; e < BN / 2; ++e) {
          const float p0 = ex2_approx(fmaf(x[2 * e], sl2, neg_m));
          const float p1 = ex2_approx(fmaf(x[2 * e + 1], sl2, neg_m));
          __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<uint32_t*>(&bb);
          // the row sum adds the P values the PV product multiplies (bf16),
          // so a row's normalisation matches its weights exactly
          rs += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
        }
        tmem_st32(tmem + lane_off + sb * BN, pk);
        tmem_wait_st();
        l += rs;
        tc_fence_before();
        mbar_arrive(bar(Bars::p_full + sb));
      }
      if (!ok) break;
      // the row sum for the epilogue warps, in buffer k % 2 with its own
      // barrier: a tile of at most NS key tiles needs no PV of its own
      // before its softmax ends, so the softmax can finish tile k while the
      // epilogue has yet to wait for tile k - 1 (one barrier for both would
      // then be two phases ahead of that wait); it cannot finish tile k + 1,
      // whose Q is loaded only after the epilogue of tile k - 1
      // (the epilogue warps have read the row sums of tile k - 2 from this
      // buffer: they arrive on l_free right after reading them)
      if (k >= 2 && !(ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::l_free + (k & 1)),
                                                             ((k - 2) >> 1) & 1, abort))))
        break;
      lbuf[(k & 1) * BM + r] = l;
      mbar_arrive(bar(Bars::l_ready + (k & 1)));
    }
  } else {
    // ------------------------------------------------------------ Q and epilogue
    const int ew = warp - kEpiWarp0;
    const int r = threadIdx.x - kEpiWarp0 * 32;  // row (TMEM lane) of this thread
    const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
    bool ok = true;
    int q_issued = 0;  // tiles whose Q chunks the leader (warp 8, lane 0) has loaded
    TileInfo prev{};
    for (int k = 0; ok; ++k) {
      const int t = tile_of(k);
      const bool has = t < n_work;
      TileInfo ti{};
      if (has) {
        ti = info(t);
        // Q of tile k replaces tile k - 1's once the last S of tile k - 1 is
        // done (all four warps wait: the epilogue of tile k - 1 follows it)
        if (k > 0)
          ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::q_empty), (k - 1) & 1, abort));
        if (!ok) break;
        if (ew == 0 && lane == 0) {
          mbar_arrive_expect_tx(bar(Bars::q_full), Ly::kChunks * BM * 128);
          for (int c = 0; c < Ly::kChunks; ++c)
            tma_load_4d(base + Ly::kQ + c * Ly::kQChunk, &tm_q, bar(Bars::q_full), c * 64,
                        ti.h0, ti.p0, ti.b);
        }
        q_issued = k + 1;
      }
      if (k > 0) {
        // ---- epilogue of tile k - 1: O / l as bf16, each thread its row
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar(Bars::o_last), (k - 1) & 1, abort) &&
                            mbar_wait(bar(Bars::l_ready + ((k - 1) & 1)), ((k - 1) >> 1) & 1, abort));
        if (!ok) break;
        tc_fence_after();
        const float lsum = lbuf[((k - 1) & 1) * BM + r];
        mbar_arrive(bar(Bars::l_free + ((k - 1) & 1)));  // the buffer may take tile k + 1's sums
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        uint32_t ob[D / 2];
#pragma unroll
        for (int c = 0; c < Ly::kChunks; ++c) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + Ly::kColO + 64 * c + 32 * h, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                        __uint_as_float(o[2 * e + 1]) * inv);
              ob[32 * c + 16 * h + e] = *reinterpret_cast<uint32_t*>(&bb);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Bars::o_free));  // the next tile's first PV may overwrite O
        const int i = prev.p0 + (r >> gp_log2);
        if (i < T_) {
          const int hrow = prev.h0 + (r & ((1 << gp_log2) - 1));
          // 32-byte stores: each writes a whole sector (the rows of a warp lie
          // 512 bytes or more apart, so 16-byte stores would half-fill them)
          uint32_t* dst = reinterpret_cast<uint32_t*>(out + (((long)prev.b * T_ + i) * Hq + hrow) * D);
#pragma unroll
          for (int e = 0; e < D / 16; ++e) st_global_v8(dst + 8 * e, ob + 8 * e);
        }
      }
      if (!has) break;
      prev = ti;
    }
    if (ew == 0 && lane == 0 && *abort && q_issued > 0)  // the last Q load lands before exit
      mbar_wait(bar(Bars::q_full), (q_issued - 1) & 1, nullptr);
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
                      RowIntervals rows, KeyBits kb, void* out, int* status, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  const int gp_log2 = gqa_pack_log2(L.Hq, L.Hkv);
  constexpr int DF = D;
  const uint64_t es = 2;
  {  // q_hat [B, T, Hq, D]: dims (D, Hq, T, B)
    const uint64_t dims[4] = {(uint64_t)DF, (uint64_t)L.Hq, (uint64_t)T, (uint64_t)B};
    const uint64_t str[3] = {DF * es, (uint64_t)L.Hq * DF * es, (uint64_t)T * L.Hq * DF * es};
    const uint32_t box[4] = {64, (uint32_t)(1 << gp_log2), (uint32_t)(BM >> gp_log2), 1};
    if (!make_map(&tq, q_hat, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // K, V [B * Hkv, cap, D]; only positions < kv.len exist (rows past it read as 0)
    const uint64_t dims[3] = {(uint64_t)DF, (uint64_t)kv.len, (uint64_t)B * L.Hkv};
    const uint64_t str[2] = {DF * es, (uint64_t)kv.cap * DF * es};
    const uint32_t box[3] = {64, BN, 1};
    if (!make_map(&tk, kv.k, 3, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_map(&tv, kv.v, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  using Ly = Layout<D>;
  const bool extras = kb.bits != nullptr || L.softcap > 0.f;
  auto kern = extras ? attn_sm100_kernel<D, true> : attn_sm100_kernel<D, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
  if (e != cudaSuccess) return e;
  const float scale_log2 = L.scale * 1.4426950408889634f;
  const int bp = BM >> gp_log2;  // positions per tile
  const int n_work = (T + bp - 1) / bp * (L.Hq >> gp_log2) * B;
  if (n_work == 0) return cudaSuccess;
  // persistent: one CTA per SM (the shared memory admits one), at most one per tile
  int dev = 0, n_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_work < n_sm ? n_work : n_sm);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Ly::kAlloc;
  cfg.stream = s;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, rows, kb,
                         static_cast<__nv_bfloat16*>(out), T, L.Hq, L.Hkv, L.layer_type, L.window,
                         scale_log2, softcap_log2(L), gp_log2, n_work, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool attention_sm100_supported(const LayerCfg& L) {
  return L.dtype == 0 && (L.d == 64 || L.d == 128 || L.d == 256 || L.d == 512);
}

cudaError_t launch_attention_sm100(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                   RowIntervals rows, KeyBits kb, void* out, int* status,
                                   cudaStream_t s) {
  switch (L.d) {
    case 64: return run_sm100<64>(L, B, T, q_hat, kv, rows, kb, out, status, s);
    case 128: return run_sm100<128>(L, B, T, q_hat, kv, rows, kb, out, status, s);
    case 256: return run_sm100<256>(L, B, T, q_hat, kv, rows, kb, out, status, s);
    case 512: return launch_attention_pair(L, B, T, q_hat, kv, rows, kb, out, status, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace g4
