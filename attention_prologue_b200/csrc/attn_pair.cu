// Prefill attention for head_dim 512: the global layers of the larger
// variants ("Gemma 4" overview blog, "Global attention layers": a global
// head dim of 512 with few KV heads, K = V on the 31B-class models), causal,
// on the 5th-generation tensor cores.
//
// A 128-row fp32 output accumulator of 512 columns fills the whole tensor
// memory of an SM, leaving no room for the scores.  So a cluster of two CTAs
// shares 128 query rows and splits the head dims: CTA r holds dims
// [256 r, 256 r + 256) of Q, K, V and O (256 accumulator columns each).  The
// QK^T MMA of each CTA then yields only a partial score over its half of the
// dims, and the two partials of every 64-key tile are swapped through
// distributed shared memory (DSMEM).
//
// DSMEM moves ~21 GB/s per direction and SM (about 0.8 us per 16 KB), so
// the swap is the cost to minimise and to hide:
//  - each partial goes as a 16-bit integer, already in log2 units (times
//    scale * log2 e), with one fp32 step per row and tile: q = round(y /
//    step), step = max |y| / 32766 over the row's 64 keys -- 16 KB + 512 B
//    per tile and direction.  A CTA adds the peer's decoded partial to its
//    own fp32 one, so the logits of the two CTAs differ by at most step / 2
//    (~1e-3 log2 units at softmax scale 1, ~1e-4 at 1/sqrt(d): at scale 1 an
//    fp16 partial was 20x coarser and moved outputs by ~0.02).  Each CTA
//    normalises its half of O with its own row sums, so each half is exactly
//    consistent with its P.  Encoding and decoding use FMA and byte-permute
//    instructions, no conversions: the transcendental/conversion pipe (16
//    per clock per SM) already carries exp2 and the bf16 packing of P.
//  - sender warps read and send each partial as soon as its MMA is done,
//    while the softmax warps work on earlier tiles; the inbox has two slots.
//  - the sends are st.async: the bytes complete the receiver's mbarrier, no
//    fence.  The rows of warp w travel on their own channel (an mbarrier per
//    inbox slot and warp, 4 KB per tile), and softmax warp w acknowledges
//    its slot straight back to sender warp w of the peer.
//  - the first 128 of the CTA's 256 Q dims live in tensor memory (the QK^T
//    MMA reads them as a TMEM A operand), the other 128 in shared memory;
//    the room saved holds a third K stage: K and V tiles take ~2-3 us to
//    arrive from L2 under this load, so the rings bound the rate.
//
//   warps 0, 2   TMA producers: Q once + K tiles (warp 0), V tiles (warp 2);
//                64 keys x 256 dims, 3 K and 2 V stages, no multicast
//   warp 1       owns TMEM; one thread issues the MMAs, whichever is ready:
//                  S_j  = Q K_j^T   (M 128, N 64, K 256; A half TMEM, half smem)
//                  O   += P_j V_j   (M 128, N 256, K 64; P from TMEM)
//                with S up to two tiles ahead of PV (three S buffers)
//   warps 8..11  senders: own partial of S_j -> int16 + step -> the peer's inbox
//   warps 4..7   softmax (lazy rescale when a row max grows by more than
//                2^16): copy the TMEM half of Q in at the start; then per
//                tile the own partial of S_j + the peer's,
//                mask, lazy O rescale, P_j as bf16 into TMEM over S_j; at the
//                end normalise and store O
// TMEM columns: S buffers at 0, 64 and 128, Q (dims 0..127, bf16 pairs) at
// 192, O at 256.
//
// Every wait is bounded (sm100.cuh); on a timeout the CTA records
// G4ATTN_EDEVICE, drains its copies and MMAs, frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "g4attn.h"
#include "g4attn_internal.h"
#include "sm100.cuh"

namespace g4 {

using namespace sm100;

namespace {

constexpr int BM = 128;       // query rows per cluster
constexpr int BN = 64;        // keys per tile
constexpr int DH = 256;       // head dims per CTA
constexpr int kNS = 3;        // S buffers in TMEM
constexpr int kStagesK = 3;
constexpr int kStagesV = 2;
constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kSenderWarp0 = 8;
constexpr int kChunks = DH / 64;                 // 64-element (128-byte) columns
constexpr int kQTmemChunks = 2;                  // Q chunks kept in TMEM (dims 0..127)
constexpr int kSlots = 2;                        // inbox slots
constexpr uint32_t kQChunk = BM * 128;
constexpr uint32_t kKVChunk = BN * 128;
constexpr uint32_t kQ = 0;                       // Q chunks 2, 3 (dims 128..255)
constexpr uint32_t kK = kQ + (kChunks - kQTmemChunks) * kQChunk;
constexpr uint32_t kV = kK + kStagesK * kChunks * kKVChunk;  // also stages Q chunks 0, 1
constexpr uint32_t kX = kV + kStagesV * kChunks * kKVChunk;  // inbox: the peer's partials
constexpr uint32_t kXSlot = BM * BN * 2;                     // one tile of int16 partials
constexpr uint32_t kXS = kX + kSlots * kXSlot;               // inbox: the fp32 step of each row
constexpr uint32_t kXWarp = kXSlot / 4 + 32 * 4;             // bytes of the 32 rows of one warp
constexpr uint32_t kBars = kXS + kSlots * BM * 4;
static_assert(kQTmemChunks * kQChunk <= kStagesV * kChunks * kKVChunk, "Q staging fits the V ring");
constexpr uint32_t kAlloc = kBars + 512;
static_assert(kAlloc <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = kNS * BN;  // 192
constexpr uint32_t kColO = 256;
static_assert(kColQ + kQTmemChunks * 32 <= kColO, "TMEM columns overlap");

struct Bars {  // 8-byte words from kBars
  enum {
    q_full = 0,
    q_tmem = 1,                 // the TMEM half of Q is in place (staging area free)
    k_full = 2,                 // [3]
    k_empty = 5,                // [3]
    v_full = 8,                 // [2]
    v_empty = 10,               // [2]
    rx_full = 12,               // [kSlots][4 warps] the peer's partials of a warp's rows (tx bytes)
    tx_ok = rx_full + 4 * kSlots,  // [kSlots][4] the peer has consumed a warp's rows of a slot
    drain = tx_ok + 4 * kSlots,
    o_last = drain + 1,         // single phase: the last PV
    s_full = o_last + 1,        // [kNS] partial S_j in TMEM
    p_full = s_full + kNS,      // [kNS] P_j in TMEM
    o_done = p_full + kNS,      // [kNS] PV_j done (one per S buffer: rescale waits stay in one phase)
    s_read = o_done + kNS,      // [kNS] the senders have read S_j (P_j may overwrite it)
    count = s_read + kNS
  };
};
static_assert(8 * Bars::count + 16 <= kAlloc - kBars, "barriers and scalars overflow their area");

struct Scalars {
  uint32_t tmem_base;
  int abort;
  int klo, khi;
};

// 64 fp32 partial scores -> log2 units y -> 32 packed pairs of 16-bit
// integers q = round(y / step); returns step = max |y| / 32766.  The
// rounding adds 1.5 * 2^23 in one FMA: the sum lies in [2^23, 2^24), where
// the float's unit is 1, so its low 16 bits are q in two's complement.
// (|y / step| <= 32766 (1 + 2^-22) also with the approximate reciprocal.)
__device__ __forceinline__ float pack_partial(const uint32_t* sr, float scale_log2, uint32_t* h) {
  float y[BN];
  float amax = 1e-30f;
#pragma unroll
  for (int c = 0; c < BN; ++c) {
    y[c] = __uint_as_float(sr[c]) * scale_log2;
    amax = fmaxf(amax, fabsf(y[c]));
  }
  const float inv = 32766.f * rcp_approx(amax);
#pragma unroll
  for (int e = 0; e < BN / 2; ++e) {
    const float f0 = fmaf(y[2 * e], inv, 12582912.f);
    const float f1 = fmaf(y[2 * e + 1], inv, 12582912.f);
    h[e] = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x5410);
  }
  return amax * (1.f / 32766.f);
}

}  // namespace

// kExtras: the padding mask and the logit soft-cap are compiled in.
template <bool kExtras>
__global__ void __launch_bounds__(kThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, RowIntervals rows, KeyBits kb,
                     __nv_bfloat16* __restrict__ out, int T_, int Hq, int Hkv, int layer_type,
                     int window, float scale_log2, float cap2, int gp_log2, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // the 128-byte-swizzle atoms need a 1024-byte base
    if (threadIdx.x == 0) record_status(status, G4ATTN_EDEVICE);
    return;
  }
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t bars = base + kBars;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  Scalars* sc = reinterpret_cast<Scalars*>(smem_raw + kBars + 8 * Bars::count);
  volatile int* abort = &sc->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
  const int dcol0 = (int)rank * DH;
  const int tile = (int)(gridDim.x >> 1) - 1 - (int)(blockIdx.x >> 1);  // latest rows first
  const int b = blockIdx.z;
  const int h0 = blockIdx.y << gp_log2;
  const int p0 = tile * (BM >> gp_log2);
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
    for (int c = 0; c < 4 * kSlots; ++c) {  // channel (slot, warp) = (c >> 2, c & 3)
      mbar_init(bar(Bars::rx_full + c), 1);
      mbar_init(bar(Bars::tx_ok + c), 1);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(bar(Bars::s_full + s), 1);
      mbar_init(bar(Bars::p_full + s), 4 * 32);
      mbar_init(bar(Bars::o_done + s), 1);
      mbar_init(bar(Bars::s_read + s), 4 * 32);
    }
    mbar_init(bar(Bars::drain), 1);
    mbar_init(bar(Bars::o_last), 1);
    // every channel expects its first tile before the peer can send it
    for (int c = 0; c < 4 * kSlots; ++c) mbar_arrive_expect_tx(bar(Bars::rx_full + c), kXWarp);
    sc->abort = 0;
    sc->klo = 0x7fffffff;
    sc->khi = -1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(base + kBars + 8 * Bars::count, kTmemCols);
    tmem_relinquish();
  }
  int lo = 1, hi = 0;
  const int r = threadIdx.x & 127;  // row (TMEM lane) of a softmax or sender thread
  __syncthreads();
  const int i = p0 + (r >> gp_log2);
  const int hrow = h0 + (r & ((1 << gp_log2) - 1));
  if (warp >= kSoftmaxWarp0 && warp < kSenderWarp0 && i < T_) {
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
    if (lo <= hi) {  // a row left without keys (padding) widens nothing
      atomicMin(&sc->klo, lo);
      atomicMax(&sc->khi, hi);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers exist before any remote access
  const uint32_t tmem = sc->tmem_base;
  // same in both CTAs (same rows); no row with a key: one key tile, all masked
  const bool none = sc->khi < sc->klo;
  const int kt0 = none ? 0 : sc->klo / BN;
  const int n_tiles = none ? 1 : sc->khi / BN - kt0 + 1;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      const uint32_t ring = base + (is_k ? kK : kV);
      const int full = is_k ? Bars::k_full : Bars::v_full;
      const int empty = is_k ? Bars::k_empty : Bars::v_empty;
      const int nst = is_k ? kStagesK : kStagesV;
      int n_load = n_tiles;
      if (is_k) {  // Q chunks 0, 1 into the V ring (staging), 2, 3 to their place
        mbar_arrive_expect_tx(bar(Bars::q_full), BM * DH * 2);
        for (int c = 0; c < kChunks; ++c)
          tma_load_4d(c < kQTmemChunks ? base + kV + c * kQChunk
                                       : base + kQ + (c - kQTmemChunks) * kQChunk,
                      &tm_q, bar(Bars::q_full), dcol0 + c * 64, h0, p0, b);
      } else if (!mbar_wait(bar(Bars::q_tmem), 0, abort)) {  // staging area still in use
        n_load = 0;
      }
      int issued = 0;
      for (int j = 0; j < n_load; ++j) {
        const int s = j % nst;
        if (!mbar_wait(bar(empty + s), ((j / nst) & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(bar(full + s), BN * DH * 2);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(ring + (s * kChunks + c) * kKVChunk, tm, bar(full + s), dcol0 + c * 64,
                      (kt0 + j) * BN, b * Hkv + kvh);
        issued = j + 1;
      }
      if (*abort) {  // let the copies already issued land before the CTA exits
        if (is_k) mbar_wait(bar(Bars::q_full), 0, nullptr);
        for (int j = max(0, issued - nst); j < issued; ++j)
          mbar_wait(bar(full + j % nst), (j / nst) & 1, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BM, BN, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16(BM, DH, 0, 1);
      // descriptors: per-MMA ones are constant offsets from these bases
      const uint64_t dq0 = desc_sw128(base + kQ, 16, 1024);
      const uint64_t dk0 = desc_sw128(base + kK, 16, 1024);
      const uint64_t dv0 = desc_sw128(base + kV, kKVChunk, 1024);
      auto issue_s = [&](int j) {
        const int s = j % kStagesK;
        const uint64_t dk = desc_add(dk0, s * kChunks * kKVChunk);
        const uint32_t d = tmem + (j % kNS) * BN;
#pragma unroll
        for (int kc = 0; kc < DH / 16; ++kc) {
          const int c = kc >> 2, sub = kc & 3;
          const uint64_t bd = desc_add(dk, c * kKVChunk + sub * 32);
          if (c < kQTmemChunks) {  // A from TMEM: 16 dims = 8 packed columns per step
            mma_ts(d, tmem + kColQ + kc * 8, bd, idesc_s, kc > 0 ? 1u : 0u);
          } else {
            mma_ss(d, desc_add(dq0, (c - kQTmemChunks) * kQChunk + sub * 32), bd, idesc_s, 1u);
          }
        }
        mma_commit(bar(Bars::s_full + j % kNS));
        mma_commit(bar(Bars::k_empty + s));
      };
      auto issue_pv = [&](int j) {
        const int s = j % kStagesV;
        const uint64_t dv = desc_add(dv0, s * kChunks * kKVChunk);
        const uint32_t pa = tmem + (j % kNS) * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // A = P_j in TMEM: row m in lane m, 16 keys = 8 packed columns per step
          mma_ts(tmem + kColO, pa + kk * 8, desc_add(dv, kk * 16 * 128), idesc_o,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(Bars::v_empty + s));
        mma_commit(bar(Bars::o_done + j % kNS));
      };
      // Issue whichever MMA is ready, S in order and PV in order: S_j may go
      // once its K tile is in and PV_{j-kNS} (which reads P_{j-kNS} from the
      // buffer S_j overwrites) has been issued before it (tensor-core order);
      // PV_j once P_j and its V tile are in.  (Here the exchange, not the
      // issue, bounds the rate: one issuer suffices.)  No progress for 2 s
      // sets the abort flag.
      bool ok = mbar_wait(bar(Bars::q_full), 0, abort) && mbar_wait(bar(Bars::q_tmem), 0, abort);
      if (ok) tc_fence_after();
      int ns = 0, np = 0;
      uint64_t t_idle = 0;
      for (uint32_t spin = 0; ok && np < n_tiles;) {
        bool did = false;
        if (np < ns && mbar_test(bar(Bars::p_full + np % kNS), (np / kNS) & 1) &&
            mbar_test(bar(Bars::v_full + np % kStagesV), (np / kStagesV) & 1)) {
          tc_fence_after();
          issue_pv(np++);
          did = true;
        }
        if (ns < n_tiles && ns < np + kNS &&
            mbar_test(bar(Bars::k_full + ns % kStagesK), (ns / kStagesK) & 1)) {
          tc_fence_after();
          issue_s(ns++);
          did = true;
        }
        if (did) {
          spin = 0;  // (the timer is read only while idle: it is slow)
        } else if (spin++ == 0) {
          t_idle = globaltimer_ns();
        } else if ((spin & 63) == 0) {
          if (*abort) ok = false;
          else if (globaltimer_ns() - t_idle > 2000000000ull) {
            *abort = 1;
            ok = false;
          }
        }
      }
      if (ok && n_tiles > 0) mma_commit(bar(Bars::o_last));
      if (*abort) {  // every MMA issued so far completes before TMEM is freed
        mma_commit(bar(Bars::drain));
        mbar_wait(bar(Bars::drain), 0, nullptr);
      }
    }
  } else if (warp >= kSenderWarp0) {
    // ------------------------------------------------------------ senders
    const uint32_t lane_off = (uint32_t)((warp - kSenderWarp0) * 32) << 16;
    const int w = warp - kSenderWarp0;
    const uint32_t peer_rx = map_peer(bar(Bars::rx_full + w), peer);
    const uint32_t inbox_row = base + kX + r * (BN * 2);  // 16-byte slot q at q ^ (r & 7)
    for (int j = 0; j < n_tiles; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + j % kNS), (j / kNS) & 1, abort)))
        break;
      tc_fence_after();
      uint32_t h[BN / 2];
      float step;
      {
        uint32_t sr[BN];
        tmem_ld32(tmem + lane_off + (j % kNS) * BN, sr);
        tmem_ld32(tmem + lane_off + (j % kNS) * BN + 32, sr + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(Bars::s_read + j % kNS));
        step = pack_partial(sr, scale_log2, h);
      }
      // the peer has consumed this warp's rows of tile j - kSlots from the slot
      const int sl = j % kSlots;
      if (j >= kSlots &&
          !__all_sync(0xffffffffu, mbar_wait(bar(Bars::tx_ok + 4 * sl + w),
                                             ((j - kSlots) / kSlots) & 1, abort)))
        break;
      const uint32_t slot = inbox_row + (uint32_t)sl * kXSlot;
      const uint32_t rbar = peer_rx + 32u * (uint32_t)sl;
#pragma unroll
      for (int q = 0; q < BN / 8; ++q)
        st_async_v4(map_peer(slot + ((q ^ (r & 7)) << 4), peer), rbar, h[4 * q], h[4 * q + 1],
                    h[4 * q + 2], h[4 * q + 3]);
      st_async_b32(map_peer(base + kXS + ((uint32_t)sl * BM + r) * 4, peer), rbar,
                   __float_as_uint(step));
    }
    // the peer's last accesses to this CTA are its acknowledgements of the
    // last tiles: wait for them (bounded) before the shared memory goes
    for (int j = max(0, n_tiles - kSlots); j < n_tiles; ++j)
      mbar_wait(bar(Bars::tx_ok + 4 * (j % kSlots) + w), (j / kSlots) & 1, nullptr);
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax
    const int sw = warp - kSoftmaxWarp0;
    const uint32_t lane_off = (uint32_t)(sw * 32) << 16;
    const uint32_t peer_tx = map_peer(bar(Bars::tx_ok + sw), peer);
    float m_used = -INFINITY, l = 0.f;
    // Q dims 0..127 of row r: staged (128-byte swizzle) -> TMEM as bf16 pairs
    bool ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::q_full), 0, abort));
    if (ok) {
#pragma unroll
      for (int c = 0; c < kQTmemChunks; ++c) {
        const uint4* row = reinterpret_cast<const uint4*>(smem_raw + kV + c * kQChunk + r * 128);
        uint32_t qw[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint4 v = row[g ^ (r & 7)];
          qw[4 * g] = v.x;
          qw[4 * g + 1] = v.y;
          qw[4 * g + 2] = v.z;
          qw[4 * g + 3] = v.w;
        }
        tmem_st32(tmem + lane_off + kColQ + 32 * c, qw);
      }
      tmem_wait_st();
      fence_proxy_async_smem();  // the V loads may now overwrite the staging area
      tc_fence_before();
      mbar_arrive(bar(Bars::q_tmem));
    }
    for (int j = 0; j < n_tiles; ++j) {
      const int sb = j % kNS;
      // the padding bits of this key tile (all kept without a mask), read
      // before the wait so the load overlaps it
      const uint64_t keep =
          (kExtras && kb.bits) ? kb.bits[(long)b * kb.words + kt0 + j] : ~0ull;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::s_full + sb), (j / kNS) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      float x[BN];
      {
        uint32_t sr[BN];  // own partial (fp32)
        tmem_ld32(tmem + lane_off + sb * BN, sr);
        tmem_ld32(tmem + lane_off + sb * BN + 32, sr + 32);
        tmem_wait_ld();
        // + the peer's partial of S_j (int16 pairs and a step, in log2 units)
        ok = __all_sync(0xffffffffu, mbar_wait_cluster(bar(Bars::rx_full + 4 * (j % kSlots) + sw),
                                                        (j / kSlots) & 1, abort));
        if (!ok) break;
        const uint4* in = reinterpret_cast<const uint4*>(smem_raw + kX + (j % kSlots) * kXSlot +
                                                         r * (BN * 2));
        const float step =
            *reinterpret_cast<const float*>(smem_raw + kXS + ((j % kSlots) * BM + r) * 4);
#pragma unroll
        for (int q = 0; q < BN / 8; ++q) {
          const uint4 v = in[q ^ (r & 7)];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // int16 q -> float exactly: flip the sign bits (q + 32768 in
            // [0, 65535]), place each half below the exponent of 2^23, then
            // subtract 2^23 + 32768
            const uint32_t u = w[e] ^ 0x80008000u;
            const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7610)) - 8421376.f;
            const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7632)) - 8421376.f;
            const int c = 8 * q + 2 * e;
            x[c] = fmaf(f0, step, __uint_as_float(sr[c]) * scale_log2);
            x[c + 1] = fmaf(f1, step, __uint_as_float(sr[c + 1]) * scale_log2);
          }
        }
      }
      // the slot's rows of this warp are read (the values are in x): re-arm
      // the channel for tile j + kSlots, then let the peer's sender refill it
      __syncwarp();
      if (lane == 0) {
        if (j + kSlots < n_tiles)
          mbar_arrive_expect_tx(bar(Bars::rx_full + 4 * (j % kSlots) + sw), kXWarp);
        mbar_arrive_remote(peer_tx + 32u * (uint32_t)(j % kSlots));
      }
      // x: logits of S_j in log2 units (soft-capped there when asked)
      if (kExtras && cap2 > 0.f) {
        const float k = 1.f / cap2;
#pragma unroll
        for (int c = 0; c < BN; ++c) x[c] = cap2 * tanh_fast(x[c] * k);
      }
      const int key0 = (kt0 + j) * BN;
      float mt = -INFINITY;
      if (key0 >= lo && key0 + BN - 1 <= hi && (!kExtras || keep == ~0ull)) {
#pragma unroll
        for (int c = 0; c < BN; ++c) mt = fmaxf(mt, x[c]);
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          x[c] = (key0 + c >= lo && key0 + c <= hi && (!kExtras || ((keep >> c) & 1))) ? x[c]
                                                                                     : -INFINITY;
          mt = fmaxf(mt, x[c]);
        }
      }
      const bool first = m_used == -INFINITY;
      const bool grow = !first && mt > m_used + 16.f;
      if (__any_sync(0xffffffffu, grow)) {
        // PV_{j-1} must be done; S_j done implies PV_{j-kNS} is, so o_done
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
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + kColO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(tmem + lane_off + kColO + c0, o);
        }
        tmem_wait_st();
      }
      if (first && mt != -INFINITY) m_used = mt;
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      float rs = 0.f;
      uint32_t pk[BN / 2];
#pragma unroll
      for (int e = 0; e < BN / 2; ++e) {
        const float e0 = ex2_approx(x[2 * e] + neg_m);
        const float e1 = ex2_approx(x[2 * e + 1] + neg_m);
        __nv_bfloat162 bb = __floats2bfloat162_rn(e0, e1);
        pk[e] = *reinterpret_cast<uint32_t*>(&bb);
        // the row sum adds the P values the PV product multiplies (bf16)
        rs += __uint_as_float(pk[e] << 16) + __uint_as_float(pk[e] & 0xffff0000u);
      }
      // P_j overwrites S_j: the senders must have read it
      ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::s_read + sb), (j / kNS) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      tmem_st32(tmem + lane_off + sb * BN, pk);
      tmem_wait_st();
      l += rs;
      tc_fence_before();
      mbar_arrive(bar(Bars::p_full + sb));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_tiles > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(Bars::o_last), 0, abort));
    if (ok && n_tiles > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* dst = out + (((long)b * T_ + i) * Hq + hrow) * (2 * DH) + dcol0;
#pragma unroll 1
      for (int c0 = 0; c0 < DH; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + kColO + c0, o);
        tmem_wait_ld();
        if (i < T_) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 bb = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv,
                                                      __uint_as_float(o[2 * e + 1]) * inv);
            pk[e] = *reinterpret_cast<uint32_t*>(&bb);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) record_status(status, G4ATTN_EDEVICE);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_attention_pair(const LayerCfg& L, int B, int T, const void* q_hat, KVSrc kv,
                                  RowIntervals rows, KeyBits kb, void* out, int* status,
                                  cudaStream_t s) {
  if (L.d != 2 * DH) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv;
  const int gp_log2 = gqa_pack_log2(L.Hq, L.Hkv);
  const uint64_t es = 2, D = 2 * DH;
  {  // q_hat [B, T, Hq, 512]: dims (512, Hq, T, B)
    const uint64_t dims[4] = {D, (uint64_t)L.Hq, (uint64_t)T, (uint64_t)B};
    const uint64_t str[3] = {D * es, (uint64_t)L.Hq * D * es, (uint64_t)T * L.Hq * D * es};
    const uint32_t box[4] = {64, (uint32_t)(1 << gp_log2), (uint32_t)(BM >> gp_log2), 1};
    if (!make_bf16_map(&tq, q_hat, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {  // K, V [B * Hkv, cap, 512]; rows at positions >= kv.len read as zero
    const uint64_t dims[3] = {D, (uint64_t)kv.len, (uint64_t)B * L.Hkv};
    const uint64_t str[2] = {D * es, (uint64_t)kv.cap * D * es};
    const uint32_t box[3] = {64, BN, 1};
    if (!make_bf16_map(&tk, kv.k, 3, dims, str, box)) return cudaErrorInvalidValue;
    if (!make_bf16_map(&tv, kv.v, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  const bool extras = kb.bits != nullptr || L.softcap > 0.f;
  auto kern = extras ? attn_pair_kernel<true> : attn_pair_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kAlloc);
  if (e != cudaSuccess) return e;
  const float scale_log2 = L.scale * 1.4426950408889634f;
  const int bp = BM >> gp_log2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((T + bp - 1) / bp * 2, L.Hq >> gp_log2, B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, rows, kb,
                         static_cast<__nv_bfloat16*>(out), T, L.Hq, L.Hkv, L.layer_type,
                         L.window, scale_log2, softcap_log2(L), gp_log2, status);
  if (e != cudaSuccess) return e;
  count_launch();
  return cudaGetLastError();
}

}  // namespace g4
