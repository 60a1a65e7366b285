// Split-KV decode on tensor cores for bf16 caches ("Gemma 4" Keras docs,
// "Gemma4ConditionalGenerate": decoding over the per-layer KV cache;
// "Gemma 4" overview blog, "Shared KV Cache").
//
// The query heads of one KV head (g <= 8; grouped-query attention) form the
// N = 8 side of m16n8k16 MMAs, so every cache byte is read once per KV head
// and the arithmetic stays far below the tensor pipe's rate: the kernel is an
// HBM stream.
//
// CTA = (chunk of positions, KV head, sequence), 5 warps:
//   warp 4     TMA producer: 16-key K and V tiles (128-byte swizzled boxes of
//              64 dims) into a ring of NS stages (128-192 KB in flight)
//   warps 0-3  take tiles round-robin (tile i: warp i % 4, stage i % NS with
//              NS a multiple of 4, so every stage has one consumer); per tile:
//                S^T = K Q^T            (16 keys x 8 heads, ldmatrix + mma)
//                online softmax per head (the thread's two heads are the same
//                in S^T and in its O^T accumulators: no shuffles for O)
//                O^T += V^T P^T         (ldmatrix.trans for V^T, movmatrix
//                                        turns P into the B operand)
// At the end the 4 warps' partial softmaxes are merged in shared memory and
// the chunk's (m, l, o~) are written for the combine kernel (decode.cu).
#include <cuda.h>

#include "common.cuh"
#include "g4attn.h"
#include "sm100.cuh"

namespace g4 {

using namespace sm100;

namespace {

constexpr int kConsumers = 4;
constexpr int kThreadsDm = (kConsumers + 1) * 32;
constexpr int kKeys = 16;  // keys per tile

template <int D>
struct DmLayout {
  static constexpr int kBoxes = D / 64;
  static constexpr uint32_t kBox = kKeys * 128;            // 16 keys x 64 dims, 2 KB
  static constexpr uint32_t kTile = kBoxes * kBox;         // K (or V) of one tile
  static constexpr uint32_t kStage = 2 * kTile;            // K then V
  // Stage count: a multiple of the consumer count, so stage s is only ever
  // consumed by warp s % 4 and that warp waits its phases in order (a parity
  // wait is only meaningful when the previous phase is known to be complete).
  static constexpr int kFit = (192 * 1024) / kStage > 16 ? 16 : (192 * 1024) / kStage;
  static constexpr int kStages = kFit - kFit % kConsumers;
  static_assert(kStages >= kConsumers, "at least one stage per consumer");
  static constexpr uint32_t kQ = kStages * kStage;         // q_hat [8][D] bf16
  static constexpr uint32_t kBars = kQ + 8 * D * 2;        // full[NS], empty[NS]
  static constexpr uint32_t kAlloc = kBars + 2 * kStages * 8 + 64;
  static constexpr uint32_t kMerge = kConsumers * 8 * D * 4 + kConsumers * 8 * 8;
  static_assert(kMerge <= kQ, "merge buffer fits");
};

// single-tensor caches: warps that rebuild K (with the 5 others, two warps
// per sub-partition, so the consumers keep their 252 registers)
constexpr int kRebuilders = 3;

// Shared-memory plan of a single-tensor decode (set by the host): a ring of
// loaded V tiles, and a smaller ring of rebuilt K boxes (one per 64-dim box
// that has rotated dims) whose slots are free again once the S product of
// their tile is done, so the load ring keeps more tiles in flight.
struct DmSingle {
  int ns;              // load stages (a multiple of 4)
  uint32_t stage;      // bytes per load stage (one V tile)
  int nrs;             // rebuilt slots (a multiple of the rebuilders)
  uint32_t rb;         // the rebuilt ring: [nrs][nrb] boxes
  uint32_t q, bars;    // q_hat [8][D]; full, empty, ready [NS] each, rebuilt-slot free [nrs]
  uint32_t freq;       // [R] the rotated pairs' frequencies in turns (64-bit fractions)
  uint32_t wab;        // [R] float2: (w_k[k], w_k[k + D/2])
  uint32_t box_slot;   // 4 bits per 64-dim box: its rebuilt slot, 15 = loaded tile
  uint32_t slot_box;   // 4 bits per rebuilt slot: its box
  int nrb;             // rebuilt boxes
  int nw;              // bf16 pair-words per half that the rotation covers
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// D (16x8, fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of (key, dim) inside a K or V tile: box dim/64, row key, the
// 16-byte chunk of the dim swizzled by the row (128-byte swizzle).
__device__ __forceinline__ uint32_t tile_off(int key, int dim) {
  return (uint32_t)((dim >> 6) * (kKeys * 128) + key * 128 + ((((dim & 63) >> 3) ^ (key & 7)) << 4));
}

}  // namespace

// kSingle: a single-tensor cache of a K=V layer.  The cache holds V =
// RMSNorm(k_raw) alone and K = RoPE(V * w_k) is rebuilt per tile: w_k folds
// into the query on the unrotated dims (q.(V*w) = (q*w).V), so only the
// 64-dim boxes that hold rotated dims are rebuilt, by three extra warps
// taking tiles in turn, into a slot of the rebuilt ring; the S product reads
// those boxes from there.
// The angle of key pos0 + j is pos0 f then j f: cos/sin of pos0 f come from
// one fp64-reduced sincos per pair and tile, those of j f (with w_k folded
// in) from a per-CTA table.  V is the loaded tile itself.
template <int D, bool kSingle>
__global__ void __launch_bounds__(kThreadsDm + (kSingle ? kRebuilders * 32 : 0), 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __nv_bfloat16* __restrict__ q_raw, const __nv_bfloat16* __restrict__ wq,
                      const int32_t* __restrict__ len, int cap, int rolling, int Hq, int Hkv,
                      int layer_type, int window, float scale_log2, float cap2, KeyMask km,
                      float eps, int chunk, int nc, float* __restrict__ part_ml,
                      float* __restrict__ part_o, int* status,
                      const __nv_bfloat16* __restrict__ wk_single, DmSingle sp,
                      const __grid_constant__ RopeParams rope) {
  using Ly = DmLayout<D>;
  const int NS = kSingle ? sp.ns : Ly::kStages;
  const uint32_t kStageB = kSingle ? sp.stage : Ly::kStage;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the swizzled boxes assume a 1024-byte aligned base
    if (threadIdx.x == 0) record_status(status, G4ATTN_EDEVICE);
    return;
  }
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + (kSingle ? sp.bars : Ly::kBars);
  __shared__ int s_abort;
  volatile int* abort = &s_abort;

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
  const int lo = layer_type == 0 ? max(0, P - window + 1) : 0;
  const int c0 = (lo & ~15) + c * chunk;  // chunk start, 16-aligned
  if (c0 > P) return;
  const int c1 = min(P + 1, c0 + chunk);
  const int t0 = c0 >> 4;
  const int n_t = ((c1 - 1) >> 4) - t0 + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bars + 8 * s, 1);             // full: producer's expect_tx
      mbar_init(bars + 8 * (NS + s), 1);      // empty: the consuming warp
      if (kSingle) mbar_init(bars + 8 * (2 * NS + s), 32);  // ready: a rebuilding warp
    }
    if (kSingle)
      for (int r = 0; r < sp.nrs; ++r) mbar_init(bars + 8 * (3 * NS + r), 1);  // slot r free
    s_abort = 0;
    fence_barrier_init();
  }
  // query prologue (RMSNorm * w_q, RoPE at P) of the g heads into q_hat; rows g..7 zero
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + (kSingle ? sp.q : Ly::kQ));
  if (warp < kConsumers) {
    for (int hh = warp; hh < 8; hh += kConsumers) {
      if (hh < g) {
        float y0[D / 64], y1[D / 64];
        prologue_vec<__nv_bfloat16, D>(q_raw + ((long)b * Hq + kvh * g + hh) * D, wq, P, &rope,
                                       eps, y0, y1);
        if constexpr (kSingle) {  // w_k folds into the query on the unrotated pairs
          float w0[D / 64], w1[D / 64];
          Vec<__nv_bfloat16, D / 64>::load(wk_single + lane * (D / 64), w0);
          Vec<__nv_bfloat16, D / 64>::load(wk_single + D / 2 + lane * (D / 64), w1);
#pragma unroll
          for (int e = 0; e < D / 64; ++e)
            if (lane * (D / 64) + e >= rope.rotated_pairs) {
              y0[e] *= w0[e];
              y1[e] *= w1[e];
            }
        }
        store_vec<__nv_bfloat16, D>(qs + hh * D, y0, y1);
      } else {
        for (int k = lane; k < D; k += 32) qs[hh * D + k] = __float2bfloat16_rn(0.f);
      }
    }
  }
  if constexpr (kSingle) {
    // per rotated pair k: its frequency and (w_k[k], w_k[k + D/2]), in shared
    // memory (lane-indexed reads of the kernel's parameter space serialise)
    unsigned long long* fq = reinterpret_cast<unsigned long long*>(smem + sp.freq);
    float2* wab = reinterpret_cast<float2*>(smem + sp.wab);
    for (int k = threadIdx.x; k < rope.rotated_pairs; k += blockDim.x) {
      fq[k] = rope.turns[k];
      wab[k] = make_float2(__bfloat162float(wk_single[k]), __bfloat162float(wk_single[k + D / 2]));
    }
  }
  __syncthreads();

  float acc[D / 16][4];  // O^T of this thread: dims 16mt + lane/4 (+8) x heads hA, hB
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;  // heads hA = 2(lane%4), hB = hA+1

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int issued = 0;
      for (int i = 0; i < n_t; ++i) {
        const int s = i % NS;
        if (!mbar_wait(bars + 8 * (NS + s), ((i / NS) & 1) ^ 1, abort)) break;
        const int pos = (t0 + i) * kKeys;
        const int slot = rolling ? pos % cap : pos;  // rolling caches: cap % 16 == 0
        const uint32_t st = base + s * kStageB;
        mbar_arrive_expect_tx(bars + 8 * s, kSingle ? Ly::kTile : Ly::kStage);
#pragma unroll
        for (int bx = 0; bx < Ly::kBoxes; ++bx) {
          tma_load_3d(st + bx * Ly::kBox, &tm_k, bars + 8 * s, bx * 64, slot, b * Hkv + kvh);
          if constexpr (!kSingle)
            tma_load_3d(st + Ly::kTile + bx * Ly::kBox, &tm_v, bars + 8 * s, bx * 64, slot,
                        b * Hkv + kvh);
        }
        issued = i + 1;
      }
      if (*abort)  // let the copies already issued land before the CTA exits
        for (int i = max(0, issued - NS); i < issued; ++i)
          mbar_wait(bars + 8 * (i % NS), (i / NS) & 1, nullptr);
    }
  } else if (kSingle && warp > kConsumers) {
    // ------------------------------------------------------------ K rebuild
    // Rebuilder rw takes tiles i = rw (mod 3); NS and nrs are multiples of
    // 3, so every stage and every rebuilt slot has one rebuilder, which waits
    // its phases in order.  The rotated dims form nch 16-byte chunks (8
    // pairs) per half.  When nch divides 32 (every Gemma 4 K=V shape:
    // R = d/8) lane l keeps chunk c = l % nch and takes kpl consecutive keys
    // from j0; the 8 pairs' angles start from one sincos each per tile and
    // step key to key by the angle addition formulas.  Other nch: any (key,
    // chunk) per item, one sincos per pair and item.
    const int rw = warp - kConsumers - 1;
    const int R = rope.rotated_pairs, nch = sp.nw / 4;
    const unsigned long long* fq = reinterpret_cast<const unsigned long long*>(smem + sp.freq);
    const float2* wab = reinterpret_cast<const float2*>(smem + sp.wab);
    const bool fixed_c = 32 % nch == 0;
    const int c = fixed_c ? lane % nch : 0, grp = fixed_c ? 32 / nch : 1;
    const int kpl = grp >= kKeys ? 1 : kKeys / grp, j0 = (fixed_c ? lane / nch : 0) * kpl;
    float wa[8], wb[8], cd[8], sd[8];  // per pair of chunk c: weights, the angle of one key
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int k = 8 * c + t;
      wa[t] = wb[t] = cd[t] = 1.f;
      sd[t] = 0.f;
      if (fixed_c && k < R) {
        const float2 u = wab[k];
        wa[t] = u.x;
        wb[t] = u.y;
        rope_sincos_turns(1, fq[k], &sd[t], &cd[t]);
      }
    }
    // one item: key j, chunk cc, the pairs' angles (cs, sn) at pos0 + j
    auto item = [&](const uint8_t* sk, uint8_t* sr, int j, int cc, const float* cs,
                    const float* sn, const float* ua, const float* ub) {
      const int da = 8 * cc, db = D / 2 + 8 * cc;
      const uint32_t oa = tile_off(j, da), ob = tile_off(j, db);
      const uint4 xa = *reinterpret_cast<const uint4*>(sk + oa);
      const uint4 xb = *reinterpret_cast<const uint4*>(sk + ob);
      const uint32_t wa4[4] = {xa.x, xa.y, xa.z, xa.w}, wb4[4] = {xb.x, xb.y, xb.z, xb.w};
      uint32_t ra[4], rb[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float a[2] = {__uint_as_float(wa4[h] << 16), __uint_as_float(wa4[h] & 0xffff0000u)};
        float bb[2] = {__uint_as_float(wb4[h] << 16), __uint_as_float(wb4[h] & 0xffff0000u)};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = 2 * h + e;
          if (da + t < R) {  // unrotated pairs pass through exactly
            const float p = a[e] * ua[t], q = bb[e] * ub[t];
            a[e] = p * cs[t] - q * sn[t];
            bb[e] = p * sn[t] + q * cs[t];
          }
        }
        ra[h] = pack_bf16(a[0], a[1]);
        rb[h] = pack_bf16(bb[0], bb[1]);
      }
      const int sa = (sp.box_slot >> (4 * (da >> 6))) & 15;
      const int sb = (sp.box_slot >> (4 * (db >> 6))) & 15;
      *reinterpret_cast<uint4*>(sr + sa * Ly::kBox + (oa & (Ly::kBox - 1))) =
          make_uint4(ra[0], ra[1], ra[2], ra[3]);
      *reinterpret_cast<uint4*>(sr + sb * Ly::kBox + (ob & (Ly::kBox - 1))) =
          make_uint4(rb[0], rb[1], rb[2], rb[3]);
    };
    for (int i = rw; i < n_t; i += kRebuilders) {
      const int s = i % NS, rs = i % sp.nrs;
      if (!__all_sync(0xffffffffu, mbar_wait(bars + 8 * s, (i / NS) & 1, abort))) break;
      // the slot's previous tile has been read by its S product
      if (i >= sp.nrs && !__all_sync(0xffffffffu, mbar_wait(bars + 8 * (3 * NS + rs),
                                                             ((i / sp.nrs) - 1) & 1, abort)))
        break;
      const long pos0 = (long)(t0 + i) * kKeys;
      const uint8_t* sk = smem + s * kStageB;
      uint8_t* sr = smem + sp.rb + rs * (sp.nrb * Ly::kBox);  // this tile's rebuilt boxes
      if (fixed_c) {
        if (j0 < kKeys) {
          float cs[8], sn[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            cs[t] = 1.f;
            sn[t] = 0.f;
            if (8 * c + t < R) rope_sincos_turns((uint32_t)(pos0 + j0), fq[8 * c + t], &sn[t], &cs[t]);
          }
          for (int m = 0; m < kpl; ++m) {
            item(sk, sr, j0 + m, c, cs, sn, wa, wb);
#pragma unroll
            for (int t = 0; t < 8; ++t) {  // the angle of the next key
              const float cn = cs[t] * cd[t] - sn[t] * sd[t];
              sn[t] = sn[t] * cd[t] + cs[t] * sd[t];
              cs[t] = cn;
            }
          }
        }
      } else {
        for (int it = lane; it < kKeys * nch; it += 32) {
          const int j = it / nch, cc = it - j * nch;
          float cs[8], sn[8], ua[8], ub[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int k = 8 * cc + t;
            cs[t] = ua[t] = ub[t] = 1.f;
            sn[t] = 0.f;
            if (k < R) {
              rope_sincos_turns((uint32_t)(pos0 + j), fq[k], &sn[t], &cs[t]);
              ua[t] = wab[k].x;
              ub[t] = wab[k].y;
            }
          }
          item(sk, sr, j, cc, cs, sn, ua, ub);
        }
      }
      // the rest of the rebuilt boxes (dims past the rotated words) is V as loaded
      for (int it = lane; it < sp.nrb * kKeys * 8; it += 32) {
        const int sl = it / (kKeys * 8), r = it - sl * (kKeys * 8);
        const int j = r >> 3, bx = (sp.slot_box >> (4 * sl)) & 15;
        const int dim = bx * 64 + (r & 7) * 8;
        if ((dim & (D / 2 - 1)) < 8 * nch) continue;
        const uint32_t o = tile_off(j, dim);
        *reinterpret_cast<uint4*>(sr + sl * Ly::kBox + (o & (Ly::kBox - 1))) =
            *reinterpret_cast<const uint4*>(sk + o);
      }
      mbar_arrive(bars + 8 * (2 * NS + s));
    }
  } else if (warp < kConsumers) {
    // ------------------------------------------------------------ consumers
    // B operand of S^T = K Q^T for every 16-dim step: q_hat[head = lane/4][dims]
    uint32_t qb[D / 16][2];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const __nv_bfloat16* qr = qs + (lane >> 2) * D + kk * 16 + (lane & 3) * 2;
      qb[kk][0] = *reinterpret_cast<const uint32_t*>(qr);
      qb[kk][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
    }
    for (int i = warp; i < n_t; i += kConsumers) {
      const int s = i % NS;
      // two-tensor caches: the copy landed; single-tensor: K is rebuilt too
      const uint32_t wbar = bars + 8 * ((kSingle ? 2 * NS : 0) + s);
      if (!__all_sync(0xffffffffu, mbar_wait(wbar, (i / NS) & 1, abort))) break;
      const uint32_t kb = base + s * kStageB, vb = kb + Ly::kTile;
      // single-tensor: this tile's rebuilt boxes
      const uint32_t rbb = kSingle ? base + sp.rb + (i % sp.nrs) * (sp.nrb * Ly::kBox) : 0u;
      const int pos0 = (t0 + i) * kKeys;
      if (pos0 + kKeys - 1 > P) {  // last tile: zero V rows past P (never written)
        const int first = P - pos0 + 1;
        uint8_t* vrow = smem + s * kStageB + (kSingle ? 0 : Ly::kTile);
        for (int e = lane; e < (kKeys - first) * Ly::kBoxes * 8; e += 32) {
          const int rr = first + e / (Ly::kBoxes * 8), rest = e % (Ly::kBoxes * 8);
          *reinterpret_cast<uint4*>(vrow + (rest >> 3) * Ly::kBox + rr * 128 + (rest & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();  // a later TMA refill of this stage comes after these writes
        __syncwarp();
      }
      // S^T (16 keys x 8 heads)
      // two accumulators over alternate 16-dim steps halve the chain of
      // dependent MMAs (summed below)
      float sc[4] = {0.f, 0.f, 0.f, 0.f}, sc2[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int mi = lane >> 3;
        const int key = (lane & 7) + (mi & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t a[4];
          // single-tensor cache: the boxes with rotated dims come from their slot
          uint32_t src = kb;
          if constexpr (kSingle) {
            const uint32_t sl = (sp.box_slot >> (4 * (kk >> 2))) & 15u;
            if (sl != 15u) src = rbb + sl * Ly::kBox - (kk >> 2) * Ly::kBox;
          }
          ldsm_x4(src + tile_off(key, kk * 16 + (mi >> 1) * 8), a);
          mma16816((kk & 1) ? sc2 : sc, a, qb[kk][0], qb[kk][1]);
        }
      }
      if constexpr (kSingle) {  // the rebuilt slot is free for the tile nrs later
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + 8 * (3 * NS + i % sp.nrs));
      }
      // masked scores in log2 units: rows = keys pos0 + lane/4 (+8), cols = heads;
      // a padding key of the prompt (km) is masked like one outside [lo, P]
      const int kA = pos0 + (lane >> 2), kB = kA + 8;
      auto kept = [&](int k) {
        return !km.keep || k >= km.len || km.keep[(long)b * km.len + k] != 0;
      };
      const bool vA = kA >= lo && kA <= P && kept(kA), vB = kB >= lo && kB <= P && kept(kB);
      float r[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) r[e] = (sc[e] + sc2[e]) * scale_log2;
      if (cap2 > 0.f) {  // soft-cap in log2 units
#pragma unroll
        for (int e = 0; e < 4; ++e) r[e] = cap2 * tanh_fast(r[e] * (1.f / cap2));
      }
      const float x0 = vA ? r[0] : -INFINITY;  // (kA, head hA)
      const float x1 = vA ? r[1] : -INFINITY;  // (kA, head hB)
      const float x2 = vB ? r[2] : -INFINITY;  // (kB, head hA)
      const float x3 = vB ? r[3] : -INFINITY;  // (kB, head hB)
      float tA = fmaxf(x0, x2), tB = fmaxf(x1, x3);
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        tA = fmaxf(tA, __shfl_xor_sync(0xffffffffu, tA, o));
        tB = fmaxf(tB, __shfl_xor_sync(0xffffffffu, tB, o));
      }
      const float nA = fmaxf(mA, tA), nB = fmaxf(mB, tB);
      const float ngA = nA == -INFINITY ? 0.f : -nA, ngB = nB == -INFINITY ? 0.f : -nB;
      const float cA = ex2_approx(mA + ngA), cB = ex2_approx(mB + ngB);  // 0 while m = -inf
      const float p0 = ex2_approx(x0 + ngA), p2 = ex2_approx(x2 + ngA);
      const float p1 = ex2_approx(x1 + ngB), p3 = ex2_approx(x3 + ngB);
      float sA = p0 + p2, sB = p1 + p3;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        sA += __shfl_xor_sync(0xffffffffu, sA, o);
        sB += __shfl_xor_sync(0xffffffffu, sB, o);
      }
      lA = lA * cA + sA;
      lB = lB * cB + sB;
      mA = nA;
      mB = nB;
      // P^T as the B operand: transpose the (keys x heads) 8x8 blocks
      const uint32_t pb0 = movm_t(pack_bf16(p0, p1));
      const uint32_t pb1 = movm_t(pack_bf16(p2, p3));
      {
        const int mi = lane >> 3;
        const int key = (lane & 7) + (mi >> 1) * 8;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          acc[mt][0] *= cA;
          acc[mt][1] *= cB;
          acc[mt][2] *= cA;
          acc[mt][3] *= cB;
          uint32_t a[4];
          ldsm_x4_t((kSingle ? kb : vb) + tile_off(key, mt * 16 + (mi & 1) * 8), a);
          mma16816(acc[mt], a, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + 8 * (NS + s));
    }
  }
  __syncthreads();  // every tile consumed: no copy is in flight, the ring can be reused
  if (*abort) {
    // an empty partial (m = -inf, l = 0, o~ = 0): the combine then ignores
    // this chunk instead of reading what an earlier call left in the buffer
    if (threadIdx.x == 0) record_status(status, G4ATTN_EDEVICE);
    for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
      const int h = e / D, dim = e - h * D;
      const long pidx = ((long)b * Hq + kvh * g + h) * nc + c;
      part_o[pidx * D + dim] = 0.f;
      if (dim == 0) {
        part_ml[2 * pidx] = -INFINITY;
        part_ml[2 * pidx + 1] = 0.f;
      }
    }
    return;
  }
  // merge the 4 warps' partial softmaxes (each relative to its own maxima)
  float* red = reinterpret_cast<float*>(smem);                           // [4][8][D]
  float* rml = reinterpret_cast<float*>(smem + kConsumers * 8 * D * 4);  // [4][8][m, l]
  if (warp < kConsumers) {
    const int hA = 2 * (lane & 3), hB = hA + 1, dr = lane >> 2;
    float* ra = red + (warp * 8 + hA) * D;
    float* rb = red + (warp * 8 + hB) * D;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      ra[mt * 16 + dr] = acc[mt][0];
      rb[mt * 16 + dr] = acc[mt][1];
      ra[mt * 16 + dr + 8] = acc[mt][2];
      rb[mt * 16 + dr + 8] = acc[mt][3];
    }
    if (lane < 4) {
      rml[(warp * 8 + hA) * 2] = mA;
      rml[(warp * 8 + hA) * 2 + 1] = lA;
      rml[(warp * 8 + hB) * 2] = mB;
      rml[(warp * 8 + hB) * 2 + 1] = lB;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
    const int h = e / D, dim = e - h * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, rml[(w * 8 + h) * 2]);
    float den = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float mw = rml[(w * 8 + h) * 2];
      const float a = mw == -INFINITY ? 0.f : ex2_approx(mw - M);
      den += a * rml[(w * 8 + h) * 2 + 1];
      o += a * red[(w * 8 + h) * D + dim];
    }
    const long pidx = ((long)b * Hq + kvh * g + h) * nc + c;
    part_o[pidx * D + dim] = o;
    if (dim == 0) {  // the combine kernel works in natural-log units
      part_ml[2 * pidx] = M * 0.69314718055994531f;
      part_ml[2 * pidx + 1] = den;
    }
  }
}

bool decode_mma_supported(const LayerCfg& L, int cap, int rolling) {
  return L.dtype == 0 && L.Hq / L.Hkv <= 8 && (!rolling || cap % kKeys == 0);
}

template <int D>
static cudaError_t run_mma(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                           const void* cache_k, const void* cache_v, const void* wk_single,
                           const int32_t* len, int cap, int rolling, KeyMask km,
                           const DecodePlan& plan, float* part_ml, float* part_o, int* status,
                           cudaStream_t s) {
  using Ly = DmLayout<D>;
  const bool single = cache_v == nullptr;  // single-tensor cache of a K=V layer
  CUtensorMap tk, tv;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)cap, (uint64_t)B * L.Hkv};
  const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)cap * D * 2};
  const uint32_t box[3] = {64, kKeys, 1};
  if (!make_bf16_map(&tk, cache_k, 3, dims, str, box)) return cudaErrorInvalidValue;
  if (!make_bf16_map(&tv, single ? cache_k : cache_v, 3, dims, str, box))
    return cudaErrorInvalidValue;
  DmSingle sp{};
  uint32_t smem_bytes = Ly::kAlloc;
  if (single) {
    // the 64-dim boxes that hold rotated dims (pairs k < R: dims k and k + D/2)
    const int R = L.rope.rotated_pairs;
    uint32_t rot = 0;
    for (int k = 0; k < R; ++k) rot |= (1u << (k / 64)) | (1u << ((k + D / 2) / 64));
    sp.box_slot = 0xffffffffu;
    for (int bx = 0; bx < Ly::kBoxes; ++bx)
      if ((rot >> bx) & 1u) {
        sp.box_slot = (sp.box_slot & ~(15u << (4 * bx))) | ((uint32_t)sp.nrb << (4 * bx));
        sp.slot_box |= (uint32_t)bx << (4 * sp.nrb);
        ++sp.nrb;
      }
    sp.nw = (R + 7) / 8 * 4;  // whole 16-byte chunks of each half
    sp.stage = Ly::kTile;
    const uint32_t rbytes = sp.nrb * Ly::kBox;  // one rebuilt slot
    const uint32_t fixed = 8 * D * 2 + (3 * 12 + 6) * 8 + 16 * (uint32_t)R + 64;
    const uint32_t budget = 227 * 1024 - 1024 - fixed;  // 1 KB: static shared memory
    // 12 load stages (a multiple of the 4 consumers and the 3 rebuilders)
    // and 6 rebuilt slots (a multiple of the rebuilders); the largest head
    // (d 512: 16 KB tiles, two rebuilt boxes) fills the 227 KB with them
    sp.ns = 4 * kRebuilders;
    sp.nrs = 2 * kRebuilders;
    if (sp.ns * sp.stage + sp.nrs * rbytes > budget || (uint32_t)sp.ns * sp.stage < Ly::kMerge)
      return cudaErrorInvalidValue;
    sp.rb = sp.ns * sp.stage;
    sp.q = sp.rb + sp.nrs * rbytes;
    sp.bars = sp.q + 8 * D * 2;
    sp.freq = (sp.bars + (3 * sp.ns + sp.nrs) * 8 + 15) & ~15u;
    sp.wab = sp.freq + 8 * R;
    smem_bytes = sp.wab + 8 * R + 64;
  }
  auto kern = single ? decode_mma_kernel<D, true> : decode_mma_kernel<D, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.n_chunks, L.Hkv, B);
  kern<<<grid, kThreadsDm + (single ? kRebuilders * 32 : 0), smem_bytes, s>>>(
      tk, tv, static_cast<const __nv_bfloat16*>(q_raw), static_cast<const __nv_bfloat16*>(wq), len,
      cap, rolling, L.Hq, L.Hkv, L.layer_type, L.window, L.scale * 1.4426950408889634f,
      softcap_log2(L), km, L.eps, plan.chunk, plan.n_chunks, part_ml, part_o, status,
      static_cast<const __nv_bfloat16*>(wk_single), sp, L.rope);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_decode_mma(const LayerCfg& L, int B, const void* q_raw, const void* wq,
                              const void* cache_k, const void* cache_v, const void* wk_single,
                              const int32_t* len, int cap, int rolling, KeyMask km,
                              const DecodePlan& plan, float* part_ml, float* part_o,
                              int* status, cudaStream_t s) {
#define G4_MMA(D)                                                                          \
  return run_mma<D>(L, B, q_raw, wq, cache_k, cache_v, wk_single, len, cap, rolling, km, \
                    plan, part_ml, part_o, status, s)
  switch (L.d) {
    case 64: G4_MMA(64);
    case 128: G4_MMA(128);
    case 256: G4_MMA(256);
    case 512: G4_MMA(512);
  }
#undef G4_MMA
  return cudaErrorInvalidValue;
}

}  // namespace g4
