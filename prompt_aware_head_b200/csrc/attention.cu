// Flash-style attention over selected (query block, key block) tiles on
// sm_100a: tcgen05 MMA with TMEM accumulators, TMA-staged K/V tiles gathered
// through the block lists, a persistent CTA per SM taking work items from an
// atomic queue.
//
// What is computed follows the inferensys glossary ("block-sparse": only
// connected (query block, key block) pairs are computed) and the SD.Next
// sparse-attention commit log ("flex consumer": every selected tile is
// computed in full).  Per query row q of block i:
//     O_q = softmax(Q_q K_S^T * scale) V_S,  S = tokens of the kept blocks,
// with the online (running max / running sum) softmax of flash attention.
//
// B200 design (not from the pages):
//  * The tensor core runs at full rate only with M = 128, so a work item is
//    a PAIR of 64-row query blocks (i0, i1) of one head that shares a 128-row
//    tile.  It walks the sorted union of the two block lists; each union
//    entry carries two membership bits, and the softmax warps of a half give
//    zero probability to key blocks their query block did not select (and
//    skip their exponentials).  The planner picks, per head, the pairing
//    stride (1, 2 or 4 blocks apart) with the smallest total union.
//  * One step = two key blocks (N = 128): S = Q K^T is one asm block of
//    d/16 SS MMAs into TMEM; P is written back to TMEM as bf16 and
//    O += P V is one asm block of TS MMAs (A from TMEM).  S is double
//    buffered in TMEM so the MMAs of step g+1 overlap the softmax of step g.
//  * Warp roles: warp 0 TMA producer for Q and K, warp 10 TMA producer for V,
//    warp 1 issues the S MMAs and warp 11 the PV MMAs (one thread each),
//    warps 2-9 softmax / correction / epilogue (two warps per tile row, one
//    per key block of a step).
//  * Rescaling of O (in TMEM) happens only when a row's running max grows by
//    more than 2^8; otherwise the stale max is kept (exact after the final
//    division by the running sum).
//  * Every mbarrier wait is bounded; on timeout the kernel records an error,
//    drains its own TMA loads and MMAs, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

// Work item: x = bh, y = i0 | i1 << 16 (i1 = 0xFFFF: none), z = union
// length (key blocks), w = offset of the union list in int32 units (-1 dense).
struct AttnArgs {
  const int4* items;       // execution order (sparse mode)
  const int32_t* ulist;    // packed union entries j | bits << 16
  const int* n_items_dev;  // sparse mode: item count written by the planner
  int n_items_host;        // dense mode: item count
  int dense;               // 1: implicit full lists, pairs (2m, 2m+1)
  int N, nB, npairs_dense;
  int H, g;                // query heads; query heads per key/value head (K and V hold B H / g heads)
  __nv_bfloat16* O;
  float scale_log2;
  int* err;
  // Token-level key mask inside kept tiles, or null: word [b][j] holds bit r
  // set when key 64 j + r of batch b may be attended.
  const unsigned long long* kmask;
  // Work queue: work[0] is the next item to hand out, work[1] counts the CTAs
  // that have finished; the last CTA to finish resets both to 0.
  int* work;
  int queue;  // 1: items from the queue; 0: dealt by CTA index (small launches)
};

// Mask word of the key block of union entry e for the item's batch.  The
// kernel is built twice: without a key mask every word is all ones at
// compile time, so the unmasked kernel carries none of the masking code.
template <bool kMask>
__device__ __forceinline__ unsigned long long key_word(const AttnArgs& a, int bh, uint32_t e) {
  if constexpr (kMask) return __ldg(a.kmask + static_cast<size_t>(bh / a.H) * a.nB + (e & 0xFFFFu));
  else return ~0ull;
}

constexpr int kThreads = 384;  // Q/K producer, S issuer, 8 softmax warps, V producer, PV issuer
constexpr float kRescaleThreshold = 8.0f;       // log2 units: rescale O when the max grows by > 2^8
constexpr uint32_t kBackoffNs = 40;            // producer poll back-off (ns)

struct Item {
  int bh, i0, i1, len, off;
  int rot;  // the item walks its union list starting at entry rot (wrapping)
};

// Online softmax is exact in any key-block order, so each item starts its
// walk at an item-dependent offset: CTAs working on the same head then read
// different K/V blocks at any moment instead of all sweeping the same ones
// (which throttles L2).  The offset is a hash of (head, query block).
__device__ __forceinline__ int item_rotation(int bh, int i0, int len) {
  if (len <= 1) return 0;
  const uint32_t h = (static_cast<uint32_t>(bh) * 0x9E3779B1u) ^ (static_cast<uint32_t>(i0 + 1) * 0x85EBCA77u);
  return static_cast<int>((h >> 7) % static_cast<uint32_t>(len));
}

__device__ __forceinline__ Item load_item(const AttnArgs& a, int k) {
  Item it;
  if (a.dense) {
    it.bh = k / a.npairs_dense;
    const int m = k % a.npairs_dense;
    it.i0 = 2 * m;
    it.i1 = (2 * m + 1 < a.nB) ? 2 * m + 1 : kNoBlock;
    it.len = a.nB;
    it.off = -1;
  } else {
    const int4 v = a.items[k];
    it.bh = v.x;
    it.i0 = v.y & 0xFFFF;
    it.i1 = (v.y >> 16) & 0xFFFF;
    it.len = v.z;
    it.off = v.w;
  }
  it.rot = item_rotation(it.bh, it.i0, it.len);
  return it;
}

// Union entry e of an item: key block j in the low 16 bits, membership bits
// (bit 16: query block i0 selected j, bit 17: i1 selected j).
__device__ __forceinline__ uint32_t load_entry(const AttnArgs& a, const Item& it, int e) {
  int pos = e + it.rot;  // e < len, rot < len
  if (pos >= it.len) pos -= it.len;
  if (a.dense) return static_cast<uint32_t>(pos) | ((it.i1 == kNoBlock ? 1u : 3u) << 16);
  return static_cast<uint32_t>(a.ulist[it.off + pos]);
}

// Items are handed out through a queue (an atomic counter in the workspace):
// CTA c starts on item c, then takes the next item when it is ready for one,
// so CTAs that drew short items take more of them and all finish together.
// The items stay in the planner's order (each head's longest item first, then
// head-major, longest first within a head), so the CTAs still work through
// one head's K / V at a time.  In each CTA the Q / K producer takes the
// items and publishes each through a ring of kRing slots in shared memory;
// the other roles read the ring in the same order.
constexpr int kRing = 8;
constexpr uint32_t kRingReaders = 11;  // V producer, two MMA issuers, eight softmax warps

// The static deal of small launches (a few items per CTA, where the queue's
// atomics and final fence cost more than the balance gains): pass r gives
// CTA c item r G + c, or r G + G - 1 - c on odd passes.
__device__ __forceinline__ int item_index(int r, int cta, int G) {
  return r * G + ((r & 1) ? (G - 1 - cta) : cta);
}

// Reader side of the ring: the r-th item of this CTA (total when none is left).
__device__ __forceinline__ bool ring_take(int r, const int* ring, uint64_t* ring_full, uint64_t* ring_empty,
                                          volatile int* abort_flag, int* err, int* k) {
  const int slot = r & (kRing - 1);
  if (!mbar_wait(&ring_full[slot], (r / kRing) & 1, abort_flag, err)) return false;
  *k = ring[slot];
  mbar_arrive(&ring_empty[slot]);
  return true;
}

// ---------------------------------------------------------------- MMA issue
// S = Q K^T for one step: NK = d/16 MMAs, A = Q tile (K-major SW128 smem),
// B = K pair (K-major SW128 smem).  Descriptor start addresses advance by
// 32 B per 16-element K slice inside a 128-B swizzle atom, and by one
// 64-column chunk (16 KB: 128 rows x 128 B) every 4 slices.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
  if constexpr (D == 64) {
    asm volatile(
        "{\n .reg .pred p0, p1;\n .reg .b64 a1, a2, a3, b1, b2, b3;\n"
        " setp.eq.b32 p0, 1, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " add.s64 a1, %1, 2;\n add.s64 a2, %1, 4;\n add.s64 a3, %1, 6;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, p1;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p0, p1;\n .reg .b64 a1, a2, a3, a4, a5, a6, a7, b1, b2, b3, b4, b5, b6, b7;\n"
        " setp.eq.b32 p0, 1, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " add.s64 a1, %1, 2;\n add.s64 a2, %1, 4;\n add.s64 a3, %1, 6;\n"
        " add.s64 a4, %1, 1024;\n add.s64 a5, %1, 1026;\n add.s64 a6, %1, 1028;\n add.s64 a7, %1, 1030;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " add.s64 b4, %2, 1024;\n add.s64 b5, %2, 1026;\n add.s64 b6, %2, 1028;\n add.s64 b7, %2, 1030;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a4, b4, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a5, b5, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a6, b6, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], a7, b7, %3, p1;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc)
        : "memory");
  }
}

// O_c += P_c V_c for the step's key blocks c = 0 (and 1 when nblk = 2): each
// key block accumulates into its own O (TMEM columns d0 / d1), so the two
// softmax warps that own a row's two blocks keep independent running maxima.
// A = P (bf16 in TMEM, 8 columns per 16 keys; each block's P sits in the
// first half of that block's own 64 S columns, so block 1's starts 64 in),
// B = the block's V (MN-major SW128 smem [d/64 chunks][64 keys][128 B];
// 16 keys = 2 KB per slice; bdesc0 / bdesc1 address blocks 0 / 1).
__device__ __forceinline__ void issue_pv(uint32_t d0, uint32_t d1, uint32_t a_tmem, uint64_t bdesc0, uint64_t bdesc1,
                                         uint32_t idesc, uint32_t accumulate, int nblk) {
  if (nblk == 2) {
    asm volatile(
        "{\n .reg .pred p0, p1;\n .reg .b32 t1, t2, t3, t4, t5, t6, t7;\n"
        " .reg .b64 b1, b2, b3, b5, b6, b7;\n"
        " setp.ne.b32 p0, %6, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " add.u32 t1, %2, 8;\n add.u32 t2, %2, 16;\n add.u32 t3, %2, 24;\n add.u32 t4, %2, 64;\n"
        " add.u32 t5, %2, 72;\n add.u32 t6, %2, 80;\n add.u32 t7, %2, 88;\n"
        " add.s64 b1, %3, 128;\n add.s64 b2, %3, 256;\n add.s64 b3, %3, 384;\n"
        " add.s64 b5, %4, 128;\n add.s64 b6, %4, 256;\n add.s64 b7, %4, 384;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %3, %5, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t1], b1, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t2], b2, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t3], b3, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%1], [t4], %4, %5, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%1], [t5], b5, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%1], [t6], b6, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%1], [t7], b7, %5, p1;\n}\n" ::"r"(d0),
        "r"(d1), "r"(a_tmem), "l"(bdesc0), "l"(bdesc1), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred p0, p1;\n .reg .b32 t1, t2, t3;\n .reg .b64 b1, b2, b3;\n"
        " setp.ne.b32 p0, %4, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " add.u32 t1, %1, 8;\n add.u32 t2, %1, 16;\n add.u32 t3, %1, 24;\n"
        " add.s64 b1, %2, 128;\n add.s64 b2, %2, 256;\n add.s64 b3, %2, 384;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t1], b1, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t2], b2, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t3], b3, %3, p1;\n}\n" ::"r"(d0),
        "r"(a_tmem), "l"(bdesc0), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// ---------------------------------------------------------------- softmax arithmetic
// Packed fp32 pair operations (Blackwell f32x2 FMA-pipe instructions).
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n .reg .b64 ra, rb;\n mov.b64 ra, {%0, %1};\n mov.b64 rb, {%2, %3};\n add.f32x2 ra, ra, rb;\n"
      " mov.b64 {%0, %1}, ra;\n}\n"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^y for a pair of values on the FMA pipe, to take load off the MUFU unit.
// Range reduction y = j + f with j = round(y) (adding 1.5 * 2^23 leaves the
// integer in the low mantissa bits) and f in [-0.5, 0.5]; 2^f by a degree-3
// polynomial fitted here with the Remez exchange algorithm for minimax
// relative error on [-0.5, 0.5] (max relative error 7.5e-5, far below the
// bf16 resolution P is stored in); 2^j is added into the exponent field.
// y is clamped at -125 so the exponent stays in the normal range.
__device__ __forceinline__ void exp2_poly2(float y0, float y1, float& p0, float& p1) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f, c2 = 0.2426111251115799f,
                  c3 = 0.0551716685295105f;
  y0 = fmaxf(y0, -125.f);
  y1 = fmaxf(y1, -125.f);
  float t0 = y0, t1 = y1;
  add2(t0, t1, kMagic, kMagic);
  float j0 = t0, j1 = t1;
  add2(j0, j1, -kMagic, -kMagic);
  float f0 = y0, f1 = y1;
  add2(f0, f1, -j0, -j1);
  float q0, q1;
  fma2(q0, q1, f0, f1, c3, c3, c2, c2);
  fma2(q0, q1, q0, q1, f0, f1, c1, c1);
  fma2(q0, q1, q0, q1, f0, f1, c0, c0);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// One pass over 64 of a row's S values (raw fp32 bits, one key block):
// p = 2^(x*c - m), packed to bf16 pairs in pk[0..32), accumulated into the
// pair sums s[8]; the raw max is tracked into mv0/mv1 when kTrack is set.
// One pair in four goes through the polynomial, the rest through MUFU ex2.
template <bool kTrack>
__device__ __forceinline__ void exp_half(const uint32_t* x, float c, float m, uint32_t* pk, float (&s)[8],
                                         float& mv0, float& mv1) {
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float x0 = __uint_as_float(x[2 * q]), x1 = __uint_as_float(x[2 * q + 1]);
    if (kTrack) {
      if (q & 1) mv1 = max3f(mv1, x0, x1);
      else mv0 = max3f(mv0, x0, x1);
    }
    float y0, y1, p0, p1;
    fma2(y0, y1, x0, x1, c, c, -m, -m);
    if ((q & 3) == 0) {
      exp2_poly2(y0, y1, p0, p1);
    } else {
      p0 = ex2(y0);
      p1 = ex2(y1);
    }
    add2(s[2 * (q & 3)], s[2 * (q & 3) + 1], p0, p1);
    pk[q] = pack_bf16x2(p0, p1);
  }
}

__device__ __forceinline__ float sum8(const float (&s)[8]) {
  return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

__device__ __forceinline__ float row_max(const uint32_t (&x)[128], bool b0, bool b1) {
  float mv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    if (!(ch < 2 ? b0 : b1)) continue;
#pragma unroll
    for (int q = 0; q < 16; ++q)
      mv[q & 3] = max3f(mv[q & 3], __uint_as_float(x[32 * ch + 2 * q]), __uint_as_float(x[32 * ch + 2 * q + 1]));
  }
  return fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3]));
}

// ---------------------------------------------------------------- kernel
template <int D>
struct AttnSmem {
  static constexpr int kTile = 128 * D * 2;      // 128 rows x D bf16 (a Q tile, or a K / V pair)
  static constexpr int kVBlock = 64 * D * 2;     // one V block, laid out [D/64 chunks][64 keys][128 B]
  static constexpr int kChunk = 128 * 128;       // one 64-column chunk of a 128-row tile
  // K and V live in separate rings: a K stage is free as soon as its S MMA
  // completes, a V stage once its PV MMA does.  Q is double-buffered, so the
  // next item's Q tile lands during the current item (an item boundary no
  // longer waits for it); at d = 128 that takes a K stage: Q 2 + K 2 + V 3
  // tiles of 32 KB = 224 KB (V is read later in a step than K, so it keeps
  // the deeper ring).
  static constexpr int kQBuf = 2;
  static constexpr int kNK = (D == 128) ? 2 : 4;
  static constexpr int kNV = (D == 128) ? 3 : 4;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBuf * kTile;
  static constexpr int kV = kK + kNK * kTile;
  static constexpr int kBar = kV + kNV * kTile;     // mbarriers + flags (512 B)
  static constexpr int kX = kBar + 512;              // softmax pair exchange: [2][4][2][32] floats
  static constexpr int kBytes = kX + 2048;
  // The dynamic shared memory window starts 1 KB-aligned when a kernel has no
  // static shared memory; the slack covers a smaller alignment, and the kernel
  // checks the padding it needs against it before touching anything.
  static constexpr int kAlloc = (kBytes + 1024 <= 232448) ? kBytes + 1024 : 232448;
  static_assert(kBytes <= kAlloc, "dynamic shared memory above the 227 KB per-CTA limit");
};

template <int D, bool kMask>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using S = AttnSmem<D>;
  constexpr int NK = S::kNK, NV = S::kNV, QB = S::kQBuf;
  constexpr uint32_t kTxBlock = 64 * D * 2;  // bytes of one 64-row block
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if (pad + S::kBytes > static_cast<uint32_t>(S::kAlloc)) {  // uniform across the CTA: nothing started yet
    if (threadIdx.x == 0) {
      atomicOr(a.err, kErrSmemAlign);
      if (a.queue && atomicAdd(a.work + 1, 1) == static_cast<int>(gridDim.x) - 1) {  // the last CTA resets the queue
        atomicExch(a.work, 0);
        atomicExch(a.work + 1, 0);
      }
    }
    return;
  }
  uint8_t* sm = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kBar);
  uint64_t* q_full = bars + 0;              // [QB]
  uint64_t* q_empty = bars + 2;             // [QB] after the last S MMA of an item
  uint64_t* s_full = bars + 4;              // [2]
  uint64_t* p_full = bars + 6;              // [2]
  uint64_t* o_final = bars + 9;             // after the last PV of an item
  uint64_t* drain = bars + 10;              // [2] abort path (one per MMA issuer)
  uint64_t* k_full = bars + 12;             // [NK]
  uint64_t* k_empty = k_full + NK;          // [NK] after the S MMA that read the stage
  uint64_t* v_full = k_empty + NK;          // [NV]
  uint64_t* v_empty = v_full + NV;          // [NV] after the PV MMA that read the stage
  uint64_t* pair_l = v_empty + NV;          // [4 quads]: row-sum exchange at the end of an item
  uint64_t* pair_g = pair_l + 4;            // [4 quads]: exchange slot released
  uint64_t* ring_full = pair_g + 4;         // [kRing] the item in the slot is published
  uint64_t* ring_empty = ring_full + kRing; // [kRing] every reader has taken it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring_empty + kRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* ring = reinterpret_cast<int*>(tmem_slot + 2);  // [kRing] item indices

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
    }
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    mbar_init(drain + 1, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], kRingReaders);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&pair_l[i], 2);
      mbar_init(&pair_g[i], 2);
    }
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // the work items come from the planner
  const uint32_t tm = *tmem_slot;
  const int total = a.dense ? a.n_items_host : *reinterpret_cast<const volatile int*>(a.n_items_dev);

  if (warp == 0) {
    // ======================= TMA producer: Q and K =======================
    if (lane == 0) {
      uint32_t g = 0, t = 0;
      int k_phase[NK], q_phase[2] = {-1, -1};
      for (int i = 0; i < NK; ++i) k_phase[i] = -1;
      bool ok = true;
      // The first item of CTA c is item c (no wait on the queue to start); the
      // queue hands out the items after the first G.  Each take is made one
      // item ahead of its use, so the atomic's latency hides behind the
      // current item's loads (a taken index below total is always used).
      const int G = static_cast<int>(gridDim.x);
      int k_next = min(static_cast<int>(blockIdx.x), total);
      for (int r = 0; ok; ++r) {
        int k;
        if (a.queue) {  // publish the item to the other roles
          const int slot = r & (kRing - 1);
          if (r >= kRing && !mbar_wait(&ring_empty[slot], (r / kRing - 1) & 1, abort_flag, a.err, kBackoffNs)) {
            ok = false;
            break;
          }
          k = k_next;
          ring[slot] = k;
          mbar_arrive(&ring_full[slot]);
          if (k < total) k_next = min(G + atomicAdd(a.work, 1), total);
        } else {
          k = min(item_index(r, static_cast<int>(blockIdx.x), G), total);
        }
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        const int qb = t % QB;
        const uint32_t uq = t / QB;
        if (uq >= 1 && !mbar_wait(&q_empty[qb], (uq - 1) & 1, abort_flag, a.err, kBackoffNs)) { ok = false; break; }
        const int row0 = it.bh * a.N, krow0 = kv_head(it.bh, a.H, a.g) * a.N;
        uint8_t* qdst = sm + S::kQ + qb * S::kTile;
        mbar_expect_tx(&q_full[qb], (it.i1 != kNoBlock ? 2u : 1u) * kTxBlock);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_2d(qdst + c * S::kChunk, &tmQ, 64 * c, row0 + 64 * it.i0, &q_full[qb]);
          if (it.i1 != kNoBlock) tma_load_2d(qdst + c * S::kChunk + 8192, &tmQ, 64 * c, row0 + 64 * it.i1, &q_full[qb]);
        }
        q_phase[qb] = uq & 1;
        // union entries are prefetched one step ahead: the TMA coordinates of a
        // step then never wait on a global load
        uint32_t e0n = load_entry(a, it, 0);
        uint32_t e1n = it.len > 1 ? load_entry(a, it, 1) : 0u;
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint32_t e0 = e0n, e1 = nblk == 2 ? e1n : 0u;
          if (2 * s + 2 < it.len) e0n = load_entry(a, it, 2 * s + 2);
          if (2 * s + 3 < it.len) e1n = load_entry(a, it, 2 * s + 3);
          const int j0 = e0 & 0xFFFF, j1 = e1 & 0xFFFF;
          const int kst = g % NK;
          const uint32_t uk = g / NK;
          if (uk >= 1 && !mbar_wait(&k_empty[kst], (uk - 1) & 1, abort_flag, a.err, kBackoffNs)) { ok = false; break; }
          uint8_t* kdst = sm + S::kK + kst * S::kTile;
          mbar_expect_tx(&k_full[kst], nblk * kTxBlock);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(kdst + c * S::kChunk, &tmK, 64 * c, krow0 + 64 * j0, &k_full[kst]);
            if (nblk == 2) tma_load_2d(kdst + c * S::kChunk + 8192, &tmK, 64 * c, krow0 + 64 * j1, &k_full[kst]);
          }
          k_phase[kst] = uk & 1;
        }
        ++t;
      }
      if (!ok || *abort_flag) {
        // Drain: let every load this thread issued land before the CTA exits.
        for (int i = 0; i < NK; ++i)
          if (k_phase[i] >= 0) mbar_wait_drain(&k_full[i], k_phase[i], a.err);
        for (int b = 0; b < QB; ++b)
          if (q_phase[b] >= 0) mbar_wait_drain(&q_full[b], q_phase[b], a.err);
      }
    }
  } else if (warp == 10) {
    // ======================= TMA producer: V =======================
    // A second issuing warp: one thread issues a TMA instruction in about 170
    // cycles, so Q/K and V come from separate warps, and a V block (all of d)
    // is one 3D box.
    if (lane == 0) {
      uint32_t g = 0;
      int v_phase[NV];
      for (int i = 0; i < NV; ++i) v_phase[i] = -1;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        int k = min(item_index(r, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x)), total);
        if (a.queue && !ring_take(r, ring, ring_full, ring_empty, abort_flag, a.err, &k)) { ok = false; break; }
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        const int row0 = kv_head(it.bh, a.H, a.g) * a.N;  // of V
        uint32_t e0n = load_entry(a, it, 0);
        uint32_t e1n = it.len > 1 ? load_entry(a, it, 1) : 0u;
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint32_t e0 = e0n, e1 = nblk == 2 ? e1n : 0u;
          if (2 * s + 2 < it.len) e0n = load_entry(a, it, 2 * s + 2);
          if (2 * s + 3 < it.len) e1n = load_entry(a, it, 2 * s + 3);
          const int vst = g % NV;
          const uint32_t uv = g / NV;
          if (uv >= 1 && !mbar_wait(&v_empty[vst], (uv - 1) & 1, abort_flag, a.err, kBackoffNs)) { ok = false; break; }
          uint8_t* vdst = sm + S::kV + vst * S::kTile;
          mbar_expect_tx(&v_full[vst], nblk * kTxBlock);
          if constexpr (D == 128) {
            tma_load_3d(vdst, &tmV, 0, row0 + 64 * (e0 & 0xFFFF), 0, &v_full[vst]);
            if (nblk == 2) tma_load_3d(vdst + S::kVBlock, &tmV, 0, row0 + 64 * (e1 & 0xFFFF), 0, &v_full[vst]);
          } else {
            tma_load_2d(vdst, &tmV, 0, row0 + 64 * (e0 & 0xFFFF), &v_full[vst]);
            if (nblk == 2) tma_load_2d(vdst + S::kVBlock, &tmV, 0, row0 + 64 * (e1 & 0xFFFF), &v_full[vst]);
          }
          v_phase[vst] = uv & 1;
        }
      }
      if (!ok || *abort_flag) {
        for (int i = 0; i < NV; ++i)
          if (v_phase[i] >= 0) mbar_wait_drain(&v_full[i], v_phase[i], a.err);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer: S = Q K^T =======================
    // S and PV are issued by two warps (a thread that issues MMAs blocks while
    // the tensor core drains them, and one thread doing both serialised the
    // pipeline).  With two issuers the tensor core no longer orders S after
    // PV, so S_g waits for PV_{g-2} to complete before overwriting that
    // S / P buffer: PV_{g-2}'s commit releases V stage (g-2) % NV, and that
    // barrier's older phases are complete because S_{g-1} waited for PV_{g-3}.
    if (lane == 0) {
      uint32_t g = 0, t = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        int k = min(item_index(r, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x)), total);
        if (a.queue && !ring_take(r, ring, ring_full, ring_empty, abort_flag, a.err, &k)) { ok = false; break; }
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        const int qb = t % QB;
        if (!mbar_wait(&q_full[qb], (t / QB) & 1, abort_flag, a.err)) { ok = false; break; }
        const uint64_t adesc = smem_desc_sw128(smem_u32(sm + S::kQ + qb * S::kTile), 16, 1024);
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int kst = g % NK;
          if (!mbar_wait(&k_full[kst], (g / NK) & 1, abort_flag, a.err)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(&v_empty[(g - 2) % NV], ((g - 2) / NV) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm + S::kK + kst * S::kTile), 16, 1024);
          issue_qk<D>(tm + (g & 1) * 128, adesc, bdesc, idesc_bf16_f32(128, 64 * nblk, 0, 0));
          tc_commit(&s_full[g & 1]);
          tc_commit(&k_empty[kst]);  // the S MMA has read the K stage
          if (s == nsteps - 1) tc_commit(&q_empty[qb]);
        }
        ++t;
      }
      if (!ok || *abort_flag) {
        // Drain: wait until every MMA this thread issued has completed.
        tc_commit(drain);
        mbar_wait_drain(drain, 0, a.err);
      }
    }
  } else if (warp == 11) {
    // ======================= MMA issuer: O_c += P_c V_c =======================
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      uint32_t g = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        int k = min(item_index(r, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x)), total);
        if (a.queue && !ring_take(r, ring, ring_full, ring_empty, abort_flag, a.err, &k)) { ok = false; break; }
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int vst = g % NV;
          if (!mbar_wait(&p_full[g & 1], (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
          if (!mbar_wait(&v_full[vst], (g / NV) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint32_t vaddr = smem_u32(sm + S::kV + vst * S::kTile);
          const uint64_t bdesc0 = smem_desc_sw128(vaddr, 64 * 128, 1024);  // LBO: next 64-column chunk of d
          const uint64_t bdesc1 = smem_desc_sw128(vaddr + S::kVBlock, 64 * 128, 1024);
          issue_pv(tm + 256, tm + 384, tm + (g & 1) * 128, bdesc0, bdesc1, idesc_pv, s > 0 ? 1u : 0u, nblk);
          tc_commit(&v_empty[vst]);  // V stage free; PV_g complete (S_{g+2} and O rescales wait on it)
          if (s == nsteps - 1) tc_commit(o_final);
        }
      }
      if (!ok || *abort_flag) {
        tc_commit(drain + 1);
        mbar_wait_drain(drain + 1, 0, a.err);
      }
    }
  } else {
    // ======================= softmax / epilogue (warps 2..9) =======================
    // Two warps per TMEM lane quadrant: warp (quad, cb) owns the 32 tile rows
    // of its quadrant and key block cb of every step (S columns 64*cb ..,
    // P columns 64*cb .. 64*cb+31, accumulator O_cb at TMEM column 256 + 128*cb).  Each
    // runs its own online softmax (running max m, sum l) with no per-step
    // synchronisation; the two partial results of a row are merged once per
    // item in the epilogue:  O = (w0 O_0 + w1 O_1) / (w0 l_0 + w1 l_1),
    // w_c = 2^(m_c - max(m_0, m_1)).
    const int sw = warp - 2;                   // 0..7
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int cb = sw >> 2;                    // key block of the step this warp handles
    const int row = quad * 32 + lane;          // tile row = TMEM lane
    const int half = row >> 6;                 // 0: query block i0, 1: i1
    const uint32_t t_lane = tm + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t o_own = t_lane + 256 + 128 * cb;
    constexpr int DH = D / 2;                  // output columns this warp writes
    float* xbuf = reinterpret_cast<float*>(sm + S::kX);  // [4 quads][2 warps][2 values][32 lanes]
    const float c = a.scale_log2;
    uint32_t g = 0, t = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      int k = min(item_index(r, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x)), total);
      if (a.queue) {  // every softmax warp reads the ring; each releases the slot once
        const int slot = r & (kRing - 1);
        if (!warp_wait(&ring_full[slot], (r / kRing) & 1, abort_flag, a.err)) { ok = false; break; }
        k = ring[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&ring_empty[slot]);
      }
      if (k >= total) break;
      const Item it = load_item(a, k);
      const int nsteps = (it.len + 1) >> 1;
      const int qblk = half ? it.i1 : it.i0;
      const bool row_valid = qblk != kNoBlock;
      __nv_bfloat16* orow =
          a.O + (static_cast<size_t>(it.bh) * a.N + static_cast<size_t>(qblk) * 64 + (row & 63)) * D + cb * DH;
      if (nsteps == 0) {
        if (row_valid) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int q = 0; q < DH / 8; ++q) reinterpret_cast<uint4*>(orow)[q] = z;
        }
        continue;
      }
      float m = -INFINITY, l = 0.f;
      // this warp's union entry per step, prefetched one step ahead
      uint32_t en = cb < it.len ? load_entry(a, it, cb) : 0u;
      unsigned long long wn = cb < it.len ? key_word<kMask>(a, it.bh, en) : ~0ull;  // its key mask word, likewise
      for (int s = 0; s < nsteps; ++s, ++g) {
        const int sb = g & 1;
        const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
        const bool present = cb < nblk;        // this warp's key block exists in the step
        const uint32_t e = present ? en : 0u;
        const unsigned long long wm = wn;
        if (2 * s + 2 + cb < it.len) {
          en = load_entry(a, it, 2 * s + 2 + cb);
          wn = key_word<kMask>(a, it.bh, en);
        }
        if (!warp_wait(&s_full[sb], (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        // this half's query block selected the key block, and the key mask leaves some of its keys
        const bool bm = ((e >> (16 + half)) & 1u) && wm != 0ull;
        uint32_t pk[32];
        float alpha = 1.f, sum = 0.f;
        bool rescale = false;
        if (bm) {
          uint32_t x[64];
          const uint32_t s_col = t_lane + sb * 128 + cb * 64;
          tmem_ld32(s_col, x);
          tmem_ld32(s_col + 32, x + 32);
          tmem_wait_ld();
          const bool partial = wm != ~0ull;  // the same for every row of the warp
          if (partial) {  // masked keys take no part in the max and get probability 0
#pragma unroll
            for (int q = 0; q < 64; ++q)
              if (!((wm >> q) & 1ull)) x[q] = 0xFF800000u;  // -inf
          }
          float mv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int q = 0; q < 32; ++q)
            mv[q & 3] = max3f(mv[q & 3], __uint_as_float(x[2 * q]), __uint_as_float(x[2 * q + 1]));
          const float mx = fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])) * c;  // c > 0
          // Running max: set by the first selected block, raised again only
          // when it grows by more than 2^8 (then O_cb is rescaled); otherwise
          // the stale max is kept (exact after the final division by the sum).
          {  // as selects (no per-row branch): the exponential is taken in every row
            const bool first = m == -INFINITY;
            const bool grow = !first && mx > m + kRescaleThreshold;
            const float a_ = ex2(m - mx);
            alpha = grow ? a_ : 1.f;
            rescale = grow;
            m = (first || grow) ? mx : m;
          }
          float sv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          float mv0 = 0.f, mv1 = 0.f;
          exp_half<false>(x, c, m, pk, sv, mv0, mv1);
          if (partial) {  // exactly 0 for masked keys (the polynomial path floors 2^y at 2^-125)
#pragma unroll
            for (int q = 0; q < 32; ++q)
              pk[q] &= (((wm >> (2 * q)) & 1ull) ? 0x0000FFFFu : 0u) | (((wm >> (2 * q + 1)) & 1ull) ? 0xFFFF0000u : 0u);
          }
          sum = sum8(sv);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) pk[q] = 0u;
        }
        l = l * alpha + sum;
        if (__any_sync(0xffffffffu, rescale)) {
          // O_cb holds PV results up to step g-1: wait for PV_{g-1} (its commit
          // releases V stage (g-1) % NV; that barrier's earlier phases are
          // complete because S_g, issued after PV_{g-2}, is), then scale.
          if (!warp_wait(&v_empty[(g - 1) % NV], ((g - 1) / NV) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t o[32];
            tmem_ld32(o_own + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(o_own + cc, o);
          }
        }
        // P of this key block (bf16 pairs) over the first half of the block's own
        // S columns, which only this warp reads: no race with the partner warp.
        if (present) tmem_st32(t_lane + sb * 128 + cb * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;
      // epilogue: merge the two partial results of each row, O -> bf16 -> global
      float* xm = xbuf + (quad * 2) * 64;        // [2 warps][m, l][32]
      xm[cb * 64 + lane] = m;
      xm[cb * 64 + 32 + lane] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&pair_l[quad]);
      if (!warp_wait(&pair_l[quad], t & 1, abort_flag, a.err)) { ok = false; break; }
      const float m_o = xm[(1 - cb) * 64 + lane], l_o = xm[(1 - cb) * 64 + 32 + lane];
      __syncwarp();
      if (lane == 0) mbar_arrive(&pair_g[quad]);  // both read: the slot may be written again
      if (!warp_wait(&pair_g[quad], t & 1, abort_flag, a.err)) { ok = false; break; }
      const float m0 = cb ? m_o : m, l0 = cb ? l_o : l, m1 = cb ? m : m_o, l1 = cb ? l : l_o;
      const bool o1_valid = it.len >= 2;         // O_1 is only written when a step has two blocks
      const float mmax = fmaxf(m0, o1_valid ? m1 : -INFINITY);
      const float w0 = l0 > 0.f ? ex2(m0 - mmax) : 0.f;
      const float w1 = (o1_valid && l1 > 0.f) ? ex2(m1 - mmax) : 0.f;
      const float lt = w0 * l0 + w1 * l1;
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float f0 = w0 * inv, f1 = w1 * inv;
      const bool any_w1 = __any_sync(0xffffffffu, w1 != 0.f);
      if (!warp_wait(o_final, t & 1, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < DH; cc += 32) {
        uint32_t o0[32], o1[32];
        tmem_ld32(t_lane + 256 + cb * DH + cc, o0);
        if (o1_valid) tmem_ld32(t_lane + 384 + cb * DH + cc, o1);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = __uint_as_float(o0[q]) * f0;
        if (any_w1) {  // rows with w1 == 0 never read O_1 (it may be stale when unused)
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = (w1 != 0.f) ? fmaf(__uint_as_float(o1[q]), f1, v[q]) : v[q];
        }
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
            u.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
            u.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
            u.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
            dst[q] = u;
          }
        }
      }
      tc_fence_before();
      ++t;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (a.queue && threadIdx.x == 0) {
    __threadfence();  // this CTA's takes from the queue come before its count
    if (atomicAdd(a.work + 1, 1) == static_cast<int>(gridDim.x) - 1) {  // the last CTA resets the queue
      atomicExch(a.work, 0);
      atomicExch(a.work + 1, 0);
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// Packs a key mask of bytes, [B][N] (nonzero = may be attended), into one
// 64-bit word per (batch, key block): bit r for key 64 j + r.  One thread per
// word, four 16-byte loads each.
__global__ void key_mask_words_kernel(const uint8_t* __restrict__ km, unsigned long long* __restrict__ words,
                                      int n_words) {
  grid_dep_wait();
  const int w = blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= n_words) return;
  const uint4* src = reinterpret_cast<const uint4*>(km + static_cast<size_t>(w) * 64);
  unsigned long long bits = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 u = __ldg(src + v);
    const uint32_t parts[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if ((parts[p] >> (8 * b)) & 0xFFu) bits |= 1ull << (16 * v + 4 * p + b);
  }
  words[w] = bits;
}

// Zero output for skipped heads.
__global__ void zero_heads_kernel(__nv_bfloat16* __restrict__ O, int BH, int H, uint64_t head_bits,
                                  size_t per_head_vec) {
  const int bh = blockIdx.y;
  if ((head_bits >> (bh % H)) & 1ull) return;
  uint4* dst = reinterpret_cast<uint4*>(O) + static_cast<size_t>(bh) * per_head_vec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < per_head_vec;
       e += static_cast<size_t>(gridDim.x) * blockDim.x)
    dst[e] = z;
}

// Diagnostic: the polynomial exp2 used for one in four softmax exponentials.
__global__ void exp2_poly_kernel(const float* __restrict__ y, float* __restrict__ out, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    exp2_poly2(y[i], y[i + 1], out[i], out[i + 1]);
  } else if (i < n) {
    float dummy;
    exp2_poly2(y[i], 0.f, out[i], dummy);
  }
}

cudaError_t launch_exp2_poly(const float* y, float* out, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, s>>>(y, out, n);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2D view [rows = B*H*N][d] bf16, 64 x 64 boxes, 128-byte swizzle.
// 3D view of V for d = 128: (64 columns, rows, 2 chunks of 64 columns), box
// 64 x 64 x 2, so one TMA instruction moves a whole 64-row block laid out as
// [chunk][64 rows][128 B] with 128-byte swizzle.
static bool make_map_v3(CUtensorMap* map, const void* base, size_t rows, int d) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(d / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, 128};
  cuuint32_t box[3] = {64, 64, static_cast<cuuint32_t>(d / 64)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static bool make_map(CUtensorMap* map, const void* base, size_t rows, int d) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kMask>
static cudaError_t launch_attn_kernel(const void* Q, const void* K, const void* V, int BH, int BHkv, int N,
                                      const AttnArgs& args, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const size_t rows = static_cast<size_t>(BH) * N, kv_rows = static_cast<size_t>(BHkv) * N;
  const bool v_ok = (D == 128) ? make_map_v3(&mv, V, kv_rows, D) : make_map(&mv, V, kv_rows, D);
  if (!make_map(&mq, Q, rows, D) || !make_map(&mk, K, kv_rows, D) || !v_ok) return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  static int configured_dev_mask = 0;
  if (!(configured_dev_mask & (1 << (di.id & 31)))) {
    e = cudaFuncSetAttribute(sparse_attn_kernel<D, kMask>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnSmem<D>::kAlloc);
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << (di.id & 31);
  }
  return launch_pdl(sparse_attn_kernel<D, kMask>, dim3(di.sm_count), dim3(kThreads), AttnSmem<D>::kAlloc, s, mq, mk,
                    mv, args);
}

static cudaError_t launch_attn(const void* Q, const void* K, const void* V, int BH, int BHkv, int N, int d,
                               const AttnArgs& args, cudaStream_t s) {
  if (args.kmask) {
    if (d == 128) return launch_attn_kernel<128, true>(Q, K, V, BH, BHkv, N, args, s);
    return launch_attn_kernel<64, true>(Q, K, V, BH, BHkv, N, args, s);
  }
  if (d == 128) return launch_attn_kernel<128, false>(Q, K, V, BH, BHkv, N, args, s);
  return launch_attn_kernel<64, false>(Q, K, V, BH, BHkv, N, args, s);
}

// The queue pays off from about 8 items per CTA (measured on the joint and
// video workloads, 21 and 42 items per CTA: 4 % faster); below that (SDXL,
// one layer of the stack: 3-5 items per CTA) the static deal is faster.
int use_queue(long long items) {
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return 1;
  return items >= 8ll * di.sm_count ? 1 : 0;
}

cudaError_t launch_attention_run(const void* Q, const void* K, const void* V, int B, int H, int Hkv, int N, int d,
                                 const uint8_t* key_mask, uint64_t head_bits, float scale, void* O, void* ws,
                                 cudaStream_t s) {
  const int BH = B * H, nB = N / kBlock;
  const WsLayout wl = ws_layout(B, H, N, d);
  char* base = static_cast<char*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base + wl.header);
  unsigned long long* kmask = nullptr;
  if (key_mask) {
    kmask = reinterpret_cast<unsigned long long*>(base + wl.kmask);
    const int n_words = B * nB;
    cudaError_t e = launch_pdl(key_mask_words_kernel, dim3((n_words + 127) / 128), dim3(128), 0, s, key_mask,
                               kmask, n_words);
    if (e != cudaSuccess) return e;
  }
  const uint64_t all = (H >= 64) ? ~0ull : ((1ull << H) - 1ull);
  if ((head_bits & all) != all) {
    const size_t per_head_vec = static_cast<size_t>(N) * d / 8;
    zero_heads_kernel<<<dim3(64, BH), 256, 0, s>>>(static_cast<__nv_bfloat16*>(O), BH, H, head_bits, per_head_vec);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  AttnArgs args{};
  args.items = reinterpret_cast<const int4*>(base + wl.items);
  args.ulist = reinterpret_cast<const int32_t*>(base + wl.ulist);
  args.n_items_dev = &hdr->n_items;
  args.n_items_host = 0;
  args.dense = 0;
  args.N = N;
  args.nB = nB;
  args.npairs_dense = (nB + 1) / 2;
  args.H = H;
  args.g = H / Hkv;
  args.O = static_cast<__nv_bfloat16*>(O);
  args.scale_log2 = scale * 1.4426950408889634f;
  args.err = &hdr->err;
  args.kmask = kmask;
  args.work = &hdr->next_item;
  args.queue = use_queue(B * __builtin_popcountll(head_bits & all) * args.npairs_dense);
  return launch_attn(Q, K, V, BH, B * Hkv, N, d, args, s);
}

cudaError_t launch_dense_attention(const void* Q, const void* K, const void* V, int B, int H, int Hkv, int N,
                                   int d, float scale, void* O, void* ws, cudaStream_t s) {
  const int BH = B * H, nB = N / kBlock;
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  AttnArgs args{};
  args.items = nullptr;
  args.ulist = nullptr;
  args.n_items_dev = nullptr;
  args.npairs_dense = (nB + 1) / 2;
  args.n_items_host = BH * args.npairs_dense;
  args.dense = 1;
  args.N = N;
  args.nB = nB;
  args.H = H;
  args.g = H / Hkv;
  args.O = static_cast<__nv_bfloat16*>(O);
  args.scale_log2 = scale * 1.4426950408889634f;
  args.err = &hdr->err;
  args.work = &hdr->next_item;
  args.queue = use_queue(args.n_items_host);
  return launch_attn(Q, K, V, BH, B * Hkv, N, d, args, s);
}

}  // namespace sa
