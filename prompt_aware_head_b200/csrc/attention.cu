// Flash-style attention over selected (query block, key block) tiles on
// sm_100a: tcgen05 MMA with TMEM accumulators, TMA-staged K/V tiles gathered
// through the block lists, a persistent CTA per SM.
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
//  * Warp roles: warp 0 TMA producer, warp 1 MMA issuer (one thread), warps
//    2-5 softmax / correction / epilogue (one thread per tile row).
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
  __nv_bfloat16* O;
  float scale_log2;
  int* err;
};

constexpr int kThreads = 192;
constexpr int kNoBlock = 0xFFFF;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows by > 2^8

struct Item {
  int bh, i0, i1, len, off;
};

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
  return it;
}

// Union entry e of an item: key block j in the low 16 bits, membership bits
// (bit 16: query block i0 selected j, bit 17: i1 selected j).
__device__ __forceinline__ uint32_t load_entry(const AttnArgs& a, const Item& it, int e) {
  if (a.dense) return static_cast<uint32_t>(e) | ((it.i1 == kNoBlock ? 1u : 3u) << 16);
  return static_cast<uint32_t>(a.ulist[it.off + e]);
}

__device__ __forceinline__ int item_index(int r, int cta, int G) {
  return r * G + ((r & 1) ? (G - 1 - cta) : cta);  // boustrophedon over the CTAs
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

// O += P V for one step of 64 * nblk keys: A = P (bf16 in TMEM, 8 columns
// per 16 keys), B = V pair (MN-major SW128 smem; 16 keys = 2 KB per slice).
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate, int nblk) {
  if (nblk == 2) {
    asm volatile(
        "{\n .reg .pred p0, p1;\n .reg .b32 t1, t2, t3, t4, t5, t6, t7;\n"
        " .reg .b64 b1, b2, b3, b4, b5, b6, b7;\n"
        " setp.ne.b32 p0, %4, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " add.u32 t1, %1, 8;\n add.u32 t2, %1, 16;\n add.u32 t3, %1, 24;\n add.u32 t4, %1, 32;\n"
        " add.u32 t5, %1, 40;\n add.u32 t6, %1, 48;\n add.u32 t7, %1, 56;\n"
        " add.s64 b1, %2, 128;\n add.s64 b2, %2, 256;\n add.s64 b3, %2, 384;\n add.s64 b4, %2, 512;\n"
        " add.s64 b5, %2, 640;\n add.s64 b6, %2, 768;\n add.s64 b7, %2, 896;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t1], b1, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t2], b2, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t3], b3, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t4], b4, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t5], b5, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t6], b6, %3, p1;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t7], b7, %3, p1;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
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
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [t3], b3, %3, p1;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// ---------------------------------------------------------------- kernel
template <int D>
struct AttnSmem {
  static constexpr int kTile = 128 * D * 2;      // 128 rows x D bf16
  static constexpr int kChunk = 128 * 128;       // one 64-column chunk of a 128-row tile
  static constexpr int kStages = (D == 128) ? 2 : 4;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kBytes = kBar + 1024;     // barriers + flags
  static constexpr int kAlloc = kBytes + 1024;   // slack for 1024-B alignment
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
  using S = AttnSmem<D>;
  constexpr int NST = S::kStages;
  constexpr uint32_t kTxBlock = 64 * D * 2;  // bytes of one 64-row block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kBar);
  uint64_t* q_full = bars + 0;              // [2]
  uint64_t* q_empty = bars + 2;             // [2]
  uint64_t* s_full = bars + 4;              // [2]
  uint64_t* p_full = bars + 6;              // [2]
  uint64_t* o_done = bars + 8;              // after every PV
  uint64_t* o_final = bars + 9;             // after the last PV of an item
  uint64_t* drain = bars + 10;              // abort path
  uint64_t* k_full = bars + 12;             // [NST]
  uint64_t* v_full = k_full + NST;          // [NST]
  uint64_t* kv_empty = v_full + NST;        // [NST]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kv_empty + NST);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
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
  const uint32_t tm = *tmem_slot;
  const int G = gridDim.x, cta = blockIdx.x;
  const int total = a.dense ? a.n_items_host : *reinterpret_cast<const volatile int*>(a.n_items_dev);

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      uint32_t g = 0, t = 0;
      int ld_phase[NST];
      int q_phase[2] = {-1, -1};
      for (int s = 0; s < NST; ++s) ld_phase[s] = -1;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int k = item_index(r, cta, G);
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        const int qb = t & 1;
        if (t >= 2 && !mbar_wait(&q_empty[qb], ((t >> 1) - 1) & 1, abort_flag, a.err)) { ok = false; break; }
        const int row0 = it.bh * a.N;
        uint8_t* qdst = sm + S::kQ + qb * S::kTile;
        mbar_expect_tx(&q_full[qb], (it.i1 != kNoBlock ? 2u : 1u) * kTxBlock);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_2d(qdst + c * S::kChunk, &tmQ, 64 * c, row0 + 64 * it.i0, &q_full[qb]);
          if (it.i1 != kNoBlock) tma_load_2d(qdst + c * S::kChunk + 8192, &tmQ, 64 * c, row0 + 64 * it.i1, &q_full[qb]);
        }
        q_phase[qb] = (t >> 1) & 1;
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int st = g % NST;
          const uint32_t u = g / NST;
          if (u >= 1 && !mbar_wait(&kv_empty[st], (u - 1) & 1, abort_flag, a.err)) { ok = false; break; }
          const uint32_t e0 = load_entry(a, it, 2 * s);
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint32_t e1 = nblk == 2 ? load_entry(a, it, 2 * s + 1) : 0u;
          const int j0 = e0 & 0xFFFF, j1 = e1 & 0xFFFF;
          uint8_t* kdst = sm + S::kK + st * S::kTile;
          uint8_t* vdst = sm + S::kV + st * S::kTile;
          mbar_expect_tx(&k_full[st], nblk * kTxBlock);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(kdst + c * S::kChunk, &tmK, 64 * c, row0 + 64 * j0, &k_full[st]);
            if (nblk == 2) tma_load_2d(kdst + c * S::kChunk + 8192, &tmK, 64 * c, row0 + 64 * j1, &k_full[st]);
          }
          mbar_expect_tx(&v_full[st], nblk * kTxBlock);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_2d(vdst + c * S::kChunk, &tmV, 64 * c, row0 + 64 * j0, &v_full[st]);
            if (nblk == 2) tma_load_2d(vdst + c * S::kChunk + 8192, &tmV, 64 * c, row0 + 64 * j1, &v_full[st]);
          }
          ld_phase[st] = u & 1;
        }
        ++t;
      }
      if (!ok || *abort_flag) {
        // Drain: let every load this thread issued land before the CTA exits.
        for (int s = 0; s < NST; ++s)
          if (ld_phase[s] >= 0) {
            mbar_wait_drain(&k_full[s], ld_phase[s], a.err);
            mbar_wait_drain(&v_full[s], ld_phase[s], a.err);
          }
        for (int b = 0; b < 2; ++b)
          if (q_phase[b] >= 0) mbar_wait_drain(&q_full[b], q_phase[b], a.err);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      uint32_t g = 0, t = 0;
      bool ok = true, have_pend = false;
      uint32_t pg = 0, pst = 0, pacc = 0, plast = 0;
      int pnblk = 0;
      auto do_pv = [&]() -> bool {
        if (!mbar_wait(&p_full[pg & 1], (pg >> 1) & 1, abort_flag, a.err)) return false;
        if (!mbar_wait(&v_full[pst], (pg / NST) & 1, abort_flag, a.err)) return false;
        tc_fence_after();
        const uint64_t bdesc = smem_desc_sw128(smem_u32(sm + S::kV + pst * S::kTile), S::kChunk, 1024);
        issue_pv(tm + 256, tm + (pg & 1) * 128, bdesc, idesc_pv, pacc, pnblk);
        tc_commit(&kv_empty[pst]);
        tc_commit(o_done);
        if (plast) tc_commit(o_final);
        return true;
      };
      for (int r = 0; ok; ++r) {
        const int k = item_index(r, cta, G);
        if (k >= total) break;
        const Item it = load_item(a, k);
        const int nsteps = (it.len + 1) >> 1;
        if (nsteps == 0) continue;
        const int qb = t & 1;
        if (!mbar_wait(&q_full[qb], (t >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
        const uint64_t adesc = smem_desc_sw128(smem_u32(sm + S::kQ + qb * S::kTile), 16, 1024);
        for (int s = 0; s < nsteps; ++s, ++g) {
          const int st = g % NST;
          if (!mbar_wait(&k_full[st], (g / NST) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sm + S::kK + st * S::kTile), 16, 1024);
          issue_qk<D>(tm + (g & 1) * 128, adesc, bdesc, idesc_bf16_f32(128, 64 * nblk, 0, 0));
          tc_commit(&s_full[g & 1]);
          if (s == nsteps - 1) tc_commit(&q_empty[qb]);
          if (have_pend && !do_pv()) { ok = false; break; }
          have_pend = true;
          pg = g;
          pst = st;
          pnblk = nblk;
          pacc = s > 0 ? 1u : 0u;
          plast = (s == nsteps - 1) ? 1u : 0u;
        }
        ++t;
      }
      if (ok && have_pend && !do_pv()) ok = false;
      if (!ok || *abort_flag) {
        // Drain: wait until every MMA this thread issued has completed.
        tc_commit(drain);
        mbar_wait_drain(drain, 0, a.err);
      }
    }
  } else {
    // ======================= softmax / epilogue (warps 2..5) =======================
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;          // tile row = TMEM lane
    const int half = row >> 6;                 // 0: query block i0, 1: i1
    const uint32_t t_lane = tm + (static_cast<uint32_t>(quad * 32) << 16);
    const float c = a.scale_log2;
    uint32_t g = 0, t = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = item_index(r, cta, G);
      if (k >= total) break;
      const Item it = load_item(a, k);
      const int nsteps = (it.len + 1) >> 1;
      const int qblk = half ? it.i1 : it.i0;
      const bool row_valid = qblk != kNoBlock;
      __nv_bfloat16* orow = a.O + (static_cast<size_t>(it.bh) * a.N + static_cast<size_t>(qblk) * 64 + (row & 63)) * D;
      if (nsteps == 0) {
        if (row_valid) {
          uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int q = 0; q < D / 8; ++q) reinterpret_cast<uint4*>(orow)[q] = z;
        }
        continue;
      }
      float m = -INFINITY, l = 0.f;
      for (int s = 0; s < nsteps; ++s, ++g) {
        const int sb = g & 1;
        if (!warp_wait(&s_full[sb], (g >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const int nblk = (2 * s + 1 < it.len) ? 2 : 1;
        const uint32_t e0 = load_entry(a, it, 2 * s);
        const uint32_t e1 = nblk == 2 ? load_entry(a, it, 2 * s + 1) : 0u;
        const bool b0 = (e0 >> (16 + half)) & 1u;
        const bool b1 = (e1 >> (16 + half)) & 1u;
        const uint32_t s_col = t_lane + sb * 128;
        uint32_t x[128];
        if (b0) {
          tmem_ld32(s_col, x);
          tmem_ld32(s_col + 32, x + 32);
        }
        if (b1) {
          tmem_ld32(s_col + 64, x + 64);
          tmem_ld32(s_col + 96, x + 96);
        }
        if (b0 || b1) tmem_wait_ld();
        float mx = -INFINITY;
        if (b0) {
#pragma unroll
          for (int q = 0; q < 64; ++q) mx = fmaxf(mx, __uint_as_float(x[q]));
        }
        if (b1) {
#pragma unroll
          for (int q = 64; q < 128; ++q) mx = fmaxf(mx, __uint_as_float(x[q]));
        }
        mx *= c;  // c > 0: max commutes with the scaling
        const float m_new = fmaxf(m, mx);
        float m_use = m, alpha = 1.f;
        bool rescale = false;
        if (m == -INFINITY) {
          m_use = m_new;
        } else if (m_new - m > kRescaleThreshold) {
          m_use = m_new;
          alpha = ex2(m - m_new);
          rescale = true;
        }
        float sum = 0.f;
        uint32_t pk[64];
        if (b0) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const float p0 = ex2(fmaf(__uint_as_float(x[2 * q]), c, -m_use));
            const float p1 = ex2(fmaf(__uint_as_float(x[2 * q + 1]), c, -m_use));
            sum += p0 + p1;
            pk[q] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) pk[q] = 0u;
        }
        if (b1) {
#pragma unroll
          for (int q = 32; q < 64; ++q) {
            const float p0 = ex2(fmaf(__uint_as_float(x[2 * q]), c, -m_use));
            const float p1 = ex2(fmaf(__uint_as_float(x[2 * q + 1]), c, -m_use));
            sum += p0 + p1;
            pk[q] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int q = 32; q < 64; ++q) pk[q] = 0u;
        }
        l = l * alpha + sum;
        m = m_use;
        if (__any_sync(0xffffffffu, rescale)) {
          // O (TMEM) holds PV results up to step g-1: wait for PV_{g-1}, then scale.
          if (!warp_wait(o_done, (g - 1) & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t o[32];
            tmem_ld32(t_lane + 256 + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
            tmem_st32(t_lane + 256 + cc, o);
          }
        }
        tmem_st32(s_col, pk);
        if (nblk == 2) tmem_st32(s_col + 32, pk + 32);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16 -> global
      if (!warp_wait(o_final, t & 1, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t o[32];
        tmem_ld32(t_lane + 256 + cc, o);
        tmem_wait_ld();
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            dst[q] = v;
          }
        }
      }
      tc_fence_before();
      ++t;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// ---------------------------------------------------------------- planner
// One CTA per head (b, h).  Picks the pairing stride s in {1, 2, 4} that
// minimises the summed union length, builds every pair's sorted union list
// with membership bits, and orders the pairs by union length (longest
// first) for the persistent kernel.  Validates every block index.
constexpr int kPlanThreads = 512;

__device__ __forceinline__ int pair_partner(int a, int s, int nB) {
  return (a + s < nB) ? a + s : -1;
}

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ counts, int nB, int cap,
                                                            int H, uint64_t head_bits, int4* __restrict__ head_items,
                                                            int* __restrict__ head_np, int32_t* __restrict__ ulist,
                                                            int* __restrict__ err) {
  __shared__ uint32_t bm[kPlanThreads / 32][2][kMaxBlocks / 32];
  __shared__ int lens[kMaxBlocks];
  __shared__ uint32_t keys[kMaxBlocks];
  __shared__ int totals[3];
  __shared__ int s_best;
  const int bh = blockIdx.x, t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int nw = kPlanThreads / 32, nwords = (nB + 31) / 32;
  if (!((head_bits >> (bh % H)) & 1ull)) {
    if (t == 0) head_np[bh] = 0;
    return;
  }
  if (t < 3) totals[t] = 0;
  __syncthreads();
  // Marks the lists of query blocks a and b (b < 0: none) in this warp's bitmaps.
  auto mark = [&](int a, int b) {
    for (int q = lane; q < kMaxBlocks / 32; q += 32) {
      bm[w][0][q] = 0u;
      bm[w][1][q] = 0u;
    }
    __syncwarp();
    for (int side = 0; side < 2; ++side) {
      const int qb = side ? b : a;
      if (qb < 0) continue;
      int cnt = counts[static_cast<size_t>(bh) * nB + qb];
      if (cnt > cap || cnt < 0) {
        if (lane == 0) atomicOr(err, kErrBadIndex);
        cnt = cnt < 0 ? 0 : cap;
      }
      const int32_t* lst = idx + (static_cast<size_t>(bh) * nB + qb) * cap;
      for (int e = lane; e < cnt; e += 32) {
        const int j = lst[e];
        if (j < 0 || j >= nB) {
          atomicOr(err, kErrBadIndex);
          continue;
        }
        atomicOr(&bm[w][side][j >> 5], 1u << (j & 31));
      }
    }
    __syncwarp();
  };
  const int strides[3] = {1, 2, 4};
  for (int si = 0; si < 3; ++si) {
    const int s = strides[si];
    int local = 0;
    for (int a = w; a < nB; a += nw) {
      if ((a / s) & 1) continue;
      mark(a, pair_partner(a, s, nB));
      int u = 0;
      for (int q = lane; q < nwords; q += 32) u += __popc(bm[w][0][q] | bm[w][1][q]);
      local += __reduce_add_sync(0xffffffffu, u);
      __syncwarp();
    }
    if (lane == 0) atomicAdd(&totals[si], local);
  }
  __syncthreads();
  if (t == 0) {
    int best = 0;
    for (int si = 1; si < 3; ++si)
      if (totals[si] < totals[best]) best = si;
    s_best = strides[best];
  }
  __syncthreads();
  const int s = s_best;
  for (int a = t; a < kMaxBlocks; a += kPlanThreads) keys[a] = 0xFFFFFFFFu;
  __syncthreads();
  for (int a = w; a < nB; a += nw) {
    if ((a / s) & 1) continue;
    const int b = pair_partner(a, s, nB);
    mark(a, b);
    // compaction: lane q owns bitmap word q (blocks 32q .. 32q+31), ascending
    int base = 0;
    int32_t* out = ulist + (static_cast<size_t>(bh) * nB + a) * nB;
    for (int q0 = 0; q0 < nwords; q0 += 32) {
      const int q = q0 + lane;
      const uint32_t wa = q < nwords ? bm[w][0][q] : 0u;
      const uint32_t wb = q < nwords ? bm[w][1][q] : 0u;
      uint32_t un = wa | wb;
      const int cnt = __popc(un);
      int incl = cnt;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = base + incl - cnt;
      while (un) {
        const int bit = __ffs(un) - 1;
        un &= un - 1;
        const uint32_t mbits = ((wa >> bit) & 1u) | (((wb >> bit) & 1u) << 1);
        out[pos++] = static_cast<int32_t>((32 * q + bit) | (mbits << 16));
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      lens[a] = base;
      keys[a] = (static_cast<uint32_t>(0xFFFF - base) << 16) | static_cast<uint32_t>(a);
    }
    __syncwarp();
  }
  __syncthreads();
  // bitonic sort of keys ascending (= union length descending, then a ascending)
  for (int size = 2; size <= kMaxBlocks; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int e = t; e < kMaxBlocks; e += kPlanThreads) {
        const int p = e ^ stride;
        if (p > e) {
          const bool up = (e & size) == 0;
          const uint32_t x = keys[e], y = keys[p];
          if ((x > y) == up) {
            keys[e] = y;
            keys[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  int np = 0;
  for (int a = 0; a < nB; ++a) np += ((a / s) & 1) ? 0 : 1;
  for (int r = t; r < np; r += kPlanThreads) {
    const int a = static_cast<int>(keys[r] & 0xFFFFu);
    const int b = pair_partner(a, s, nB);
    int4 v;
    v.x = bh;
    v.y = a | ((b < 0 ? kNoBlock : b) << 16);
    v.z = lens[a];
    v.w = static_cast<int>((static_cast<size_t>(bh) * nB + a) * nB);
    head_items[static_cast<size_t>(bh) * nB + r] = v;
  }
  if (t == 0) head_np[bh] = np;
}

// Concatenates the per-head item lists in head order (one CTA).
__global__ void __launch_bounds__(1024) compact_items_kernel(const int4* __restrict__ head_items,
                                                             const int* __restrict__ head_np, int BH, int nB,
                                                             int4* __restrict__ items, int* __restrict__ n_items) {
  __shared__ int base_s;
  if (threadIdx.x == 0) base_s = 0;
  __syncthreads();
  for (int bh = 0; bh < BH; ++bh) {
    const int np = head_np[bh];
    const int base = base_s;
    for (int r = threadIdx.x; r < np; r += blockDim.x) items[base + r] = head_items[static_cast<size_t>(bh) * nB + r];
    __syncthreads();
    if (threadIdx.x == 0) base_s = base + np;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_items = base_s;
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

template <int D>
static cudaError_t launch_attn_kernel(const void* Q, const void* K, const void* V, int BH, int N,
                                      const AttnArgs& args, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const size_t rows = static_cast<size_t>(BH) * N;
  if (!make_map(&mq, Q, rows, D) || !make_map(&mk, K, rows, D) || !make_map(&mv, V, rows, D))
    return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  static int configured_dev_mask = 0;
  if (!(configured_dev_mask & (1 << (di.id & 31)))) {
    e = cudaFuncSetAttribute(sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem<D>::kAlloc);
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << (di.id & 31);
  }
  sparse_attn_kernel<D><<<di.sm_count, kThreads, AttnSmem<D>::kAlloc, s>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

static cudaError_t launch_attn(const void* Q, const void* K, const void* V, int BH, int N, int d,
                               const AttnArgs& args, cudaStream_t s) {
  if (d == 128) return launch_attn_kernel<128>(Q, K, V, BH, N, args, s);
  return launch_attn_kernel<64>(Q, K, V, BH, N, args, s);
}

cudaError_t launch_sparse_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                    const int32_t* idx, const int32_t* counts, int cap, uint64_t head_bits,
                                    float scale, void* O, void* ws, cudaStream_t s) {
  const int BH = B * H, nB = N / kBlock;
  const WsLayout wl = ws_layout(B, H, N, d);
  char* base = static_cast<char*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base + wl.header);
  int4* head_items = reinterpret_cast<int4*>(base + wl.head_items);
  int4* items = reinterpret_cast<int4*>(base + wl.items);
  int* head_np = reinterpret_cast<int*>(base + wl.head_np);
  int32_t* ulist = reinterpret_cast<int32_t*>(base + wl.ulist);
  plan_kernel<<<BH, kPlanThreads, 0, s>>>(idx, counts, nB, cap, H, head_bits, head_items, head_np, ulist,
                                          &hdr->err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  compact_items_kernel<<<1, 1024, 0, s>>>(head_items, head_np, BH, nB, items, &hdr->n_items);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint64_t all = (H >= 64) ? ~0ull : ((1ull << H) - 1ull);
  if ((head_bits & all) != all) {
    const size_t per_head_vec = static_cast<size_t>(N) * d / 8;
    zero_heads_kernel<<<dim3(64, BH), 256, 0, s>>>(static_cast<__nv_bfloat16*>(O), BH, H, head_bits, per_head_vec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  AttnArgs args{};
  args.items = items;
  args.ulist = ulist;
  args.n_items_dev = &hdr->n_items;
  args.n_items_host = 0;
  args.dense = 0;
  args.N = N;
  args.nB = nB;
  args.npairs_dense = (nB + 1) / 2;
  args.O = static_cast<__nv_bfloat16*>(O);
  args.scale_log2 = scale * 1.4426950408889634f;
  args.err = &hdr->err;
  return launch_attn(Q, K, V, BH, N, d, args, s);
}

cudaError_t launch_dense_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                   float scale, void* O, void* ws, cudaStream_t s) {
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
  args.O = static_cast<__nv_bfloat16*>(O);
  args.scale_log2 = scale * 1.4426950408889634f;
  args.err = &hdr->err;
  return launch_attn(Q, K, V, BH, N, d, args, s);
}

}  // namespace sa
