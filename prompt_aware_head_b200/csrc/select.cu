// Block selection, control patterns and density for block-sparse attention.
//
// Selection follows the SD.Next sparse-attention commit log, "selector"
// paragraph: mean-pool query and key tiles, score the tile pairs with no
// scale and no softmax, keep the highest-scoring key tiles per query tile
// within a budget that is a fraction of the sparsifiable candidates, always
// keep the diagonal.  The "layout" paragraph adds the pins (text / other
// rows and columns dense) and drops (padding).  The "host sync" paragraph
// asks for ranking with no host-side k and density read back on demand.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

// ============================================================== ranking
// Order-preserving map of a finite fp32 score to uint32 (larger key = larger
// score); -0 ranks as +0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Warp-wide top-k over keys held as key[c] for j = 32c + lane, restricted to
// the lanes/chunks set in `cand`.  Keys compare by value, ties by lower j.
// Returns the chosen bits (same layout as cand).  The k-th largest key is
// found bit by bit from the MSB with warp-reduced counts (no sort, no host k).
template <int NC>
__device__ __forceinline__ uint32_t warp_topk(const uint32_t (&key)[NC], uint32_t cand, int k) {
  const int ncand = __reduce_add_sync(0xffffffffu, __popc(cand));
  if (k >= ncand) return cand;
  uint32_t T = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t t2 = T | (1u << b);
    int cnt = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) cnt += (((cand >> c) & 1u) && key[c] >= t2) ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= k) T = t2;
  }
  int gt = 0;
#pragma unroll
  for (int c = 0; c < NC; ++c) gt += (((cand >> c) & 1u) && key[c] > T) ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need = k - gt;
  uint32_t sel = 0;
  int eq_before = 0;
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const bool isc = (cand >> c) & 1u;
    const bool g = isc && key[c] > T;
    const bool e = isc && key[c] == T;
    const uint32_t em = __ballot_sync(0xffffffffu, e);
    const int rank = eq_before + __popc(em & lt);
    if (g || (e && rank < need)) sel |= 1u << c;
    eq_before += __popc(em);
  }
  return sel;
}

// Writes the kept columns (bit c of keep <-> j = 32c + lane) in ascending
// order to out[] and returns the count (valid in every lane).
template <int NC>
__device__ __forceinline__ int warp_emit(uint32_t keep, int32_t* out) {
  int base = 0;
  const uint32_t lt = lanemask_lt();
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const bool kb = (keep >> c) & 1u;
    const uint32_t bm = __ballot_sync(0xffffffffu, kb);
    if (kb) out[base + __popc(bm & lt)] = 32 * c + lane;
    base += __popc(bm);
  }
  return base;
}

// Top-k over candidate keys by an 8-bit radix select (4 passes, most
// significant digit first) over a per-warp shared histogram; returns the
// chosen bits like warp_topk (keys compare by value, ties by lower j).
template <int NC>
__device__ __forceinline__ uint32_t warp_topk_radix(const uint32_t (&key)[NC], uint32_t cand, int k,
                                                    uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  const int ncand = __reduce_add_sync(0xffffffffu, __popc(cand));
  if (k >= ncand) return cand;
  uint32_t prefix = 0, pmask = 0;
  int kk = k;  // rank still to place among keys matching the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0u;
    __syncwarp();
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (((cand >> c) & 1u) && (key[c] & pmask) == prefix) atomicAdd(&hist[(key[c] >> shift) & 255u], 1u);
    __syncwarp();
    // lane l owns digits 255-8l down to 248-8l
    uint32_t h[8];
    uint32_t sum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      h[b] = hist[255 - (lane * 8 + b)];
      sum += h[b];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;
    const uint32_t want = static_cast<uint32_t>(kk);
    const bool here = excl < want && want <= incl;
    const int leader = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
    uint32_t digit = 0, above = 0;
    if (lane == leader) {
      uint32_t run = excl;
      bool found = false;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (!found && run + h[b] >= want) {
          digit = 255u - static_cast<uint32_t>(lane * 8 + b);
          above = run;  // keys with a larger digit under the same prefix
          found = true;
        }
        run += h[b];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, leader);
    above = __shfl_sync(0xffffffffu, above, leader);
    prefix |= digit << shift;
    pmask |= 255u << shift;
    kk -= static_cast<int>(above);
    __syncwarp();
  }
  // prefix is now the k-th largest key: keep keys above it and the first kk equal ones
  uint32_t sel = 0;
  int eq_before = 0;
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const bool isc = (cand >> c) & 1u;
    const bool g = isc && key[c] > prefix;
    const bool e = isc && key[c] == prefix;
    const uint32_t em = __ballot_sync(0xffffffffu, e);
    const int rank = eq_before + __popc(em & lt);
    if (g || (e && rank < kk)) sel |= 1u << c;
    eq_before += __popc(em);
  }
  return sel;
}

// Top-k (0 < kk < number of candidates) over fp32 scores s[c] at j = 32c +
// lane, by value then lower j, for finite scores: a 256-bucket histogram on
// the linear map t = (s - min) * 256 / (max - min), which never puts a
// larger score in a lower bucket, locates the bucket that holds the kk-th
// score; buckets above it are kept whole and the boundary bucket is ranked
// exactly (pairwise when it holds at most 32 scores, else by the radix
// select).  Non-finite scores or a zero / overflowing range go to the radix
// select directly, which orders the same way.
template <int NC>
__device__ __forceinline__ uint32_t warp_topk_bucket(const float (&s)[NC], uint32_t cand, int kk, uint32_t* hist,
                                                     uint32_t* memk) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NC];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    key[c] = score_key(s[c]);
    if ((cand >> c) & 1u) {
      kmin = min(kmin, key[c]);
      kmax = max(kmax, key[c]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // a non-finite score has a key at or beyond those of +-inf
  const bool bad = kmax >= 0xFF800000u || kmin <= 0x007FFFFFu;
  // back from keys to the extreme scores (exact; -0 comes back as +0)
  const float mn = __uint_as_float((kmin & 0x80000000u) ? (kmin & 0x7FFFFFFFu) : ~kmin);
  const float mx = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7FFFFFFFu) : ~kmax);
  const float range = mx - mn;
  const float inv = 256.0f / range;
  if (bad || !(range > 0.0f) || !isfinite(range) || !isfinite(inv)) return warp_topk_radix<NC>(key, cand, kk, hist);
  int bin[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) bin[c] = min(255, __float2int_rz((s[c] - mn) * inv));
#pragma unroll
  for (int b = 0; b < 8; ++b) hist[lane * 8 + b] = 0u;
  __syncwarp();
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if ((cand >> c) & 1u) atomicAdd(&hist[bin[c]], 1u);
  __syncwarp();
  // lane l owns buckets 255-8l down to 248-8l
  uint32_t h[8], sum = 0;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    h[b] = hist[255 - (lane * 8 + b)];
    sum += h[b];
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const uint32_t excl = incl - sum, want = static_cast<uint32_t>(kk);
  const int leader = __ffs(__ballot_sync(0xffffffffu, excl < want && want <= incl)) - 1;
  int bstar = 0;
  uint32_t above = 0, m = 0;
  if (lane == leader) {
    uint32_t run = excl;
    bool found = false;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (!found && run + h[b] >= want) {
        bstar = 255 - (lane * 8 + b);
        above = run;
        m = h[b];
        found = true;
      }
      run += h[b];
    }
  }
  bstar = __shfl_sync(0xffffffffu, bstar, leader);
  above = __shfl_sync(0xffffffffu, above, leader);
  m = __shfl_sync(0xffffffffu, m, leader);
  const int r = kk - static_cast<int>(above);  // 1..m of the boundary bucket's scores are kept
  uint32_t sel = 0, inb = 0;
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if ((cand >> c) & 1u) {
      if (bin[c] > bstar) sel |= 1u << c;
      else if (bin[c] == bstar) inb |= 1u << c;
    }
  if (r == static_cast<int>(m)) return sel | inb;
  __syncwarp();
  if (m > 32u) return sel | warp_topk_radix<NC>(key, inb, r, hist);
  // members in ascending j: position p holds the p-th one
  const uint32_t lt = lanemask_lt();
  int pos[NC];
  int base = 0;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const bool in = (inb >> c) & 1u;
    const uint32_t bm = __ballot_sync(0xffffffffu, in);
    pos[c] = base + __popc(bm & lt);
    if (in) memk[pos[c]] = key[c];
    base += __popc(bm);
  }
  __syncwarp();
  bool win = false;
  if (lane < static_cast<int>(m)) {
    const uint32_t kl = memk[lane];
    int rank = 0;
    for (int q = 0; q < static_cast<int>(m); ++q) {
      const uint32_t kq = memk[q];
      rank += (kq > kl || (kq == kl && q < lane)) ? 1 : 0;
    }
    win = rank < r;
  }
  const uint32_t wins = __ballot_sync(0xffffffffu, win);
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (((inb >> c) & 1u) && ((wins >> pos[c]) & 1u)) sel |= 1u << c;
  __syncwarp();
  return sel;
}

// ============================================================== selection in three kernels
// The path of sa_select_blocks (and, a group of heads at a time, of
// sa_select_blocks_noalloc):
//   pool_kernel      - one CTA per 64-row block of Q and K: their means, each
//                      split into a tf32 part and the fp32 remainder, written
//                      straight into the operand images the tensor cores read;
//   score_tc_kernel  - one CTA per 128 x 256 tile of a head's scores: bulk
//                      copies of the images, 3xTF32 MMAs into TMEM, tensor
//                      stores of the scores;
//   rank_rows_kernel - one warp per row keeps the pins, the diagonal and the
//                      top k - 1 scores (bucket select).
// Kernel boundaries order the three, so every image is complete before a
// tile reads it.
//
// Operand images: block means of a head in row tiles of 128 blocks and
// column chunks of 32 (of d), each a 16 KB image of 128 rows x 128 bytes laid
// out as the K-major 128-byte-swizzled shared-memory tile the MMA descriptors
// address: row t at byte 128 t, its 16-byte group g at group g ^ (t & 7).
// Four arrays (q hi, q lo, k hi, k lo), each [slot][row tile][chunk][128][32].
// hi = tf32(x) rounded to nearest, lo = x - hi (exact); the MMAs accumulate
// A_hi B_lo + A_lo B_hi + A_hi B_hi in fp32, which leaves each product within
// about 2^-22 |a||b| of exact (the dropped lo lo term and the tf32 truncation
// of lo), as accurate as an fp32 dot product for d <= 128.
constexpr int kTcM = 128;                 // query blocks per tile (rows of A, TMEM lanes)
constexpr int kTcN = 256;                 // key blocks per tile (two row tiles of B)
constexpr int kImgBytes = kTcM * 128;     // one 128-row x 32-fp32 image: 16 KB
constexpr int kImgFloats = kImgBytes / 4;
constexpr int kTcStage = 6 * kImgBytes;   // A hi, A lo, B hi (2 tiles), B lo (2 tiles)
constexpr int kTcSmem = 2 * kTcStage + 1024 + 128;

// Instruction descriptor: kind::tf32 with tf32 A/B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Float offset of block i, dimension col inside a head's image array.
template <int D>
__device__ __forceinline__ size_t img_offset(int i, int col) {
  const int rt = i >> 7, t = i & 127, kc = col >> 5, g = (col & 31) >> 2;
  return (static_cast<size_t>(rt) * (D / 32) + kc) * kImgFloats + t * 32 + ((g ^ (t & 7)) << 2) + (col & 3);
}

// One CTA per (query/key block i, head bh = bh0 + slot): mean of the 64 rows
// of Q and K.  16-byte vector loads, fp32 sums in a fixed order (per-thread
// rows, then row groups in order), scaled by 1/64 (exact), then split into
// hi / lo and written to the images of slot (RT row tiles per head).
// HBM-bound.  GQA (g query heads per key head): the key images are indexed
// by key head, kv_head(bh) - kv0, and only the first active query head of a
// group among this launch's heads pools the shared key head.
template <int D, bool GQA>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K, float* __restrict__ qimg,
                                                   float* __restrict__ kimg, int N, int nB, int RT, int H,
                                                   uint64_t head_bits, int bh0, size_t lo_offset, int g, int kv0) {
  grid_dep_wait();
  const int i = blockIdx.x, slot = blockIdx.y, bh = bh0 + slot;
  if (!((head_bits >> (bh % H)) & 1ull)) return;
  constexpr int TPR = D / 8;     // threads per row, 8 bf16 (16 B) each
  constexpr int RG = 128 / TPR;  // row groups
  constexpr int RPT = 64 / RG;   // rows per thread
  const int t = threadIdx.x, cg = t % TPR, rg = t / TPR;
  int kvh = bh;
  bool pool_k = true;
  if (GQA) {
    kvh = kv_head(bh, H, g);
    for (int h2 = max(bh - (bh % H) % g, bh0); h2 < bh; ++h2)
      if ((head_bits >> (h2 % H)) & 1ull) pool_k = false;
  }
  const size_t base = (static_cast<size_t>(bh) * N + static_cast<size_t>(i) * kBlock) * D;
  const size_t kbase = (static_cast<size_t>(kvh) * N + static_cast<size_t>(i) * kBlock) * D;
  const uint4* q4 = reinterpret_cast<const uint4*>(Q + base);
  const uint4* k4 = reinterpret_cast<const uint4*>(K + kbase);
  uint4 qv[RPT], kv[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int row = rg + r * RG;
    qv[r] = __ldg(q4 + row * TPR + cg);
    kv[r] = pool_k ? __ldg(k4 + row * TPR + cg) : make_uint4(0, 0, 0, 0);
  }
  float aq[8], ak[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) aq[e] = ak[e] = 0.f;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const uint32_t qw[4] = {qv[r].x, qv[r].y, qv[r].z, qv[r].w};
    const uint32_t kw[4] = {kv[r].x, kv[r].y, kv[r].z, kv[r].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      aq[2 * e] += __uint_as_float(qw[e] << 16);
      aq[2 * e + 1] += __uint_as_float(qw[e] & 0xFFFF0000u);
      ak[2 * e] += __uint_as_float(kw[e] << 16);
      ak[2 * e + 1] += __uint_as_float(kw[e] & 0xFFFF0000u);
    }
  }
  __shared__ float red[2][RG][D];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    red[0][rg][cg * 8 + e] = aq[e];
    red[1][rg][cg * 8 + e] = ak[e];
  }
  __syncthreads();
  const size_t head = static_cast<size_t>(slot) * RT * (D / 32) * kImgFloats;
  const size_t khead = GQA ? static_cast<size_t>(kvh - kv0) * RT * (D / 32) * kImgFloats : head;
  for (int c = t; c < (pool_k ? 2 : 1) * D; c += 128) {
    const int which = c / D, col = c % D;
    float s = 0.f;
#pragma unroll
    for (int rgi = 0; rgi < RG; ++rgi) s += red[which][rgi][col];
    s *= (1.0f / 64.0f);
    const float hi = tf32_rn(s);
    float* img = (which ? kimg + khead : qimg + head) + img_offset<D>(i, col);
    img[0] = hi;
    img[lo_offset] = s - hi;
  }
}

// 3D tiled store (no multicast) of a shared-memory box to global memory,
// tracked by the issuing thread's bulk-async group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most n of this thread's bulk stores still read shared memory.
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

struct TcArgs {
  const float* qimg;  // q hi images; q lo at + lo_offset
  const float* kimg;  // k hi images; k lo at + lo_offset
  float* scores;      // [slot][nB][nB]
  int* err;
  size_t lo_offset;
  int nB, RT, H, bh0;
  int g, kv0;     // query heads per key head; key head of bh0 (key images are indexed from it)
  int tma_store;  // 1: scores leave through the tensor map (3D [slot][nB][nB] fp32, 128-byte swizzle)
  uint64_t head_bits;
};

// The 12 MMAs of one 32-wide chunk of d: 4 steps of K = 8, each adding
// A_hi B_lo, A_lo B_hi and A_hi B_hi (the small terms first) into D.
__device__ __forceinline__ void tc_issue_chunk(uint32_t d_tmem, uint64_t ahi, uint64_t alo, uint64_t bhi, uint64_t blo,
                                               uint32_t idesc, int accumulate) {
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const uint64_t o = 2 * s;  // 32 bytes per K = 8 step, in descriptor units
    asm volatile(
        "{\n .reg .pred p0, p1;\n setp.ne.b32 p0, %6, 0;\n setp.eq.b32 p1, 0, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %4, %5, p0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %2, %3, %5, p1;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %3, %5, p1;\n}\n" ::"r"(d_tmem),
        "l"(ahi + o), "l"(alo + o), "l"(bhi + o), "l"(blo + o), "r"(idesc), "r"((accumulate || s > 0) ? 1 : 0)
        : "memory");
  }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// One CTA (4 warps) per 128 x 256 tile of one head's scores: query blocks
// m0 = 128 blockIdx.y + r (row tile blockIdx.y of A), key blocks
// n0 = 256 blockIdx.x + c (row tiles 2 blockIdx.x and 2 blockIdx.x + 1 of B).
// Thread 0 streams the d chunks' images through two stages with bulk copies
// and issues each chunk's MMAs once its stage is full; the MMA commit frees
// the stage.  Warp w then reads TMEM lanes 32 w .. 32 w + 31 (tile rows);
// the scores leave through tensor stores of 128 x 32 boxes staged in the
// drained stage buffers, or, where the score rows do not fit a tensor map,
// as each warp's row stores.  Image rows past nB hold whatever was there:
// they only reach scores that are never written out.
template <int D>
__global__ void __launch_bounds__(128, 1) score_tc_kernel(const __grid_constant__ TcArgs a,
                                                          const __grid_constant__ CUtensorMap ms) {
  constexpr int NKC = D / 32;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + 2 * kTcStage);  // [2]
  uint64_t* empty = full + 2;                                         // [2]
  uint64_t* done = empty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  int* flags = reinterpret_cast<int*>(tslot + 1);
  volatile int* abort_flag = flags;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int slot = blockIdx.z, bh = a.bh0 + slot, nB = a.nB, RT = a.RT;
  if (!((a.head_bits >> (bh % a.H)) & 1ull)) return;
  const int rt = blockIdx.y, bt0 = 2 * blockIdx.x, nbt = (bt0 + 1 < RT) ? 2 : 1;
  const int m0 = rt * kTcM, n0 = blockIdx.x * kTcN;
  if (t == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    flags[0] = 0;
    mbar_fence_init();
  }
  if (w == 0) tmem_alloc(tslot, kTcN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_wait();  // the images come from the previous kernel
  const uint32_t tmem = *tslot;
  bool ok = true;
  if (t == 0) {
    const size_t head = static_cast<size_t>(slot) * RT * NKC * kImgFloats;
    const float* qh = a.qimg + head;
    const float* kh = a.kimg + static_cast<size_t>(kv_head(bh, a.H, a.g) - a.kv0) * RT * NKC * kImgFloats;
    const uint32_t bytes = static_cast<uint32_t>((2 + 2 * nbt) * kImgBytes);
    auto load = [&](int kc, int s) {
      unsigned char* st = sm + s * kTcStage;
      mbar_expect_tx(&full[s], bytes);
      const size_t ao = (static_cast<size_t>(rt) * NKC + kc) * kImgFloats;
      bulk_load(st, qh + ao, kImgBytes, &full[s]);
      bulk_load(st + kImgBytes, qh + a.lo_offset + ao, kImgBytes, &full[s]);
      for (int b = 0; b < nbt; ++b) {
        const size_t bo = (static_cast<size_t>(bt0 + b) * NKC + kc) * kImgFloats;
        bulk_load(st + (2 + b) * kImgBytes, kh + bo, kImgBytes, &full[s]);
        bulk_load(st + (4 + b) * kImgBytes, kh + a.lo_offset + bo, kImgBytes, &full[s]);
      }
    };
    constexpr uint32_t kIdesc = idesc_tf32_f32(kTcM, kTcN);
    int loaded = 0, multiplied = 0;
    load(0, 0);
    ++loaded;
    if (NKC > 1) {
      load(1, 1);
      ++loaded;
    }
    for (int kc = 0; kc < NKC; ++kc) {
      const int s = kc & 1;
      if (!mbar_wait(&full[s], (kc >> 1) & 1, abort_flag, a.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(sm + s * kTcStage);
      tc_issue_chunk(tmem, smem_desc_sw128(st, 16, 1024), smem_desc_sw128(st + kImgBytes, 16, 1024),
                     smem_desc_sw128(st + 2 * kImgBytes, 16, 1024), smem_desc_sw128(st + 4 * kImgBytes, 16, 1024),
                     kIdesc, kc);
      tc_commit(&empty[s]);
      ++multiplied;
      if (kc + 2 < NKC) {
        if (!mbar_wait(&empty[s], (kc >> 1) & 1, abort_flag, a.err)) {
          ok = false;
          break;
        }
        load(kc + 2, s);
        ++loaded;
      }
    }
    if (ok) {
      tc_commit(done);
    } else {  // after an abort: copies and MMAs in flight finish before the CTA leaves
      for (int x = multiplied; x < loaded; ++x) mbar_wait_drain(&full[x & 1], (x >> 1) & 1, a.err);
      if (multiplied > 0) mbar_wait_drain(&empty[(multiplied - 1) & 1], ((multiplied - 1) >> 1) & 1, a.err);
      *abort_flag = 1;
    }
  }
  ok = __syncthreads_and(ok ? 1 : 0) != 0;
  if (ok) ok = __syncthreads_and(mbar_wait(done, 0, abort_flag, a.err) ? 1 : 0) != 0;
  tc_fence_after();
  if (ok && a.tma_store) {
    // Each 32-column block: TMEM -> registers (lane = tile row) -> a 128 x 32
    // fp32 box in shared memory, 128-byte swizzled (row r at byte 128 r, its
    // 16-byte group g at g ^ (r & 7)), two boxes alternating -> one tensor
    // store per box; the store clips rows and columns past nB.
    const int r = 32 * w + lane;
#pragma unroll 1
    for (int cb = 0; cb < kTcN / 32; ++cb) {
      const int j0 = n0 + 32 * cb;
      if (j0 >= nB) break;
      unsigned char* box = sm + (cb & 1) * kImgBytes;
      if (cb >= 2) {  // the store issued from this box two blocks ago has read it
        if (t == 0) bulk_wait_read<1>();
        __syncthreads();
      }
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * w) << 16) + 32 * cb, v);
      tmem_wait_ld();
#pragma unroll
      for (int g = 0; g < 8; ++g)
        *reinterpret_cast<uint4*>(box + r * 128 + ((g ^ (r & 7)) << 4)) =
            make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic stores -> the store's reads
      __syncthreads();
      if (t == 0) tma_store_3d(&ms, box, j0, m0, slot);
    }
    if (t == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  } else if (ok) {
    const int i = m0 + 32 * w + lane;
    float* out = a.scores + (static_cast<size_t>(slot) * nB + i) * nB;
#pragma unroll 1
    for (int cb = 0; cb < kTcN / 32; ++cb) {
      const int j0 = n0 + 32 * cb;
      if (j0 >= nB) break;
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * w) << 16) + 32 * cb, r);
      tmem_wait_ld();
      if (i < nB) {
        if ((nB & 3) == 0 && j0 + 32 <= nB) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(out + j0 + c) = make_float4(
                __uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]), __uint_as_float(r[c + 3]));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (j0 + c < nB) out[j0 + c] = __uint_as_float(r[c]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (w == 0) tmem_dealloc(tmem, kTcN);
}

// ============================================================== ranking rows
// The layout's block classes as bit masks, passed by value (constant
// memory): no per-CTA load of the classes before the scores can be read.
struct ClassBits {
  uint32_t pin[32], sparse[32];
};

// One warp per query block row (head bh = bh0 + slot) of the scores
// score_tc_kernel wrote ([slot][nB][nB]): the pins,
// the diagonal (it outranks every score) and the top k - 1 other sparse
// candidates by the bucket select; the list goes out in ascending order.
// Rows of skipped heads get empty lists.  Both of a warp's rows have their
// scores loaded at the start, so the second row's load latency hides behind
// the first row's selection.
template <int NC>
__global__ void __launch_bounds__(128, NC <= 17 ? 8 : 4) rank_rows_kernel(const float* __restrict__ scores,
                                                           const __grid_constant__ ClassBits cb, int nB, int H,
                                                           uint64_t head_bits, int k, int cap,
                                                           int32_t* __restrict__ idx, int32_t* __restrict__ counts,
                                                           int bh0) {
  __shared__ uint32_t hist[4][256];
  __shared__ uint32_t memk[4][32];
  grid_dep_wait();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, slot = blockIdx.y, bh = bh0 + slot;
  const bool active_head = (head_bits >> (bh % H)) & 1ull;
  // row rr's sparse candidates' scores (0 elsewhere); both rows up front where
  // the registers allow (NC <= 9, up to 288 blocks), else each row in turn
  constexpr bool kBoth = NC <= 9;
  float sc[2][NC];
  auto load_row = [&](int rr) {
    const int i = blockIdx.x * 8 + rr * 4 + w;
    const bool sparse_row = active_head && i < nB && ((cb.sparse[i >> 5] >> (i & 31)) & 1u);
    const float* srow = scores + (static_cast<size_t>(slot) * nB + i) * nB + lane;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const bool sp = (cb.sparse[c] >> lane) & 1u;
      sc[rr][c] = (sparse_row && sp && 32 * c + lane != i) ? __ldg(srow + 32 * c) : 0.f;
    }
  };
  load_row(0);
  if (kBoth) load_row(1);
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {  // two rows per warp: one wave covers every row
    const int i = blockIdx.x * 8 + rr * 4 + w;
    if (i >= nB) return;
    if (!kBoth && rr == 1) load_row(1);
    const size_t row = static_cast<size_t>(bh) * nB + i;
    if (!active_head) {
      if (lane == 0) counts[row] = 0;
      continue;
    }
    const bool row_pin = (cb.pin[i >> 5] >> (i & 31)) & 1u;
    const bool row_sparse = (cb.sparse[i >> 5] >> (i & 31)) & 1u;
    uint32_t keep = 0;
    if (row_pin) {
#pragma unroll
      for (int c = 0; c < NC; ++c) keep |= (((cb.pin[c] | cb.sparse[c]) >> lane) & 1u) << c;
    } else if (row_sparse) {
      uint32_t cand = 0, diag = 0;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        keep |= ((cb.pin[c] >> lane) & 1u) << c;
        const bool sp = (cb.sparse[c] >> lane) & 1u;
        const bool dg = 32 * c + lane == i;
        diag |= (sp && dg ? 1u : 0u) << c;
        cand |= (sp && !dg ? 1u : 0u) << c;
      }
      if (k >= 1) {
        keep |= diag;
        const int kk = k - 1;
        const int ncand = __reduce_add_sync(0xffffffffu, __popc(cand));
        if (kk >= ncand) keep |= cand;
        else if (kk > 0) keep |= warp_topk_bucket<NC>(sc[rr], cand, kk, hist[w], memk[w]);
      }
    }
    const int n = warp_emit<NC>(keep, idx + row * cap);
    if (lane == 0) counts[row] = n;
  }
}

// ============================================================== patterns
// Control patterns at the layout's pins and drops (SD.Next commit log,
// "radial control" paragraph; inferensys glossary: sliding window, dilated,
// global tokens).  One warp per query block; the list is the same for every
// head and is replicated to each active head.
__device__ __forceinline__ bool window_cover(int i, int j, int W) {
  const int gap = kBlock * abs(i - j) - (kBlock - 1);
  return gap <= W;  // gap <= 0 means the blocks overlap in token distance 0
}

// True when some key - query offset in [64(j-i)-63, 64(j-i)+63] lies in
// [-W, W] and is a multiple of r (closed form: the first multiple of r at or
// above the interval's low end).
__device__ __forceinline__ bool dilated_cover(int i, int j, int W, int r) {
  int lo = kBlock * (j - i) - (kBlock - 1);
  int hi = kBlock * (j - i) + (kBlock - 1);
  lo = max(lo, -W);
  hi = min(hi, W);
  if (lo > hi) return false;
  const int first = lo >= 0 ? ((lo + r - 1) / r) * r : -(((-lo) / r) * r);
  return first <= hi;
}

// Output n >= 1 of SplitMix64 (Steele, Lea and Flood 2014) seeded with
// `seed`: the state advances by the odd constant 0x9E3779B97F4A7C15 per
// output and is put through the mix (xor-shift 30, multiply, xor-shift 27,
// multiply, xor-shift 31).  Counter-based: any output is computed directly.
__device__ __forceinline__ unsigned long long splitmix64_nth(unsigned long long seed, unsigned long long n) {
  unsigned long long z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// kind: 0 radial, 1 window + global, 2 dilated, 3 dense, 4 random (seed).
template <int NC>
__global__ void __launch_bounds__(128) pattern_kernel(const uint8_t* __restrict__ cls,
                                                      const int32_t* __restrict__ sparse_rank, int nB, int kind,
                                                      int W, int G, int r, int k, int BH, int H,
                                                      uint64_t head_bits, int cap, int32_t* __restrict__ idx,
                                                      int32_t* __restrict__ counts, unsigned long long seed) {
  __shared__ int32_t lst[4][NC * 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 4 + w;
  if (i >= nB) return;
  const uint8_t ci = cls[i];
  const bool row_global = ci == kSparse && (kind == 1 || kind == 2) && sparse_rank[i] < G;
  uint32_t keep = 0;
  if (ci == kPin || (ci == kSparse && (kind == 3 || row_global))) {
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int j = 32 * c + lane;
      if (j < nB && cls[j] != kDrop) keep |= 1u << c;
    }
  } else if (ci == kSparse) {
    uint32_t key[NC];
    uint32_t cand = 0, pin = 0, win = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int j = 32 * c + lane;
      key[c] = 0;
      if (j >= nB) continue;
      const uint8_t cj = cls[j];
      if (cj == kPin) pin |= 1u << c;
      if (cj != kSparse) continue;
      if (kind == 0) {
        key[c] = ~((static_cast<uint32_t>(abs(i - j)) << 16) | static_cast<uint32_t>(j));
        cand |= 1u << c;
      } else if (kind == 4) {
        // the diagonal above every draw; a draw's 21 bits above 1023 - j (nB <= 1024): distinct keys,
        // larger draw first, ties to the lower j
        const unsigned long long u =
            splitmix64_nth(seed, static_cast<unsigned long long>(i) * static_cast<unsigned long long>(nB) + j + 1);
        key[c] = (j == i) ? 0xFFFFFFFFu : ((static_cast<uint32_t>(u >> 43) << 10) | static_cast<uint32_t>(1023 - j));
        cand |= 1u << c;
      } else {
        const bool glob = sparse_rank[j] < G;
        const bool cover = (kind == 1) ? window_cover(i, j, W) : dilated_cover(i, j, W, r);
        if (glob || cover) win |= 1u << c;
      }
    }
    keep = pin | win;
    if (kind == 0 || kind == 4) keep |= warp_topk<NC>(key, cand, k);
  }
  const int n = warp_emit<NC>(keep, lst[w]);
  __syncwarp();
  for (int bh = 0; bh < BH; ++bh) {
    const bool active = (head_bits >> (bh % H)) & 1ull;
    int32_t* row = idx + (static_cast<size_t>(bh) * nB + i) * cap;
    if (active)
      for (int e = lane; e < n; e += 32) row[e] = lst[w][e];
    if (lane == 0) counts[static_cast<size_t>(bh) * nB + i] = active ? n : 0;
  }
}

// ============================================================== density
__global__ void density_kernel(const int32_t* __restrict__ counts, int nB, int H, uint64_t head_bits,
                               unsigned long long* __restrict__ tiles) {
  const int bh = blockIdx.x;
  if (!((head_bits >> (bh % H)) & 1ull)) return;
  unsigned long long s = 0;
  for (int i = threadIdx.x; i < nB; i += blockDim.x) s += static_cast<unsigned long long>(counts[static_cast<size_t>(bh) * nB + i]);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0 && s) atomicAdd(tiles, s);
}

// ============================================================== launchers
static int chunks_for(int nB) {
  const int need = (nB + 31) / 32;
  const int opts[] = {2, 4, 8, 12, 17, 24, 32};
  for (int o : opts)
    if (need <= o) return o;
  return -1;
}

// Chunk counts (32 key blocks each) the rank kernel is built for.
static int select_chunks(int nB) {
  const int need = (nB + 31) / 32;
  const int opts[] = {2, 4, 8, 9, 12, 17, 24, 32};
  for (int o : opts)
    if (need <= o) return o;
  return -1;
}

// Per-device one-time setup of a kernel's dynamic shared memory limit.
template <typename F>
static cudaError_t ensure_smem(F* kernel, size_t bytes, bool* configured, std::mutex& mu, int dev) {
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && configured[dev]) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && dev < 64) configured[dev] = true;
  return e;
}

template <int NC>
static cudaError_t launch_rank_t(const float* scores, const sa_layout* L, int bh0, int nbh, int H, uint64_t head_bits,
                                 int k, int32_t* idx, int32_t* counts, cudaStream_t s) {
  ClassBits cb;
  std::memcpy(cb.pin, L->pin_bits, sizeof cb.pin);
  std::memcpy(cb.sparse, L->sparse_bits, sizeof cb.sparse);
  return launch_pdl(rank_rows_kernel<NC>, dim3((L->nB + 7) / 8, nbh), dim3(128), 0, s, scores, cb, L->nB, H,
                    head_bits, k, L->cap, idx, counts, bh0);
}

static cudaError_t launch_rank(int nc, const float* scores, const sa_layout* L, int bh0, int nbh, int H,
                               uint64_t head_bits, int k, int32_t* idx, int32_t* counts, cudaStream_t s) {
  switch (nc) {
    case 2: return launch_rank_t<2>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 4: return launch_rank_t<4>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 8: return launch_rank_t<8>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 9: return launch_rank_t<9>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 12: return launch_rank_t<12>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 17: return launch_rank_t<17>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 24: return launch_rank_t<24>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    case 32: return launch_rank_t<32>(scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
    default: return cudaErrorInvalidValue;
  }
}

// The driver's tensor-map encoder, looked up once.
static PFN_cuTensorMapEncodeTiled_v12000 score_map_encoder() {
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

// Scores [nbh][nB][nB] fp32 as a 3D tensor (columns, rows, slots), boxes of
// 32 columns x 128 rows, 128-byte swizzle.  Needs rows of whole 16-byte
// groups (nB % 4 == 0) and a 16-byte aligned base; false otherwise.
static bool make_score_map(CUtensorMap* map, float* scores, int nB, int nbh) {
  if ((nB & 3) != 0 || (reinterpret_cast<uintptr_t>(scores) & 15) != 0) return false;
  auto enc = score_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(nB), static_cast<cuuint64_t>(nB), static_cast<cuuint64_t>(nbh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(nB) * 4, static_cast<cuuint64_t>(nB) * nB * 4};
  cuuint32_t box[3] = {32, kTcM, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, scores, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Floats of one head's image array (hi or lo).
static size_t img_floats(int nB, int d) { return static_cast<size_t>((nB + kTcM - 1) / kTcM) * d * kTcM; }

// The three kernels over heads bh0 .. bh0 + nbh - 1: the images (q, k: hi
// then lo, nbh heads each) and scores are slot-indexed ([bh - bh0] ...),
// idx / counts indexed by bh.
static cudaError_t select_heads(const sa_layout* L, const void* Q, const void* K, int H, int Hkv, int d, int k,
                                uint64_t head_bits, int bh0, int nbh, float* qimg, float* kimg, float* scores, int* err,
                                int32_t* idx, int32_t* counts, cudaStream_t s) {
  static bool configured[2][64];  // per head size, per device
  static std::mutex mu;
  const int nB = L->nB, nc = select_chunks(nB), RT = (nB + kTcM - 1) / kTcM;
  if (nc < 0) return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  e = d == 128 ? ensure_smem(score_tc_kernel<128>, kTcSmem, configured[0], mu, di.id)
               : ensure_smem(score_tc_kernel<64>, kTcSmem, configured[1], mu, di.id);
  if (e != cudaSuccess) return e;
  const size_t lo = static_cast<size_t>(nbh) * img_floats(nB, d);
  const auto* q = static_cast<const __nv_bfloat16*>(Q);
  const auto* kk = static_cast<const __nv_bfloat16*>(K);
  // Key images are indexed by key head from kv0, the key head of bh0; the
  // key heads of bh0 .. bh0 + nbh - 1 are consecutive, at most nbh of them.
  const int g = H / Hkv, kv0 = (bh0 / H) * Hkv + (bh0 % H) / g;
  const dim3 pg(nB, nbh);
  if (g == 1)
    e = d == 128 ? launch_pdl(pool_kernel<128, false>, pg, dim3(128), 0, s, q, kk, qimg, kimg, L->N, nB, RT, H,
                              head_bits, bh0, lo, g, kv0)
                 : launch_pdl(pool_kernel<64, false>, pg, dim3(128), 0, s, q, kk, qimg, kimg, L->N, nB, RT, H,
                              head_bits, bh0, lo, g, kv0);
  else
    e = d == 128 ? launch_pdl(pool_kernel<128, true>, pg, dim3(128), 0, s, q, kk, qimg, kimg, L->N, nB, RT, H,
                              head_bits, bh0, lo, g, kv0)
                 : launch_pdl(pool_kernel<64, true>, pg, dim3(128), 0, s, q, kk, qimg, kimg, L->N, nB, RT, H,
                              head_bits, bh0, lo, g, kv0);
  if (e != cudaSuccess) return e;
  CUtensorMap ms;
  std::memset(&ms, 0, sizeof ms);
  const int tma_store = make_score_map(&ms, scores, nB, nbh) ? 1 : 0;  // else plain row stores
  TcArgs ta{qimg, kimg, scores, err, lo, nB, RT, H, bh0, g, kv0, tma_store, head_bits};
  const dim3 grid((nB + kTcN - 1) / kTcN, RT, nbh);
  e = d == 128 ? launch_pdl(score_tc_kernel<128>, grid, dim3(128), kTcSmem, s, ta, ms)
               : launch_pdl(score_tc_kernel<64>, grid, dim3(128), kTcSmem, s, ta, ms);
  if (e != cudaSuccess) return e;
  return launch_rank(nc, scores, L, bh0, nbh, H, head_bits, k, idx, counts, s);
}

cudaError_t launch_select(const sa_layout* L, const void* Q, const void* K, int B, int H, int Hkv, int d, int k,
                          uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out, void* ws,
                          cudaStream_t s) {
  if (k >= L->n_cand && scores_out == nullptr)  // the budget covers every candidate: dense lists, no scoring
    return launch_pattern(L, 3, 0, 0, 1, k, B, H, head_bits, idx, counts, s);
  const WsLayout wl = ws_layout(B, H, L->N, d);
  char* base = static_cast<char*>(ws);
  float* scores = scores_out ? scores_out : reinterpret_cast<float*>(base + wl.scores);
  return select_heads(L, Q, K, H, Hkv, d, k, head_bits, 0, B * H, reinterpret_cast<float*>(base + wl.qbar),
                      reinterpret_cast<float*>(base + wl.kbar), scores,
                      &reinterpret_cast<WsHeader*>(base + wl.header)->err, idx, counts, s);
}

// ============================================================== selection without allocation
// For callers that cannot allocate device memory (see sa_select_blocks_noalloc
// in sa.h): the pooled block means (and the scores when the caller takes
// none) live in this fixed, file-scope device array instead of the caller's
// workspace, a group of heads at a time.  Every process that loads the
// library holds it on every GPU it uses until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB: q-bar, k-bar (and scores), fp32
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

size_t select_noalloc_limit() { return kNoAllocScratchBytes; }

// Device address of the scratch array for the current device.  The host-side
// symbol is only a stand-in, so the address is asked of the runtime once per
// device (on the first call made with that device current) and cached.
static cudaError_t noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_select_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

// The error word the kernels of the no-allocation path record device-side
// faults in: the last 256 bytes of the scratch array, zero at load.
cudaError_t noalloc_error_word(int** out) {
  void* scratch = nullptr;
  const cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  *out = reinterpret_cast<int*>(static_cast<char*>(scratch) + kNoAllocScratchBytes - 256);
  return cudaSuccess;
}

cudaError_t launch_select_noalloc(const sa_layout* L, const void* Q, const void* K, int B, int H, int Hkv, int d,
                                  int k, uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out,
                                  cudaStream_t s) {
  const int BH = B * H, nB = L->nB;
  if (k >= L->n_cand && scores_out == nullptr)  // dense lists: no scratch used
    return launch_pattern(L, 3, 0, 0, 1, k, B, H, head_bits, idx, counts, s);
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  // Per group of G heads: the q and k operand images (hi and lo) and (unless
  // the caller takes them) the scores, then a word for the kernels' error
  // bits.  Every value that reaches an output is written for each active head
  // before it is read: nothing needs clearing.
  const size_t img = img_floats(nB, d) * sizeof(float);  // one head's hi (or lo) images
  const size_t per_head = 4 * img + (scores_out ? 0 : static_cast<size_t>(nB) * nB * sizeof(float));
  const int G = static_cast<int>(std::min<size_t>(BH, (kNoAllocScratchBytes - 256) / per_head));
  if (G < 1) return cudaErrorInvalidValue;
  char* base = static_cast<char*>(scratch);
  float* qimg = reinterpret_cast<float*>(base);
  float* kimg = reinterpret_cast<float*>(base + 2 * G * img);
  float* sc_scratch = reinterpret_cast<float*>(base + 4 * G * img);
  int* err = nullptr;
  e = noalloc_error_word(&err);
  if (e != cudaSuccess) return e;
  for (int bh0 = 0; bh0 < BH; bh0 += G) {
    const int nbh = std::min(G, BH - bh0);
    float* sc = scores_out ? scores_out + static_cast<size_t>(bh0) * nB * nB : sc_scratch;
    e = select_heads(L, Q, K, H, Hkv, d, k, head_bits, bh0, nbh, qimg, kimg, sc, err, idx, counts, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int NC>
static void launch_pattern_t(const sa_layout* L, int kind, int W, int G, int r, int k, int BH, int H,
                             uint64_t head_bits, int32_t* idx, int32_t* counts, uint64_t seed, cudaStream_t s) {
  pattern_kernel<NC><<<(L->nB + 3) / 4, 128, 0, s>>>(L->d_cls, L->d_sparse_rank, L->nB, kind, W, G, r, k, BH, H,
                                                     head_bits, L->cap, idx, counts, seed);
}

cudaError_t launch_pattern(const sa_layout* L, int kind, int W, int G, int r, int k, int B, int H,
                           uint64_t head_bits, int32_t* idx, int32_t* counts, cudaStream_t s, uint64_t seed) {
  const int BH = B * H;
  switch (chunks_for(L->nB)) {
    case 2: launch_pattern_t<2>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 4: launch_pattern_t<4>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 8: launch_pattern_t<8>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 12: launch_pattern_t<12>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 17: launch_pattern_t<17>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 24: launch_pattern_t<24>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    case 32: launch_pattern_t<32>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, seed, s); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_density(const int32_t* counts, int B, int H, int nB, uint64_t head_bits, void* ws,
                           unsigned long long* host_tiles, cudaStream_t s) {
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  cudaError_t e = cudaMemsetAsync(&hdr->tiles, 0, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return e;
  density_kernel<<<B * H, 256, 0, s>>>(counts, nB, H, head_bits, &hdr->tiles);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyAsync(host_tiles, &hdr->tiles, sizeof(unsigned long long), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(s);
}

}  // namespace sa
