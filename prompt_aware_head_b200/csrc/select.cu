// Block selection, control patterns and density for block-sparse attention.
//
// Selection follows the SD.Next sparse-attention commit log, "selector"
// paragraph: mean-pool query and key tiles, score the tile pairs with no
// scale and no softmax, keep the highest-scoring key tiles per query tile
// within a budget that is a fraction of the sparsifiable candidates, always
// keep the diagonal.  The "layout" paragraph adds the pins (text / other
// rows and columns dense) and drops (padding).  The "host sync" paragraph
// asks for ranking with no host-side k and density read back on demand.
#include <algorithm>
#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

// ============================================================== pooling
// One CTA per (query/key block i, head bh): mean of the 64 rows of Q and K.
// 16-byte vector loads, fp32 sums in a fixed order (per-thread rows, then
// row groups in order), scaled by 1/64 (exact).  HBM-bound.
template <int D>
__global__ void __launch_bounds__(128) pool_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ K, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int N, int nB, int H,
                                                   uint64_t head_bits) {
  const int i = blockIdx.x, bh = blockIdx.y;
  if (!((head_bits >> (bh % H)) & 1ull)) return;
  constexpr int TPR = D / 8;     // threads per row, 8 bf16 (16 B) each
  constexpr int RG = 128 / TPR;  // row groups
  constexpr int RPT = 64 / RG;   // rows per thread
  const int t = threadIdx.x, cg = t % TPR, rg = t / TPR;
  const size_t base = (static_cast<size_t>(bh) * N + static_cast<size_t>(i) * kBlock) * D;
  const uint4* q4 = reinterpret_cast<const uint4*>(Q + base);
  const uint4* k4 = reinterpret_cast<const uint4*>(K + base);
  uint4 qv[RPT], kv[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int row = rg + r * RG;
    qv[r] = __ldg(q4 + row * TPR + cg);
    kv[r] = __ldg(k4 + row * TPR + cg);
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
  for (int c = t; c < 2 * D; c += 128) {
    const int which = c / D, col = c % D;
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) s += red[which][g][col];
    float* out = which ? kbar : qbar;
    out[(static_cast<size_t>(bh) * nB + i) * D + col] = s * (1.0f / 64.0f);
  }
}

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

// ============================================================== score + select
// One CTA per (16 query blocks, head).  Scores s_ij = qbar_i . kbar_j in
// fp32 (CUDA-core FMA, fixed order over d), kept in shared memory; then one
// warp per row ranks its candidates.
constexpr int kSelRows = 16;
constexpr int kKeyChunk = 64;

template <int D, int NC>
__global__ void __launch_bounds__(256) score_select_kernel(const float* __restrict__ qbar,
                                                           const float* __restrict__ kbar,
                                                           const uint8_t* __restrict__ cls, int nB, int H,
                                                           uint64_t head_bits, int k, int cap,
                                                           int32_t* __restrict__ idx, int32_t* __restrict__ counts,
                                                           float* __restrict__ scores_out) {
  constexpr int R = kSelRows, CH = kKeyChunk, KS = D + 4, SW = NC * 32;
  extern __shared__ __align__(16) float smem_f[];
  float* qs = smem_f;         // [R][D]
  float* ks = qs + R * D;     // [CH][KS]
  float* sc = ks + CH * KS;   // [R][SW]
  const int bh = blockIdx.y, i0 = blockIdx.x * R, t = threadIdx.x;
  if (!((head_bits >> (bh % H)) & 1ull)) {
    for (int r = t; r < R; r += blockDim.x)
      if (i0 + r < nB) counts[static_cast<size_t>(bh) * nB + i0 + r] = 0;
    return;
  }
  for (int e = t; e < R * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    qs[e] = (i0 + r < nB) ? qbar[(static_cast<size_t>(bh) * nB + i0 + r) * D + c] : 0.f;
  }
  const int r = t >> 4, cl = t & 15;
  for (int j0 = 0; j0 < nB; j0 += CH) {
    __syncthreads();
    for (int e = t; e < CH * (D / 4); e += blockDim.x) {
      const int row = e / (D / 4), c4 = e % (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + row < nB) v = reinterpret_cast<const float4*>(kbar + (static_cast<size_t>(bh) * nB + j0 + row) * D)[c4];
      *reinterpret_cast<float4*>(ks + row * KS + c4 * 4) = v;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float4* qr = reinterpret_cast<const float4*>(qs + r * D);
#pragma unroll 8
    for (int c4 = 0; c4 < D / 4; ++c4) {
      const float4 a = qr[c4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 b = *reinterpret_cast<const float4*>(ks + (cl + 16 * u) * KS + c4 * 4);
        acc[u] = fmaf(a.x, b.x, acc[u]);
        acc[u] = fmaf(a.y, b.y, acc[u]);
        acc[u] = fmaf(a.z, b.z, acc[u]);
        acc[u] = fmaf(a.w, b.w, acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + cl + 16 * u;
      if (j < nB) sc[r * SW + j] = acc[u];
    }
  }
  __syncthreads();
  if (scores_out) {
    for (int rr = 0; rr < R && i0 + rr < nB; ++rr)
      for (int j = t; j < nB; j += blockDim.x)
        scores_out[(static_cast<size_t>(bh) * nB + i0 + rr) * nB + j] = sc[rr * SW + j];
  }
  const int w = t >> 5, lane = t & 31;
  for (int rr = w; rr < R; rr += 8) {
    const int i = i0 + rr;
    if (i >= nB) break;
    const uint8_t ci = cls[i];
    uint32_t keep = 0;
    if (ci == kPin) {
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int j = 32 * c + lane;
        if (j < nB && cls[j] != kDrop) keep |= 1u << c;
      }
    } else if (ci == kSparse) {
      uint32_t key[NC];
      uint32_t cand = 0, pin = 0;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const int j = 32 * c + lane;
        key[c] = 0;
        if (j < nB) {
          const uint8_t cj = cls[j];
          if (cj == kPin) {
            pin |= 1u << c;
          } else if (cj == kSparse) {
            key[c] = (j == i) ? 0xFFFFFFFFu : score_key(sc[rr * SW + j]);
            cand |= 1u << c;
          }
        }
      }
      keep = warp_topk<NC>(key, cand, k) | pin;
    }
    const int n = warp_emit<NC>(keep, idx + (static_cast<size_t>(bh) * nB + i) * cap);
    if (lane == 0) counts[static_cast<size_t>(bh) * nB + i] = n;
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

template <int NC>
__global__ void __launch_bounds__(128) pattern_kernel(const uint8_t* __restrict__ cls,
                                                      const int32_t* __restrict__ sparse_rank, int nB, int kind,
                                                      int W, int G, int r, int k, int BH, int H,
                                                      uint64_t head_bits, int cap, int32_t* __restrict__ idx,
                                                      int32_t* __restrict__ counts) {
  __shared__ int32_t lst[4][NC * 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 4 + w;
  if (i >= nB) return;
  const uint8_t ci = cls[i];
  const bool row_global = ci == kSparse && kind != 0 && kind != 3 && sparse_rank[i] < G;
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
      } else {
        const bool glob = sparse_rank[j] < G;
        const bool cover = (kind == 1) ? window_cover(i, j, W) : dilated_cover(i, j, W, r);
        if (glob || cover) win |= 1u << c;
      }
    }
    keep = pin | win;
    if (kind == 0) keep |= warp_topk<NC>(key, cand, k);
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

template <int D, int NC>
static cudaError_t launch_score_select_t(const float* qbar, const float* kbar, const sa_layout* L, int BH, int H,
                                         uint64_t head_bits, int k, int32_t* idx, int32_t* counts,
                                         float* scores_out, cudaStream_t s) {
  constexpr size_t smem = (kSelRows * D + kKeyChunk * (D + 4) + kSelRows * NC * 32) * sizeof(float);
  static int configured_dev_mask = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured_dev_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(score_select_kernel<D, NC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << (dev & 31);
  }
  dim3 grid((L->nB + kSelRows - 1) / kSelRows, BH);
  score_select_kernel<D, NC><<<grid, 256, smem, s>>>(qbar, kbar, L->d_cls, L->nB, H, head_bits, k, L->cap, idx,
                                                     counts, scores_out);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_score_select_d(int nc, const float* qbar, const float* kbar, const sa_layout* L, int BH,
                                         int H, uint64_t head_bits, int k, int32_t* idx, int32_t* counts,
                                         float* scores_out, cudaStream_t s) {
  switch (nc) {
    case 2: return launch_score_select_t<D, 2>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 4: return launch_score_select_t<D, 4>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 8: return launch_score_select_t<D, 8>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 12: return launch_score_select_t<D, 12>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 17: return launch_score_select_t<D, 17>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 24: return launch_score_select_t<D, 24>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    case 32: return launch_score_select_t<D, 32>(qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_select(const sa_layout* L, const void* Q, const void* K, int B, int H, int d, int k,
                          uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out, void* ws,
                          cudaStream_t s) {
  const int BH = B * H, nB = L->nB;
  const int nc = chunks_for(nB);
  if (nc < 0) return cudaErrorInvalidValue;
  if (k >= L->n_cand && scores_out == nullptr)  // the budget covers every candidate: dense lists, no scoring
    return launch_pattern(L, 3, 0, 0, 1, k, B, H, head_bits, idx, counts, s);
  const WsLayout wl = ws_layout(B, H, L->N, d);
  float* qbar = reinterpret_cast<float*>(static_cast<char*>(ws) + wl.qbar);
  float* kbar = reinterpret_cast<float*>(static_cast<char*>(ws) + wl.kbar);
  dim3 pgrid(nB, BH);
  if (d == 128)
    pool_kernel<128><<<pgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
                                           qbar, kbar, L->N, nB, H, head_bits);
  else
    pool_kernel<64><<<pgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
                                          qbar, kbar, L->N, nB, H, head_bits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (d == 128) return launch_score_select_d<128>(nc, qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
  return launch_score_select_d<64>(nc, qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
}

// ============================================================== selection without allocation
// For callers that cannot allocate device memory (see sa_select_blocks_noalloc
// in sa.h): the pooled block means live in this fixed, file-scope device
// array instead of the caller's workspace.  Every process that loads the
// library holds it on every GPU it uses until exit.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB: q-bar and k-bar, fp32
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

cudaError_t launch_select_noalloc(const sa_layout* L, const void* Q, const void* K, int B, int H, int d, int k,
                                  uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out,
                                  cudaStream_t s) {
  const int BH = B * H, nB = L->nB;
  const int nc = chunks_for(nB);
  if (nc < 0) return cudaErrorInvalidValue;
  if (k >= L->n_cand && scores_out == nullptr)  // dense lists: no scratch used
    return launch_pattern(L, 3, 0, 0, 1, k, B, H, head_bits, idx, counts, s);
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  // q-bar and k-bar are written in full for every active head by the pooling
  // kernel before the scoring kernel reads them: nothing needs clearing.
  float* qbar = static_cast<float*>(scratch);
  float* kbar = qbar + static_cast<size_t>(BH) * nB * d;
  dim3 pgrid(nB, BH);
  if (d == 128)
    pool_kernel<128><<<pgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
                                           qbar, kbar, L->N, nB, H, head_bits);
  else
    pool_kernel<64><<<pgrid, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
                                          qbar, kbar, L->N, nB, H, head_bits);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (d == 128) return launch_score_select_d<128>(nc, qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
  return launch_score_select_d<64>(nc, qbar, kbar, L, BH, H, head_bits, k, idx, counts, scores_out, s);
}

template <int NC>
static void launch_pattern_t(const sa_layout* L, int kind, int W, int G, int r, int k, int BH, int H,
                             uint64_t head_bits, int32_t* idx, int32_t* counts, cudaStream_t s) {
  pattern_kernel<NC><<<(L->nB + 3) / 4, 128, 0, s>>>(L->d_cls, L->d_sparse_rank, L->nB, kind, W, G, r, k, BH, H,
                                                     head_bits, L->cap, idx, counts);
}

cudaError_t launch_pattern(const sa_layout* L, int kind, int W, int G, int r, int k, int B, int H,
                           uint64_t head_bits, int32_t* idx, int32_t* counts, cudaStream_t s) {
  const int BH = B * H;
  switch (chunks_for(L->nB)) {
    case 2: launch_pattern_t<2>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 4: launch_pattern_t<4>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 8: launch_pattern_t<8>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 12: launch_pattern_t<12>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 17: launch_pattern_t<17>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 24: launch_pattern_t<24>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
    case 32: launch_pattern_t<32>(L, kind, W, G, r, k, BH, H, head_bits, idx, counts, s); break;
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
