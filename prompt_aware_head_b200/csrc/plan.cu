// Attention work plan: pairs of 64-row query blocks of a head that share a
// 128-row tile of the attention kernel, each with the sorted union of the two
// block lists, ordered longest first (the attention kernel consumes them).
#include <mutex>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

// ---------------------------------------------------------------- planner
// Two kernels:
//  1. plan_rows, parallel over (head, 8 query blocks): each query block's list
//     as a bitmap over key blocks (validating every index and count), then for
//     each pairing stride s = 1, 2, 4 the union size and sorted union list of
//     every pair, and per-CTA partial sums of the union sizes;
//  2. plan_order, one CTA per head: the stride with the smallest summed union,
//     its pairs ordered by union length (longest first) by rank counting, at
//     the head's place in the concatenated item list.
constexpr int kWords = kMaxBlocks / 32;  // bitmap words per row
__device__ __forceinline__ int stride_of(int si) { return 1 << si; }  // pairing strides 1, 2, 4

__device__ __forceinline__ int pair_partner(int a, int s, int nB) { return (a + s < nB) ? a + s : -1; }
__device__ __forceinline__ bool pair_first(int a, int s) { return ((a / s) & 1) == 0; }

// One CTA per 8 aligned query blocks of a head (one warp per block).  Every
// pair (a, a + s) with a / s even lies inside an aligned group of 2s <= 8
// blocks, so the CTA holds both rows of each of its pairs for s = 1, 2, 4:
// it builds the rows' bitmaps, then for each stride each pair's union size
// (summed into the CTA's partial total) and its sorted union list with
// membership bits.  lens3[si] gives the union length per first block (-1 for
// blocks that are not first under stride s).
__global__ void __launch_bounds__(256) plan_rows_kernel(const int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ counts, int nB, int cap, int H,
                                                        uint64_t head_bits, int32_t* __restrict__ ulist3,
                                                        int* __restrict__ lens3, int* __restrict__ partials,
                                                        int* __restrict__ err) {
  __shared__ uint32_t bm[8][kWords];
  __shared__ int part[8][3];
  grid_dep_wait();
  const int bh = blockIdx.y, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * 8 + w, BH = gridDim.y;
  if (!((head_bits >> (bh % H)) & 1ull)) return;
  const int nwords = (nB + 31) >> 5;
  bm[w][lane] = 0u;
  __syncwarp();
  if (i < nB) {
    int cnt = counts[static_cast<size_t>(bh) * nB + i];
    if (cnt > cap || cnt < 0) {
      if (lane == 0) atomicOr(err, kErrBadIndex);
      cnt = cnt < 0 ? 0 : cap;
    }
    const int32_t* lst = idx + (static_cast<size_t>(bh) * nB + i) * cap;
    for (int e = lane; e < cnt; e += 32) {
      const int j = lst[e];
      if (j < 0 || j >= nB) {
        atomicOr(err, kErrBadIndex);
        continue;
      }
      atomicOr(&bm[w][j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  const size_t plane = static_cast<size_t>(BH) * nB;  // entries per stride in lens3 (x nB in ulist3)
#pragma unroll
  for (int si = 0; si < 3; ++si) {
    const int s = stride_of(si);
    int u = 0;
    if (i < nB) {
      if (!pair_first(i, s)) {
        if (lane == 0) lens3[si * plane + static_cast<size_t>(bh) * nB + i] = -1;
      } else {
        const int b = pair_partner(i, s, nB);
        const uint32_t wa = lane < nwords ? bm[w][lane] : 0u;
        const uint32_t wb = (b >= 0 && lane < nwords) ? bm[w + s][lane] : 0u;
        uint32_t un = wa | wb;
        const int cnt = __popc(un);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int pos = incl - cnt;
        int32_t* out = ulist3 + (si * plane + static_cast<size_t>(bh) * nB + i) * nB;
        while (un) {  // lane q writes the union entries of key blocks 32q .. 32q+31, ascending
          const int bit = __ffs(un) - 1;
          un &= un - 1;
          const uint32_t mbits = ((wa >> bit) & 1u) | (((wb >> bit) & 1u) << 1);
          out[pos++] = static_cast<int32_t>((32 * lane + bit) | (mbits << 16));
        }
        u = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0) lens3[si * plane + static_cast<size_t>(bh) * nB + i] = u;
      }
    }
    if (lane == 0) part[w][si] = u;
  }
  __syncthreads();
  if (threadIdx.x < 3) {
    int sum = 0;
    for (int r = 0; r < 8; ++r) sum += part[r][threadIdx.x];
    partials[(static_cast<size_t>(bh) * gridDim.x + blockIdx.x) * 3 + threadIdx.x] = sum;
  }
}

constexpr int kOrderThreads = 512;
constexpr int kOrderHeads = 1024;  // heads whose sums plan_order keeps in shared memory

// Pairs of a head for stride s: first blocks a with (a / s) even.
__device__ __forceinline__ int pairs_of(int nB, int s) {
  return (nB / (2 * s)) * s + min(nB % (2 * s), s);
}

// Stride index (0, 1, 2 for s = 1, 2, 4) with the smallest summed union of
// head h (the smaller stride on ties), from the per-CTA partial sums.
__device__ __forceinline__ int best_stride_of(const int* partials, int nparts, int h) {
  int tot[3] = {0, 0, 0};
  for (int p = 0; p < nparts; ++p)
#pragma unroll
    for (int si = 0; si < 3; ++si) tot[si] += partials[(static_cast<size_t>(h) * nparts + p) * 3 + si];
  int best = 0;
  for (int si = 1; si < 3; ++si)
    if (tot[si] < tot[best]) best = si;
  return best;
}

// Per head: the pairing stride with the smallest summed union; its pairs
// ordered by union length, longest first (rank counting over unique keys),
// at closed-form offsets (the pair counts of the heads before) in the global
// item list; with `front`, each active head's longest pair moves to the
// front of the list (one per head, heads in order).  Items point into the
// chosen stride's union lists.
__global__ void __launch_bounds__(kOrderThreads) plan_order_kernel(const int* __restrict__ lens3,
                                                                   const int* __restrict__ partials, int nparts,
                                                                   int nB, int BH, int H, uint64_t head_bits,
                                                                   int front, int4* __restrict__ items,
                                                                   int* __restrict__ n_items) {
  __shared__ uint32_t keys[kMaxBlocks];
  __shared__ int tot[kOrderHeads * 3];  // summed union lengths per (head, stride) when BH <= kOrderHeads
  __shared__ int nkeys, base_sh, total_sh, act_sh, nact_sh;
  grid_dep_launch();  // the attention kernel may set up on the SMs this small grid leaves idle
  grid_dep_wait();
  const int bh = blockIdx.x, t = threadIdx.x;
  const bool shared_sums = BH <= kOrderHeads;
  if (t == 0) {
    nkeys = 0;
    base_sh = 0;
    total_sh = 0;
    act_sh = 0;
    nact_sh = 0;
  }
  if (shared_sums) {  // all threads add up the per-CTA partial sums of every head
    for (int e = t; e < BH * 3; e += kOrderThreads) tot[e] = 0;
    __syncthreads();
    for (int e = t; e < BH * nparts; e += kOrderThreads) {
      const int h = e / nparts;
      if (!((head_bits >> (h % H)) & 1ull)) continue;
#pragma unroll
      for (int si = 0; si < 3; ++si) atomicAdd(&tot[h * 3 + si], partials[static_cast<size_t>(e) * 3 + si]);
    }
  }
  __syncthreads();
  auto best_of = [&](int h) {
    if (!shared_sums) return best_stride_of(partials, nparts, h);
    int best = 0;
    for (int si = 1; si < 3; ++si)
      if (tot[h * 3 + si] < tot[h * 3 + best]) best = si;
    return best;
  };
  int my_base = 0, my_total = 0, my_act = 0, my_nact = 0;
  for (int h = t; h < BH; h += kOrderThreads) {
    const bool on = (head_bits >> (h % H)) & 1ull;
    const int p = on ? pairs_of(nB, stride_of(best_of(h))) : 0;
    my_total += p;
    my_nact += on ? 1 : 0;
    if (h < bh) {
      my_base += p;
      my_act += on ? 1 : 0;
    }
  }
  if (my_base) atomicAdd(&base_sh, my_base);
  if (my_total) atomicAdd(&total_sh, my_total);
  if (my_act) atomicAdd(&act_sh, my_act);
  if (my_nact) atomicAdd(&nact_sh, my_nact);
  __syncthreads();
  if (bh == 0 && t == 0) *n_items = total_sh;
  if (!((head_bits >> (bh % H)) & 1ull)) return;
  // With `front` (launches that take items from the work queue) every active
  // head's longest item (rank 0: on the workloads with a pinned text block,
  // the pair holding that block, dense over every non-dropped key block) goes
  // to the front of the whole list, head by head, and the rest follow
  // head-major, longest first within a head: the long items start first and
  // the list ends on short ones.  Without it the list is plainly head-major.
  const int base = base_sh, act = act_sh, nact = nact_sh;
  const int si = best_of(bh), s = stride_of(si);
  const size_t plane = static_cast<size_t>(BH) * nB;
  const int* lens = lens3 + si * plane + static_cast<size_t>(bh) * nB;
  for (int a = t; a < nB; a += kOrderThreads) {
    const int len = lens[a];
    if (len >= 0) keys[atomicAdd(&nkeys, 1)] = (static_cast<uint32_t>(0xFFFF - len) << 16) | static_cast<uint32_t>(a);
  }
  __syncthreads();
  const int n = nkeys;
  for (int e = t; e < n; e += kOrderThreads) {
    const uint32_t k = keys[e];
    int rank = 0;
    for (int f = 0; f < n; ++f) rank += keys[f] < k;  // keys are unique: ranks form a permutation
    const int a = static_cast<int>(k & 0xFFFFu);
    const int b = pair_partner(a, s, nB);
    int4 v;
    v.x = bh;
    v.y = a | ((b < 0 ? kNoBlock : b) << 16);
    v.z = 0xFFFF - static_cast<int>(k >> 16);
    v.w = static_cast<int>((si * plane + static_cast<size_t>(bh) * nB + a) * nB);
    items[front ? (rank == 0 ? act : nact + (base - act) + (rank - 1)) : base + rank] = v;
  }
}

cudaError_t launch_attention_plan(const int32_t* idx, const int32_t* counts, int B, int H, int N, int d, int cap,
                                  uint64_t head_bits, void* ws, cudaStream_t s) {
  const int BH = B * H, nB = N / kBlock, nparts = (nB + 7) / 8;
  const WsLayout wl = ws_layout(B, H, N, d);
  char* base = static_cast<char*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base + wl.header);
  int4* items = reinterpret_cast<int4*>(base + wl.items);
  int32_t* ulist = reinterpret_cast<int32_t*>(base + wl.ulist);
  int* lens = reinterpret_cast<int*>(base + wl.lens);
  int* partials = reinterpret_cast<int*>(base + wl.totals);
  cudaError_t e = launch_pdl(plan_rows_kernel, dim3(nparts, BH), dim3(256), 0, s, idx, counts, nB, cap, H, head_bits,
                             ulist, lens, partials, &hdr->err);
  if (e != cudaSuccess) return e;
  const int front = use_queue(static_cast<long long>(B) * __builtin_popcountll(head_bits) * ((nB + 1) / 2));
  return launch_pdl(plan_order_kernel, dim3(BH), dim3(kOrderThreads), 0, s, static_cast<const int*>(lens),
                    static_cast<const int*>(partials), nparts, nB, BH, H, head_bits, front, items, &hdr->n_items);
}

}  // namespace sa
