// C ABI entry points: argument validation, the layout cache, workspace
// sizing, device-error readback and status strings.  Every entry point
// validates before launching anything; hot calls never allocate or sync.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(int B, int H, int N, int d) {
  WsLayout w;
  const size_t BH = static_cast<size_t>(B) * H, nB = static_cast<size_t>(N) / kBlock;
  size_t off = 0;
  w.header = off;
  off += sizeof(WsHeader);
  const size_t img = (nB + 127) / 128 * 128 * d * sizeof(float);  // one head's operand images (hi or lo)
  w.qbar = off;
  off += align256(2 * BH * img);
  w.kbar = off;
  off += align256(2 * BH * img);
  w.scores = off;
  off += align256(BH * nB * nB * sizeof(float));
  w.items = off;
  off += align256(BH * nB * sizeof(int4));
  w.ulist = off;
  off += align256(3 * BH * nB * nB * sizeof(int32_t));
  w.lens = off;
  off += align256(3 * BH * nB * sizeof(int32_t));
  w.totals = off;
  off += align256(BH * ((nB + 7) / 8) * 3 * sizeof(int32_t));
  w.kmask = off;
  off += align256(static_cast<size_t>(B) * nB * sizeof(uint64_t));
  w.total = off;
  return w;
}

// Diagnostic for the bounded waits: one thread waits, through the same
// helper every kernel uses, on a shared-memory barrier that nothing arrives
// at.  After the wait limit the helper records kErrTimeout in *err and the
// kernel returns; nothing traps, and the context stays usable.
__global__ void wait_timeout_kernel(int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, err);  // phase 0 never completes: runs out
}

// Diagnostic: records error bits in a device error word, as a kernel that
// found a fault would.
__global__ void set_error_kernel(int* err, int bits) { atomicOr(err, bits); }

cudaError_t device_info(DeviceInfo* out) {
  static DeviceInfo cache[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 64 && cache[dev].id == dev) {
    *out = cache[dev];
    return cudaSuccess;
  }
  DeviceInfo di;
  di.id = dev;
  if ((e = cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&di.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&di.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return e;
  if (dev < 64) cache[dev] = di;
  *out = di;
  return cudaSuccess;
}

}  // namespace sa

using namespace sa;

namespace {

std::mutex g_layout_mu;
std::vector<sa_layout*> g_layouts;  // cache of live layouts

sa_status check_device(DeviceInfo* di) {
  if (device_info(di) != cudaSuccess) return SA_ERR_CUDA;
  if (di->cc_major != 10) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Head mask -> bit set; checks H and the minimum number of active heads.
sa_status head_bits_of(const uint8_t* mask, int H, int min_active, uint64_t* bits) {
  if (H <= 0 || H > kMaxHeads) return SA_ERR_SHAPE;
  if (min_active < 0) return SA_ERR_INVALID_ARG;
  uint64_t b = 0;
  int active = 0;
  for (int h = 0; h < H; ++h)
    if (!mask || mask[h]) {
      b |= 1ull << h;
      ++active;
    }
  if (active < min_active) return SA_ERR_HEAD_MASK;
  *bits = b;
  return SA_OK;
}

bool density_ok(float rho) { return std::isfinite(rho) && rho > 0.f && rho <= 1.f; }

sa_status ws_ok(const void* ws, size_t ws_bytes, int B, int H, int N, int d) {
  if (!ws) return SA_ERR_WORKSPACE;
  if (!aligned16(ws)) return SA_ERR_WORKSPACE;
  if (ws_bytes < ws_layout(B, H, N, d).total) return SA_ERR_WORKSPACE;
  return SA_OK;
}

sa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// An NVTX range around one ABI call (a no-op unless a profiler is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

}  // namespace

extern "C" {

const char* sa_version(void) { return "prompt_aware_head_b200 0.1 (sm_100a)"; }

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_SHAPE: return "unsupported shape";
    case SA_ERR_LAYOUT: return "segments do not tile the sequence";
    case SA_ERR_HEAD_MASK: return "fewer active heads than the minimum";
    case SA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SA_ERR_BAD_INDEX: return "block index out of range or count above capacity";
    case SA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case SA_ERR_UNSUPPORTED: return "device is not sm_100 (B200 class)";
    case SA_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

int sa_budget(float density, int n_cand) {
  if (n_cand <= 0) return 0;
  long k = static_cast<long>(std::floor(static_cast<double>(density) * n_cand + 1e-4));
  if (k < 1) k = 1;
  if (k > n_cand) k = n_cand;
  return static_cast<int>(k);
}

sa_status sa_budget_schedule(const float* densities, int n_steps, int n_cand, int32_t* k_out, uint8_t* dense_out) {
  if (!densities || n_steps < 1 || n_cand < 1) return SA_ERR_INVALID_ARG;
  float seen[2];
  int n_seen = 0;
  for (int t = 0; t < n_steps; ++t) {
    const float r = densities[t];
    if (!density_ok(r)) return SA_ERR_INVALID_ARG;
    bool known = false;
    for (int v = 0; v < n_seen; ++v) known = known || seen[v] == r;
    if (known) continue;
    if (n_seen == 2) return SA_ERR_INVALID_ARG;
    seen[n_seen++] = r;
  }
  for (int t = 0; t < n_steps; ++t) {
    const int k = sa_budget(densities[t], n_cand);
    if (k_out) k_out[t] = k;
    if (dense_out) dense_out[t] = k == n_cand ? 1 : 0;
  }
  return SA_OK;
}

int sa_sparse_stage_decline(int N, int min_seq_len, int is_self_attention, int has_token_mask, int is_causal) {
  const int min_len = min_seq_len >= 0 ? min_seq_len : SA_DEFAULT_MIN_SEQ_LEN;  // 0: no floor
  int why = 0;
  if (!is_self_attention) why |= SA_DECLINE_NOT_SELF_ATTENTION;
  if (has_token_mask != SA_TOKEN_MASK_NONE && has_token_mask != SA_TOKEN_MASK_KEY_PADDING) why |= SA_DECLINE_TOKEN_MASK;
  if (is_causal) why |= SA_DECLINE_CAUSAL;
  if (N < min_len) why |= SA_DECLINE_SHORT;
  return why;
}

int sa_sparse_stage_gate(int N, int min_seq_len, int is_self_attention, int has_token_mask, int is_causal) {
  return sa_sparse_stage_decline(N, min_seq_len, is_self_attention, has_token_mask, is_causal) == 0 ? 1 : 0;
}

sa_status sa_build_layout(const sa_segment* segs, int nseg, int N, int block, sa_layout** out) {
  if (!out || nseg < 0 || (nseg > 0 && !segs)) return SA_ERR_INVALID_ARG;
  if (block != kBlock || N <= 0 || N % block != 0 || N / block > kMaxBlocks) return SA_ERR_SHAPE;
  // segments must tile [0, N) in order with known kinds
  int pos = 0;
  for (int s = 0; s < nseg; ++s) {
    if (segs[s].kind < SA_SEG_TEXT || segs[s].kind > SA_SEG_OTHER || segs[s].start != pos || segs[s].len <= 0 ||
        segs[s].len > N - pos)
      return SA_ERR_LAYOUT;
    pos += segs[s].len;
  }
  if (nseg > 0 && pos != N) return SA_ERR_LAYOUT;
  DeviceInfo di;
  sa_status st = check_device(&di);
  if (st != SA_OK) return st;

  std::lock_guard<std::mutex> lock(g_layout_mu);
  for (sa_layout* L : g_layouts) {
    if (L->N == N && L->block == block && L->device == di.id && static_cast<int>(L->segs.size()) == nseg &&
        (nseg == 0 || std::memcmp(L->segs.data(), segs, sizeof(sa_segment) * nseg) == 0)) {
      ++L->refcount;
      *out = L;
      return SA_OK;
    }
  }
  sa_layout* L = new sa_layout();
  L->N = N;
  L->block = block;
  L->nB = N / block;
  L->segs.assign(segs, segs + nseg);
  L->cls.assign(L->nB, static_cast<uint8_t>(kSparse));
  // Per block: count image and padding tokens over the runs that overlap it.
  for (int b = 0; b < L->nB; ++b) {
    if (nseg == 0) break;
    const int lo = b * block, hi = lo + block;
    int img = 0, pad = 0;
    for (int s = 0; s < nseg; ++s) {
      const int a0 = std::max(lo, segs[s].start), a1 = std::min(hi, segs[s].start + segs[s].len);
      if (a1 <= a0) continue;
      if (segs[s].kind == SA_SEG_IMAGE) img += a1 - a0;
      if (segs[s].kind == SA_SEG_PAD) pad += a1 - a0;
    }
    L->cls[b] = img == block ? kSparse : (pad == block ? kDrop : kPin);
  }
  std::vector<int32_t> rank(L->nB, -1);
  int r = 0;
  for (int b = 0; b < L->nB; ++b) {
    if (L->cls[b] == kPin) ++L->n_pin;
    if (L->cls[b] == kDrop) ++L->n_drop;
    if (L->cls[b] == kSparse) rank[b] = r++;
    if (L->cls[b] == kPin) L->pin_bits[b >> 5] |= 1u << (b & 31);
    if (L->cls[b] == kSparse) L->sparse_bits[b >> 5] |= 1u << (b & 31);
  }
  L->n_cand = r;
  L->cap = L->nB - L->n_drop;
  L->device = di.id;
  cudaError_t e = cudaMalloc(&L->d_cls, L->nB);
  if (e == cudaSuccess) e = cudaMalloc(&L->d_sparse_rank, sizeof(int32_t) * L->nB);
  if (e == cudaSuccess) e = cudaMemcpy(L->d_cls, L->cls.data(), L->nB, cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(L->d_sparse_rank, rank.data(), sizeof(int32_t) * L->nB, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(L->d_cls);
    cudaFree(L->d_sparse_rank);
    delete L;
    return SA_ERR_CUDA;
  }
  L->refcount = 1;
  g_layouts.push_back(L);
  *out = L;
  return SA_OK;
}

sa_status sa_layout_info(const sa_layout* L, int* nB, int* n_pin, int* n_drop, int* n_cand, int* cap) {
  if (!L) return SA_ERR_INVALID_ARG;
  if (nB) *nB = L->nB;
  if (n_pin) *n_pin = L->n_pin;
  if (n_drop) *n_drop = L->n_drop;
  if (n_cand) *n_cand = L->n_cand;
  if (cap) *cap = L->cap;
  return SA_OK;
}

sa_status sa_layout_classes(const sa_layout* L, uint8_t* cls_out, int nB) {
  if (!L || !cls_out || nB != L->nB) return SA_ERR_INVALID_ARG;
  std::memcpy(cls_out, L->cls.data(), L->nB);
  return SA_OK;
}

sa_status sa_layout_release(sa_layout* L) {
  if (!L) return SA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_layout_mu);
  for (size_t i = 0; i < g_layouts.size(); ++i) {
    if (g_layouts[i] != L) continue;
    if (--L->refcount == 0) {
      cudaFree(L->d_cls);
      cudaFree(L->d_sparse_rank);
      g_layouts.erase(g_layouts.begin() + i);
      delete L;
    }
    return SA_OK;
  }
  return SA_ERR_INVALID_ARG;
}

sa_status sa_workspace_size(int B, int H, int N, int d, size_t* bytes) {
  if (!bytes) return SA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || H > kMaxHeads || N <= 0 || N % kBlock || N / kBlock > kMaxBlocks || (d != 64 && d != 128))
    return SA_ERR_SHAPE;
  *bytes = ws_layout(B, H, N, d).total;
  return SA_OK;
}

sa_status sa_workspace_init(void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (!ws || ws_bytes < sizeof(WsHeader)) return SA_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, sizeof(WsHeader), reinterpret_cast<cudaStream_t>(stream)));
}

// Synchronises the stream, reads the device error word at `word`, clears it
// when set, and maps its bits to a status (the first recorded kind).
static sa_status read_and_clear_error(int* word, cudaStream_t s) {
  if (cudaStreamSynchronize(s) != cudaSuccess) return SA_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SA_ERR_CUDA;
  if (err && cudaMemset(word, 0, sizeof(int)) != cudaSuccess) return SA_ERR_CUDA;
  if (err & kErrBadIndex) return SA_ERR_BAD_INDEX;
  if (err & kErrTimeout) return SA_ERR_TIMEOUT;
  if (err & kErrSmemAlign) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

sa_status sa_check(void* ws, sa_stream_t stream) {
  if (!ws) return SA_ERR_WORKSPACE;
  return read_and_clear_error(&static_cast<WsHeader*>(ws)->err, reinterpret_cast<cudaStream_t>(stream));
}

sa_status sa_check_noalloc(sa_stream_t stream) {
  DeviceInfo di;
  sa_status st = check_device(&di);
  if (st != SA_OK) return st;
  int* word = nullptr;
  if (noalloc_error_word(&word) != cudaSuccess) return SA_ERR_CUDA;
  return read_and_clear_error(word, reinterpret_cast<cudaStream_t>(stream));
}

// Key/value heads: at least one, and H a whole number of groups of them.
static bool kv_heads_ok(int H, int H_kv) { return H_kv >= 1 && H_kv <= H && H % H_kv == 0; }

sa_status sa_select_blocks_gqa(const sa_layout* L, const void* Q, const void* K, int B, int H, int H_kv, int d,
                               float density, const uint8_t* head_mask, int min_active, int32_t* idx,
                               int32_t* counts, float* scores_out, void* ws, size_t ws_bytes, sa_stream_t stream) {
  CallRange range("sa_select_blocks");
  if (!L || !Q || !K || !idx || !counts) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return SA_ERR_INVALID_ARG;
  if (B <= 0 || (d != 64 && d != 128) || !kv_heads_ok(H, H_kv)) return SA_ERR_SHAPE;
  if (static_cast<long long>(B) * H * L->N >= (1ll << 31)) return SA_ERR_SHAPE;
  if (!density_ok(density)) return SA_ERR_INVALID_ARG;
  uint64_t bits = 0;
  sa_status st = head_bits_of(head_mask, H, min_active, &bits);
  if (st != SA_OK) return st;
  if ((st = ws_ok(ws, ws_bytes, B, H, L->N, d)) != SA_OK) return st;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  if (di.id != L->device) return SA_ERR_INVALID_ARG;
  const int k = sa_budget(density, L->n_cand);
  return from_cuda(launch_select(L, Q, K, B, H, H_kv, d, k, bits, idx, counts, scores_out, ws,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

sa_status sa_select_blocks(const sa_layout* L, const void* Q, const void* K, int B, int H, int d, float density,
                           const uint8_t* head_mask, int min_active, int32_t* idx, int32_t* counts,
                           float* scores_out, void* ws, size_t ws_bytes, sa_stream_t stream) {
  return sa_select_blocks_gqa(L, Q, K, B, H, H, d, density, head_mask, min_active, idx, counts, scores_out, ws,
                              ws_bytes, stream);
}

sa_status sa_select_blocks_noalloc_gqa(const sa_layout* L, const void* Q, const void* K, int B, int H, int H_kv,
                                       int d, float density, const uint8_t* head_mask, int min_active, int32_t* idx,
                                       int32_t* counts, float* scores_out, sa_stream_t stream) {
  CallRange range("sa_select_blocks_noalloc");
  if (!L || !Q || !K || !idx || !counts) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K)) return SA_ERR_INVALID_ARG;
  if (B <= 0 || (d != 64 && d != 128) || !kv_heads_ok(H, H_kv)) return SA_ERR_SHAPE;
  if (static_cast<long long>(B) * H * L->N >= (1ll << 31)) return SA_ERR_SHAPE;
  if (!density_ok(density)) return SA_ERR_INVALID_ARG;
  uint64_t bits = 0;
  sa_status st = head_bits_of(head_mask, H, min_active, &bits);
  if (st != SA_OK) return st;
  // a cap on the call's size (not its footprint, which the head groups keep
  // within the array): the fp32 block means of Q and K of every head at once
  const size_t need = 2ull * B * H * L->nB * d * sizeof(float);
  if (need > select_noalloc_limit()) return SA_ERR_WORKSPACE;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  if (di.id != L->device) return SA_ERR_INVALID_ARG;
  const int k = sa_budget(density, L->n_cand);
  return from_cuda(launch_select_noalloc(L, Q, K, B, H, H_kv, d, k, bits, idx, counts, scores_out,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

sa_status sa_select_blocks_noalloc(const sa_layout* L, const void* Q, const void* K, int B, int H, int d,
                                   float density, const uint8_t* head_mask, int min_active, int32_t* idx,
                                   int32_t* counts, float* scores_out, sa_stream_t stream) {
  return sa_select_blocks_noalloc_gqa(L, Q, K, B, H, H, d, density, head_mask, min_active, idx, counts, scores_out,
                                      stream);
}

sa_status sa_pattern_mask(const sa_layout* L, const sa_pattern* p, int B, int H, float density,
                          const uint8_t* head_mask, int min_active, int32_t* idx, int32_t* counts,
                          sa_stream_t stream) {
  CallRange range("sa_pattern_mask");
  if (!L || !p || !idx || !counts) return SA_ERR_INVALID_ARG;
  if (B <= 0) return SA_ERR_SHAPE;
  if (p->kind < SA_PAT_RADIAL || p->kind > SA_PAT_RANDOM) return SA_ERR_INVALID_ARG;
  const bool budgeted = p->kind == SA_PAT_RADIAL || p->kind == SA_PAT_RANDOM;  // k from the density
  if (budgeted && !density_ok(density)) return SA_ERR_INVALID_ARG;
  if (!budgeted && (p->window_tokens < 0 || p->n_global_blocks < 0)) return SA_ERR_INVALID_ARG;
  if (p->kind == SA_PAT_DILATED && p->dilation < 1) return SA_ERR_INVALID_ARG;
  uint64_t bits = 0;
  sa_status st = head_bits_of(head_mask, H, min_active, &bits);
  if (st != SA_OK) return st;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  if (di.id != L->device) return SA_ERR_INVALID_ARG;
  const int k = budgeted ? sa_budget(density, L->n_cand) : 0;
  const int kind = p->kind == SA_PAT_RANDOM ? 4 : p->kind;  // the kernel's kind 3 is the dense lists
  return from_cuda(launch_pattern(L, kind, budgeted ? 0 : p->window_tokens, budgeted ? 0 : p->n_global_blocks,
                                  p->kind == SA_PAT_DILATED ? p->dilation : 1, k, B, H, bits, idx, counts,
                                  reinterpret_cast<cudaStream_t>(stream), p->seed));
}

static sa_status attention_args_ok(const void* Q, const void* K, const void* V, const void* O, int B, int H,
                                   int H_kv, int N, int d, float* scale) {
  if (!Q || !K || !V || !O) return SA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || H > kMaxHeads || (d != 64 && d != 128) || !kv_heads_ok(H, H_kv)) return SA_ERR_SHAPE;
  if (N <= 0 || N % kBlock || N / kBlock > kMaxBlocks) return SA_ERR_SHAPE;
  if (static_cast<long long>(B) * H * N >= (1ll << 31)) return SA_ERR_SHAPE;
  if (!std::isfinite(*scale) || *scale < 0.f) return SA_ERR_INVALID_ARG;
  if (*scale == 0.f) *scale = 1.0f / std::sqrt(static_cast<float>(d));
  return SA_OK;
}

sa_status sa_attention_plan(const int32_t* idx, const int32_t* counts, int B, int H, int N, int d, int cap,
                            const uint8_t* head_mask, int min_active, void* ws, size_t ws_bytes, sa_stream_t stream) {
  CallRange range("sa_attention_plan");
  if (!idx || !counts) return SA_ERR_INVALID_ARG;
  if (B <= 0 || (d != 64 && d != 128) || N <= 0 || N % kBlock || N / kBlock > kMaxBlocks) return SA_ERR_SHAPE;
  if (cap < 1 || cap > N / kBlock) return SA_ERR_SHAPE;
  // union lists of all three pairing strides are addressed with int32 offsets
  if (3ll * B * H * (N / kBlock) * (N / kBlock) >= (1ll << 31)) return SA_ERR_SHAPE;
  uint64_t bits = 0;
  sa_status st = head_bits_of(head_mask, H, min_active, &bits);
  if (st != SA_OK) return st;
  if ((st = ws_ok(ws, ws_bytes, B, H, N, d)) != SA_OK) return st;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  return from_cuda(launch_attention_plan(idx, counts, B, H, N, d, cap, bits, ws,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

sa_status sa_attention_run_masked(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N, int d,
                                  const uint8_t* key_mask, const uint8_t* head_mask, int min_active,
                                  float softmax_scale, void* O, void* ws, size_t ws_bytes, sa_stream_t stream) {
  CallRange range("sa_attention_run");
  sa_status st = attention_args_ok(Q, K, V, O, B, H, H_kv, N, d, &softmax_scale);
  if (st != SA_OK) return st;
  if (key_mask && !aligned16(key_mask)) return SA_ERR_INVALID_ARG;
  uint64_t bits = 0;
  if ((st = head_bits_of(head_mask, H, min_active, &bits)) != SA_OK) return st;
  if ((st = ws_ok(ws, ws_bytes, B, H, N, d)) != SA_OK) return st;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  return from_cuda(launch_attention_run(Q, K, V, B, H, H_kv, N, d, key_mask, bits, softmax_scale, O, ws,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

sa_status sa_attention_run_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N, int d,
                               const uint8_t* head_mask, int min_active, float softmax_scale, void* O, void* ws,
                               size_t ws_bytes, sa_stream_t stream) {
  return sa_attention_run_masked(Q, K, V, B, H, H_kv, N, d, nullptr, head_mask, min_active, softmax_scale, O, ws,
                                 ws_bytes, stream);
}

sa_status sa_attention_run(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                           const uint8_t* head_mask, int min_active, float softmax_scale, void* O, void* ws,
                           size_t ws_bytes, sa_stream_t stream) {
  return sa_attention_run_gqa(Q, K, V, B, H, H, N, d, head_mask, min_active, softmax_scale, O, ws, ws_bytes, stream);
}

sa_status sa_block_sparse_attention_masked(const void* Q, const void* K, const void* V, int B, int H, int H_kv,
                                           int N, int d, const int32_t* idx, const int32_t* counts, int cap,
                                           const uint8_t* key_mask, const uint8_t* head_mask, int min_active,
                                           float softmax_scale, void* O, void* ws, size_t ws_bytes,
                                           sa_stream_t stream) {
  sa_status st = attention_args_ok(Q, K, V, O, B, H, H_kv, N, d, &softmax_scale);
  if (st != SA_OK) return st;
  if (key_mask && !aligned16(key_mask)) return SA_ERR_INVALID_ARG;
  if ((st = sa_attention_plan(idx, counts, B, H, N, d, cap, head_mask, min_active, ws, ws_bytes, stream)) != SA_OK)
    return st;
  return sa_attention_run_masked(Q, K, V, B, H, H_kv, N, d, key_mask, head_mask, min_active, softmax_scale, O, ws,
                                 ws_bytes, stream);
}

sa_status sa_block_sparse_attention_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N,
                                        int d, const int32_t* idx, const int32_t* counts, int cap,
                                        const uint8_t* head_mask, int min_active, float softmax_scale, void* O,
                                        void* ws, size_t ws_bytes, sa_stream_t stream) {
  return sa_block_sparse_attention_masked(Q, K, V, B, H, H_kv, N, d, idx, counts, cap, nullptr, head_mask,
                                          min_active, softmax_scale, O, ws, ws_bytes, stream);
}

sa_status sa_block_sparse_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                    const int32_t* idx, const int32_t* counts, int cap, const uint8_t* head_mask,
                                    int min_active, float softmax_scale, void* O, void* ws, size_t ws_bytes,
                                    sa_stream_t stream) {
  return sa_block_sparse_attention_gqa(Q, K, V, B, H, H, N, d, idx, counts, cap, head_mask, min_active,
                                       softmax_scale, O, ws, ws_bytes, stream);
}

sa_status sa_dense_attention_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N, int d,
                                 float softmax_scale, void* O, void* ws, size_t ws_bytes, sa_stream_t stream) {
  CallRange range("sa_dense_attention");
  sa_status st = attention_args_ok(Q, K, V, O, B, H, H_kv, N, d, &softmax_scale);
  if (st != SA_OK) return st;
  if (!ws || !aligned16(ws) || ws_bytes < sizeof(WsHeader)) return SA_ERR_WORKSPACE;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  return from_cuda(launch_dense_attention(Q, K, V, B, H, H_kv, N, d, softmax_scale, O, ws,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

sa_status sa_dense_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                             float softmax_scale, void* O, void* ws, size_t ws_bytes, sa_stream_t stream) {
  return sa_dense_attention_gqa(Q, K, V, B, H, H, N, d, softmax_scale, O, ws, ws_bytes, stream);
}

sa_status sa_density(const int32_t* counts, int B, int H, int nB, const uint8_t* head_mask, double* over_active,
                     double* over_all, sa_stats* stats, void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (!counts) return SA_ERR_INVALID_ARG;
  if (B <= 0 || nB <= 0 || nB > kMaxBlocks) return SA_ERR_SHAPE;
  uint64_t bits = 0;
  sa_status st = head_bits_of(head_mask, H, 0, &bits);
  if (st != SA_OK) return st;
  if (!ws || !aligned16(ws) || ws_bytes < sizeof(WsHeader)) return SA_ERR_WORKSPACE;
  DeviceInfo di;
  if ((st = check_device(&di)) != SA_OK) return st;
  unsigned long long tiles = 0;
  if (launch_density(counts, B, H, nB, bits, ws, &tiles, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SA_ERR_CUDA;
  const int active = __builtin_popcountll(bits);
  const double cells = static_cast<double>(nB) * nB;
  const double da = active ? static_cast<double>(tiles) / (static_cast<double>(B) * active * cells) : 0.0;
  const double dall = static_cast<double>(tiles) / (static_cast<double>(B) * H * cells);
  if (over_active) *over_active = da;
  if (over_all) *over_all = dall;
  if (stats) {
    stats->density_over_active = da;
    stats->density_over_all = dall;
    stats->tiles = static_cast<int64_t>(tiles);
    stats->heads_active = active;
  }
  return SA_OK;
}

sa_status sa_debug_wait_timeout(void* ws, size_t ws_bytes, sa_stream_t stream) {
  if (!ws || !aligned16(ws) || ws_bytes < sizeof(WsHeader)) return SA_ERR_WORKSPACE;
  DeviceInfo di;
  sa_status st = check_device(&di);
  if (st != SA_OK) return st;
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(&static_cast<WsHeader*>(ws)->err);
  return from_cuda(cudaGetLastError());
}

sa_status sa_debug_noalloc_error(int bits, sa_stream_t stream) {
  if (bits != SA_ERR_BAD_INDEX && bits != SA_ERR_TIMEOUT) return SA_ERR_INVALID_ARG;
  DeviceInfo di;
  sa_status st = check_device(&di);
  if (st != SA_OK) return st;
  int* word = nullptr;
  if (noalloc_error_word(&word) != cudaSuccess) return SA_ERR_CUDA;
  set_error_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      word, bits == SA_ERR_BAD_INDEX ? kErrBadIndex : kErrTimeout);
  return from_cuda(cudaGetLastError());
}

sa_status sa_debug_exp2(const float* y, float* out, int n, sa_stream_t stream) {
  if (!y || !out || n < 0) return SA_ERR_INVALID_ARG;
  DeviceInfo di;
  sa_status st = check_device(&di);
  if (st != SA_OK) return st;
  return from_cuda(launch_exp2_poly(y, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
