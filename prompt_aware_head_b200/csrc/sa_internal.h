// Host-side internals shared by the C ABI (api.cu) and the kernel launchers.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/sa.h"

struct sa_layout {
  int N = 0, block = 64, nB = 0;
  int n_pin = 0, n_drop = 0, n_cand = 0, cap = 0;
  std::vector<sa_segment> segs;
  std::vector<uint8_t> cls;         // host copy of the block classes
  int device = -1;
  uint8_t* d_cls = nullptr;         // device [nB] block classes
  int32_t* d_sparse_rank = nullptr; // device [nB]: index among SPARSE blocks, -1 otherwise
  // block classes as bit masks over 32-block words (bit b of word c: block
  // 32 c + b); blocks past nB are in neither (DROP)
  uint32_t pin_bits[32] = {};
  uint32_t sparse_bits[32] = {};
  int refcount = 0;
};

namespace sa {

// Launches a kernel that may overlap the end of the previous kernel in its
// stream (programmatic dependent launch); the kernel calls grid_dep_wait()
// before it touches anything that kernel wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Workspace layout (byte offsets from the caller's workspace base).
struct WsLayout {
  size_t header = 0;        // WsHeader (256 B)
  size_t qbar = 0, kbar = 0;  // block means as tf32 hi / lo operand images: [2][BH][row tiles][d/32][128][32]
  size_t scores = 0;        // fp32 [BH][nB][nB] tile-pair scores (when the caller asks for none)
  size_t items = 0;         // int4 [BH*nB] attention work items (execution order)
  size_t ulist = 0;         // int32 [3 strides][BH][nB][nB] union lists (j | bits << 16)
  size_t lens = 0;          // int32 [3 strides][BH][nB] union length per first block of a pair (-1: not a first)
  size_t totals = 0;        // int32 [BH][nB/8 rounded up][3] per-CTA partial sums of union lengths
  size_t kmask = 0;         // uint64 [B][nB] key mask words (bit r: key 64 j + r may be attended)
  size_t total = 0;
};
WsLayout ws_layout(int B, int H, int N, int d);

struct DeviceInfo {
  int id = -1, sm_count = 0, cc_major = 0, cc_minor = 0;
};
cudaError_t device_info(DeviceInfo* out);

// Selection / pattern / density launchers (select.cu).  Hkv: key heads (H a
// multiple of Hkv; query head b H + h scores against key head b Hkv + h / (H / Hkv)).
cudaError_t launch_select(const sa_layout* L, const void* Q, const void* K, int B, int H, int Hkv, int d, int k,
                          uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out, void* ws,
                          cudaStream_t s);
// Selection with its scratch in a fixed device array (no workspace).
size_t select_noalloc_limit();
// Device address of the no-allocation path's error word for the current device.
cudaError_t noalloc_error_word(int** out);
cudaError_t launch_select_noalloc(const sa_layout* L, const void* Q, const void* K, int B, int H, int Hkv, int d,
                                  int k, uint64_t head_bits, int32_t* idx, int32_t* counts, float* scores_out,
                                  cudaStream_t s);
// kind: 0 radial, 1 window+global, 2 dilated, 3 dense (every non-drop block), 4 random (seed).
cudaError_t launch_pattern(const sa_layout* L, int kind, int W, int G, int r, int k, int B, int H,
                           uint64_t head_bits, int32_t* idx, int32_t* counts, cudaStream_t s, uint64_t seed = 0);
cudaError_t launch_density(const int32_t* counts, int B, int H, int nB, uint64_t head_bits, void* ws,
                           unsigned long long* host_tiles, cudaStream_t s);

// Whether the attention kernel takes its items from the work queue (1) or
// deals them by CTA index (0), from the number of items of the launch.
int use_queue(long long items);

// Work plan (plan.cu) and attention launchers (attention.cu).
cudaError_t launch_attention_plan(const int32_t* idx, const int32_t* counts, int B, int H, int N, int d, int cap,
                                  uint64_t head_bits, void* ws, cudaStream_t s);
cudaError_t launch_attention_run(const void* Q, const void* K, const void* V, int B, int H, int Hkv, int N, int d,
                                 const uint8_t* key_mask,
                                 uint64_t head_bits, float scale, void* O, void* ws, cudaStream_t s);
cudaError_t launch_dense_attention(const void* Q, const void* K, const void* V, int B, int H, int Hkv, int N,
                                   int d, float scale, void* O, void* ws, cudaStream_t s);

cudaError_t launch_exp2_poly(const float* y, float* out, int n, cudaStream_t s);


}  // namespace sa
