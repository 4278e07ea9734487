/*
 * sa.h - C ABI of a B200 (sm_100a) library for block-sparse attention driven
 * by a per-input mask: per-input block selection, per-(layer, head) head
 * skipping, and flash-style attention over only the selected tiles.
 *
 * Sources the operations follow (web pages describing the method):
 *   [SDN] SD.Next ("automatic") commit log for modules/attention/sparse:
 *         the "selector", "layout", "radial control", "host sync" and
 *         "flex consumer" paragraphs.
 *   [HS]  haagenti_sparse crate (docs.rs overview and lib.rs): AttentionMask,
 *         SparseKernel, SparseError, MIN_ACTIVE_HEADS = 4,
 *         DEFAULT_SPARSITY = 0.5.
 *   [GLO] inferensys glossary "Sparse Attention": sliding window, dilated,
 *         global and block-sparse patterns; CSR rows.
 *
 * Conventions shared by every call:
 *   - Tensors Q, K, V, O are bf16, row-major [B][H][N][d] on the device,
 *     contiguous, 16-byte aligned.  d is 64 or 128; N is a multiple of the
 *     block size (64).  nB = N / 64 blocks per head.
 *   - The caller owns every device buffer.  The library owns only layouts
 *     (sa_layout), which hold small device arrays allocated once per layout.
 *   - Hot calls (sa_select_blocks, sa_pattern_mask, sa_block_sparse_attention,
 *     sa_dense_attention) never allocate, never synchronise the host and
 *     never read device memory back; they enqueue kernels on `stream`.
 *   - Argument and shape errors are returned before anything is launched.
 *     Faults found on the device (an out-of-range block index, a bounded
 *     wait that ran out) set a sticky error word in the workspace header and
 *     the kernel skips the bad access; sa_check() reads and clears it.
 *   - Block lists are CSR-like rows of fixed capacity [GLO CSR]:
 *     idx[b][h][i][0 .. counts[b][h][i]) holds the kept key blocks of query
 *     block i in ascending order; slots at or beyond the count are left
 *     untouched and are unspecified.
 *   - head_mask is a HOST array of H bytes (nonzero = compute the head)
 *     [HS AttentionMask], or NULL for all heads.  H <= 64.  Fewer than
 *     min_active active heads is SA_ERR_HEAD_MASK [HS MIN_ACTIVE_HEADS];
 *     a skipped head gets counts 0 and O = 0.
 */
#ifndef SA_H_
#define SA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* sa_stream_t;

/* Error codes [HS SparseError]. */
typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, density outside (0, 1]   */
  SA_ERR_SHAPE = 2,        /* d not 64/128, N not a multiple of 64, B/H <= 0    */
  SA_ERR_LAYOUT = 3,       /* segments do not tile [0, N) in order               */
  SA_ERR_HEAD_MASK = 4,    /* fewer than min_active heads active                 */
  SA_ERR_WORKSPACE = 5,    /* workspace missing or smaller than sa_workspace_size */
  SA_ERR_BAD_INDEX = 6,    /* device: a block index outside [0, nB) or count > cap */
  SA_ERR_TIMEOUT = 7,      /* device: a bounded wait inside a kernel ran out     */
  SA_ERR_UNSUPPORTED = 8,  /* not a B200-class (sm_100) device                   */
  SA_ERR_CUDA = 9          /* a CUDA runtime call failed                         */
} sa_status;

/* Token segment kinds [SDN "layout"]: image/video tokens are sparsifiable;
 * text, conditioning, audio and unknown tokens pin their rows and columns;
 * padding is dropped. */
typedef enum {
  SA_SEG_TEXT = 0,   /* live prompt conditioning: pinned   */
  SA_SEG_PAD = 1,    /* padding: dropped                   */
  SA_SEG_IMAGE = 2,  /* image / video tokens: sparsifiable */
  SA_SEG_OTHER = 3   /* audio / unrecognised: pinned       */
} sa_seg_kind;

typedef struct {
  int32_t kind;   /* sa_seg_kind                 */
  int32_t start;  /* first token of the run      */
  int32_t len;    /* tokens in the run (> 0)     */
} sa_segment;

/* Block classes a layout assigns (exposed for tests and tools). */
typedef enum { SA_BLOCK_PIN = 0, SA_BLOCK_SPARSE = 1, SA_BLOCK_DROP = 2 } sa_block_class;

typedef struct sa_layout sa_layout;  /* opaque, library-owned, refcounted, cached */

/* Control patterns [SDN "radial control"; GLO sliding window, dilated, global, random]. */
typedef enum { SA_PAT_RADIAL = 0, SA_PAT_WINDOW_GLOBAL = 1, SA_PAT_DILATED = 2, SA_PAT_RANDOM = 3 } sa_pattern_kind;

typedef struct {
  int32_t kind;             /* sa_pattern_kind                                        */
  int32_t window_tokens;    /* W: keys with |q - key| <= W (window, dilated)          */
  int32_t n_global_blocks;  /* G: the first G sparsifiable blocks are global rows and
                               columns (window and dilated patterns)                  */
  int32_t dilation;         /* r: dilated keys satisfy (q - key) % r == 0 (r >= 1)    */
  uint64_t seed;            /* random pattern: SplitMix64 seed of the draw            */
} sa_pattern;

/* Optional per-call statistics [HS KernelStats]: filled only by sa_density. */
typedef struct {
  double density_over_active;  /* sum(counts) / (B * H_active * nB^2) */
  double density_over_all;     /* sum(counts) / (B * H * nB^2)        */
  int64_t tiles;               /* sum(counts) over active heads       */
  int32_t heads_active;        /* active heads in the mask            */
} sa_stats;

/*
 * sa_build_layout [SDN "layout" paragraph; the geometry "built once and
 * cached per layout" of the "host sync" paragraph].
 *   segs/nseg: runs that tile [0, N) in order (nseg == 0: the whole sequence
 *   is sparsifiable, as when a pipeline publishes no layout).  N % block == 0,
 *   block must be 64.  A block is PIN if it holds text/other tokens or mixes
 *   kinds (a tile straddling a boundary pins), DROP if it is all padding,
 *   SPARSE if it is all image.  *out receives a refcounted handle; an
 *   identical (N, block, segments) request returns the cached layout with its
 *   count raised.  May allocate and synchronise (once per layout, outside the
 *   hot loop).  Release with sa_layout_release.
 */
SA_API sa_status sa_build_layout(const sa_segment* segs, int nseg, int N, int block, sa_layout** out);

/* nB blocks, n_pin / n_drop / n_cand (= C, sparsifiable) blocks, and cap =
 * nB - n_drop, the capacity an idx row needs.  Any output pointer may be NULL. */
SA_API sa_status sa_layout_info(const sa_layout* L, int* nB, int* n_pin, int* n_drop, int* n_cand, int* cap);

/* Host copy of the per-block classes (sa_block_class), nB bytes. */
SA_API sa_status sa_layout_classes(const sa_layout* L, uint8_t* cls_out, int nB);

/* Drops one reference; the layout is freed when the count reaches zero. */
SA_API sa_status sa_layout_release(sa_layout* L);

/* Budget in kept candidates per sparse row [SDN "selector": a fraction of the
 * sparsifiable candidates]: clamp(floor(density * C + 1e-4), 1, C). */
SA_API int sa_budget(float density, int n_cand);

/*
 * Per-step budgets [SDN stage paragraph: budgets follow a precomputed
 * per-step schedule with at most two distinct values].  Checks a schedule
 * of n_steps densities, each finite and in (0, 1], with at most two distinct
 * values, and writes for step t:
 *   k_out[t]     = sa_budget(densities[t], n_cand);
 *   dense_out[t] = 1 when k_out[t] == n_cand (the selection then writes
 *                  dense lists without pooling or scoring), else 0.
 * Either output may be NULL.  Host memory only; no device is touched.
 * SA_ERR_INVALID_ARG for NULL densities, n_steps < 1, n_cand < 1, a density
 * outside (0, 1], or a third distinct value (nothing is written then).
 */
SA_API sa_status sa_budget_schedule(const float* densities, int n_steps, int n_cand, int32_t* k_out,
                                    uint8_t* dense_out);

/*
 * Whether a call takes the block-sparse path [SDN stage paragraph: the
 * stage gates on self attention, a minimum sequence length (8192 tokens by
 * default, the sparse/dense crossover measured there), and on the token
 * mask or causal flag a block-only mask cannot combine with; a backend that
 * takes the attention mask and the block mask together ("masked_block")
 * serves masked calls].  has_token_mask is an sa_token_mask kind:
 *   SA_TOKEN_MASK_NONE (0): no token mask;
 *   SA_TOKEN_MASK_GENERAL (1): a mask that depends on the query token (any
 *     [N][N] or per-query mask): declined, a block list cannot express it;
 *   SA_TOKEN_MASK_KEY_PADDING (2): a key padding mask, [B][N]: served by
 *     sa_block_sparse_attention_masked / sa_attention_run_masked, so it does
 *     not decline.
 * Returns 1 when is_self_attention != 0, the mask kind is NONE or
 * KEY_PADDING, is_causal == 0 and N >= min_seq_len, else 0 (stay dense).
 * The default floor is passed explicitly (SA_DEFAULT_MIN_SEQ_LEN); 0 means
 * no floor, so every length qualifies [SDN: 0 means no floor, the default is
 * stated rather than hidden behind a sentinel].  On B200 this library's
 * sparse step (selection, plan and attention at 30 % density, 24 heads of
 * 128) beats its dense kernel from about 1,900 tokens, so a caller there may
 * pass a floor of 2048.  Negative values are
 * reserved for a derived floor and act as the default until one is defined.
 * Any other mask kind counts as GENERAL.  Host only.
 */
#define SA_DEFAULT_MIN_SEQ_LEN 8192
typedef enum { SA_TOKEN_MASK_NONE = 0, SA_TOKEN_MASK_GENERAL = 1, SA_TOKEN_MASK_KEY_PADDING = 2 } sa_token_mask;
SA_API int sa_sparse_stage_gate(int N, int min_seq_len, int is_self_attention, int has_token_mask, int is_causal);

/* Why the gate above declines [SDN stage paragraph: the stage records why it
 * declined]: a bit set per failed condition, 0 when the call takes the
 * sparse path (sa_sparse_stage_gate returns 1 exactly then).  Host only. */
typedef enum {
  SA_DECLINE_NOT_SELF_ATTENTION = 1,
  SA_DECLINE_TOKEN_MASK = 2,
  SA_DECLINE_CAUSAL = 4,
  SA_DECLINE_SHORT = 8
} sa_decline_reason;
SA_API int sa_sparse_stage_decline(int N, int min_seq_len, int is_self_attention, int has_token_mask, int is_causal);

/*
 * sa_select_blocks [SDN "selector" + "host sync" paragraphs].
 * Per (batch, active head, 64-row query block i):
 *   qbar_i = mean of the 64 Q rows, kbar_j likewise (fp32 accumulation);
 *   s_ij = qbar_i . kbar_j as an fp32 value, with no scale and no softmax
 *   (computed on the tensor cores with each mean split into a tf32 part and
 *   its remainder: each product within about 2^-22 |q||k| of exact);
 *   a SPARSE row keeps its diagonal block, then the k-1 highest-scoring
 *   other SPARSE blocks (ties: lower block index; -0 ranks as +0), plus every
 *   PIN block; k = sa_budget(density, C).  A PIN row keeps every non-DROP
 *   block; a DROP row keeps nothing.  Lists are emitted in ascending order.
 * The rank is found on the device (no host-sized top-k, no readback).  When
 * k == C the budget covers every candidate and the call writes the dense
 * lists without pooling or scoring (unless scores_out is requested).
 *   Q, K:       device bf16 [B][H][N][d].
 *   idx:        device int32 [B][H][nB][cap]; counts: device int32 [B][H][nB].
 *   scores_out: device fp32 [B][H][nB][nB] or NULL; when given, every active
 *               head's scores are written (rows of inactive heads untouched).
 *   ws:         device workspace of at least sa_workspace_size bytes,
 *               header zeroed once with sa_workspace_init.
 */
SA_API sa_status sa_select_blocks(const sa_layout* L, const void* Q, const void* K, int B, int H, int d,
                           float density, const uint8_t* head_mask, int min_active,
                           int32_t* idx, int32_t* counts, float* scores_out,
                           void* ws, size_t ws_bytes, sa_stream_t stream);

/*
 * sa_select_blocks_noalloc: the same selection as sa_select_blocks, for
 * callers that cannot allocate device memory.  The pages have no counterpart:
 * this entry point exists for hosts that own all device memory and give
 * plugins no allocator, and for latency-critical code that must not call
 * cudaMalloc (which can synchronise the whole device).  It takes no
 * workspace: its scratch (the pooled block means as tensor-core operand
 * images, and the scores when scores_out is NULL) lives in one fixed array
 * of 16 MiB of device memory inside the library, which every GPU that loads
 * the library holds until the process exits.  The heads are processed in as
 * many groups as that array needs.  The call is capped at 2 * B * H * nB * d
 * * 4 <= 16 MiB (the fp32 block means of Q and K of every head at once; e.g.
 * B1 H24 N33280 d128 needs 12.8 MB): a cap on the call's size, not its
 * footprint, which grouping keeps within the array.  Larger calls return
 * SA_ERR_WORKSPACE before anything is launched.  The call allocates nothing.
 * The first call on a device looks up the array's device address for that
 * device, so make that first call before any stream capture.  All calls
 * share the one array, which keeps the last call's contents (each call
 * overwrites what it reads); calls that overlap on the GPU (two streams, or
 * two host threads) race on it, so serialise them.  Arguments and outputs
 * are otherwise those of sa_select_blocks; device-side errors are read with
 * sa_check_noalloc (below) instead of sa_check.
 */
SA_API sa_status sa_select_blocks_noalloc(const sa_layout* L, const void* Q, const void* K, int B, int H, int d,
                                          float density, const uint8_t* head_mask, int min_active,
                                          int32_t* idx, int32_t* counts, float* scores_out, sa_stream_t stream);

/* The device-side errors of sa_select_blocks_noalloc, which has no workspace
 * to record them in: its kernels set bits in an error word inside the same
 * fixed array (one per device).  sa_check_noalloc synchronises `stream`,
 * reads the current device's word, clears it, and returns SA_OK or the first
 * error recorded since the last read (as sa_check does for a workspace).
 * The word is shared by every call on the device, like the array. */
SA_API sa_status sa_check_noalloc(sa_stream_t stream);

/*
 * sa_pattern_mask [SDN "radial control"; GLO sliding window / dilated /
 * global].  Writes the same (idx, counts) a selection would, from a fixed
 * pattern honouring the same pins and drops:
 *   RADIAL: the selector's k = sa_budget(density, C) SPARSE blocks nearest to
 *     the diagonal (distance |i - j|, ties to the lower j).
 *   WINDOW_GLOBAL: SPARSE blocks j with some token pair |q - key| <= W
 *     between blocks i and j, plus the first G SPARSE blocks as global
 *     columns; those G blocks' rows are dense over non-DROP blocks.
 *   DILATED: SPARSE blocks holding some key with |q - key| <= W and
 *     (q - key) % r == 0 for some query of block i, plus G globals as above.
 *   RANDOM: the diagonal and k - 1 = sa_budget(density, C) - 1 other SPARSE
 *     blocks drawn uniformly without replacement, one draw per row for every
 *     head: block j of row i ranks by the top 21 bits of output i*nB + j + 1
 *     of SplitMix64 (Steele, Lea and Flood 2014) seeded with `seed`, larger
 *     first, ties to the lower j.
 * density is used by RADIAL and RANDOM only.  No workspace needed.
 */
SA_API sa_status sa_pattern_mask(const sa_layout* L, const sa_pattern* p, int B, int H, float density,
                          const uint8_t* head_mask, int min_active,
                          int32_t* idx, int32_t* counts, sa_stream_t stream);

/*
 * sa_block_sparse_attention [GLO block-sparse; SDN "flex consumer": every
 * selected tile is computed in full].  For each active head and query row q
 * of block i:  O_q = softmax(Q_q . K_S^T * scale) . V_S, with S the tokens of
 * the blocks idx[b][h][i][0 .. counts) (online softmax, fp32 accumulation,
 * bf16 MMA on tcgen05).  Rows with count 0 and skipped heads get O = 0.
 *   idx/counts/cap: as written by sa_select_blocks or sa_pattern_mask; any
 *     index outside [0, nB) or count > cap sets SA_ERR_BAD_INDEX on the
 *     device and the entry is skipped.
 *   softmax_scale: 0 means 1/sqrt(d).
 *   O: device bf16 [B][H][N][d], fully written.
 */
SA_API sa_status sa_block_sparse_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                    const int32_t* idx, const int32_t* counts, int cap,
                                    const uint8_t* head_mask, int min_active, float softmax_scale,
                                    void* O, void* ws, size_t ws_bytes, sa_stream_t stream);

/*
 * The two halves of sa_block_sparse_attention, for callers that reuse one
 * block list across calls or time the parts separately.
 * sa_attention_plan reads (idx, counts) and writes the work plan into the
 * workspace: the pairing of query blocks into 128-row tiles, the sorted
 * union of each pair's lists with membership bits, and the longest-first
 * work order.  sa_attention_run computes O from Q, K, V and the plan last
 * written to the same workspace (same B, H, N, d and head mask).
 */
SA_API sa_status sa_attention_plan(const int32_t* idx, const int32_t* counts, int B, int H, int N, int d, int cap,
                                   const uint8_t* head_mask, int min_active, void* ws, size_t ws_bytes,
                                   sa_stream_t stream);
SA_API sa_status sa_attention_run(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                                  const uint8_t* head_mask, int min_active, float softmax_scale, void* O, void* ws,
                                  size_t ws_bytes, sa_stream_t stream);

/* sa_dense_attention: the same kernel over every tile of every head (the
 * dense baseline the speedup is measured against). */
SA_API sa_status sa_dense_attention(const void* Q, const void* K, const void* V, int B, int H, int N, int d,
                             float softmax_scale, void* O, void* ws, size_t ws_bytes, sa_stream_t stream);

/*
 * Grouped key/value heads [SDN "selector": scoring runs on query heads, so
 * grouped attention needs no key expansion].  The _gqa forms take K (and V)
 * with H_kv heads, [B][H_kv][N][d], H a multiple of H_kv: query head h reads
 * key/value head h / (H / H_kv), so each run of H / H_kv consecutive query
 * heads shares one.  Selection pools each needed key head once and scores
 * every query head against its key head's block means; nothing is copied
 * or expanded.  Q, O, idx, counts, scores_out, the head mask and the
 * workspace keep their H-head shapes and sizes (sa_workspace_size(B, H, N,
 * d) covers both forms).  H_kv == H is exactly the plain form (which calls
 * these); H_kv < 1, H_kv > H or H % H_kv != 0 returns SA_ERR_SHAPE before
 * any launch.  Everything else is as in the plain form of each call.
 */
SA_API sa_status sa_select_blocks_gqa(const sa_layout* L, const void* Q, const void* K, int B, int H, int H_kv,
                                      int d, float density, const uint8_t* head_mask, int min_active,
                                      int32_t* idx, int32_t* counts, float* scores_out,
                                      void* ws, size_t ws_bytes, sa_stream_t stream);
SA_API sa_status sa_select_blocks_noalloc_gqa(const sa_layout* L, const void* Q, const void* K, int B, int H,
                                              int H_kv, int d, float density, const uint8_t* head_mask,
                                              int min_active, int32_t* idx, int32_t* counts, float* scores_out,
                                              sa_stream_t stream);
SA_API sa_status sa_block_sparse_attention_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv,
                                               int N, int d, const int32_t* idx, const int32_t* counts, int cap,
                                               const uint8_t* head_mask, int min_active, float softmax_scale,
                                               void* O, void* ws, size_t ws_bytes, sa_stream_t stream);
SA_API sa_status sa_attention_run_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N,
                                      int d, const uint8_t* head_mask, int min_active, float softmax_scale, void* O,
                                      void* ws, size_t ws_bytes, sa_stream_t stream);
SA_API sa_status sa_dense_attention_gqa(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N,
                                        int d, float softmax_scale, void* O, void* ws, size_t ws_bytes,
                                        sa_stream_t stream);

/*
 * Token-level key mask inside the kept tiles [SDN "masked_block": a backend
 * takes the attention mask and the block mask together].  key_mask is a
 * device byte array [B][N], 16-byte aligned, nonzero where key n of batch b
 * may be attended (a padding mask), or NULL for none.  Query row q of block
 * i attends to key n only when n's block is in idx[b][h][i][0 .. counts) and
 * key_mask[b][n] != 0; a row left with no key gets O = 0.  The mask is packed
 * into one 64-bit word per (batch, key block) in the workspace (one small
 * kernel), and the attention kernel applies it only to kept tiles whose word
 * is neither all ones nor zero (a zero word skips the tile).  Other arguments
 * as in the _gqa forms (H_kv = H for plain multi-head attention).
 */
SA_API sa_status sa_block_sparse_attention_masked(const void* Q, const void* K, const void* V, int B, int H,
                                                  int H_kv, int N, int d, const int32_t* idx, const int32_t* counts,
                                                  int cap, const uint8_t* key_mask, const uint8_t* head_mask,
                                                  int min_active, float softmax_scale, void* O, void* ws,
                                                  size_t ws_bytes, sa_stream_t stream);
SA_API sa_status sa_attention_run_masked(const void* Q, const void* K, const void* V, int B, int H, int H_kv, int N,
                                         int d, const uint8_t* key_mask, const uint8_t* head_mask, int min_active,
                                         float softmax_scale, void* O, void* ws, size_t ws_bytes,
                                         sa_stream_t stream);

/*
 * sa_density [SDN "host sync": density is read back only when something
 * asks].  The only call that reads device memory back: it synchronises
 * `stream`.  Any of the outputs may be NULL.
 */
SA_API sa_status sa_density(const int32_t* counts, int B, int H, int nB, const uint8_t* head_mask,
                     double* over_active, double* over_all, sa_stats* stats,
                     void* ws, size_t ws_bytes, sa_stream_t stream);

/* Workspace bytes needed by every call for these sizes (selection and
 * attention regions are disjoint, so one workspace serves both). */
SA_API sa_status sa_workspace_size(int B, int H, int N, int d, size_t* bytes);

/* Zeroes the workspace header (the sticky error word); enqueued on stream. */
SA_API sa_status sa_workspace_init(void* ws, size_t ws_bytes, sa_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace error word, and
 * returns SA_OK or the first device-side error recorded. */
SA_API sa_status sa_check(void* ws, sa_stream_t stream);

SA_API const char* sa_status_string(sa_status s);

/* Diagnostic: out[i] = 2^y[i] computed by the polynomial exponential the
 * attention softmax uses for part of its exponentials (round-to-nearest range
 * reduction, degree-3 minimax polynomial on [-0.5, 0.5], relative error below
 * 1e-4 for y >= -125; results for y < -125 are 2^-125).  Device arrays of n
 * floats.  Not on the hot path; for tests. */
SA_API sa_status sa_debug_exp2(const float* y, float* out, int n, sa_stream_t stream);

/* Diagnostic: one kernel waits, through the same bounded-wait helper every
 * kernel uses, on a barrier that nothing completes.  After the wait limit
 * (2 s) it records SA_ERR_TIMEOUT in the workspace error word and returns,
 * so the next sa_check reports SA_ERR_TIMEOUT and the device stays usable.
 * Not on the hot path; for tests. */
SA_API sa_status sa_debug_wait_timeout(void* ws, size_t ws_bytes, sa_stream_t stream);

/* Diagnostic: records `status` (SA_ERR_BAD_INDEX or SA_ERR_TIMEOUT, else
 * SA_ERR_INVALID_ARG) in the no-allocation path's error word of the current
 * device with one small kernel, as a faulting selection kernel would, so the
 * next sa_check_noalloc reports it.  Not on the hot path; for tests. */
SA_API sa_status sa_debug_noalloc_error(int status, sa_stream_t stream);

/* Library version string. */
SA_API const char* sa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_H_ */
