/*
 * CPU oracle for block-sparse attention driven by a per-input mask.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only tests/, the package smoke check and bench.py's
 * cpu_baseline / reference arm use it.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only through the seeded input
 * generator (workloads/), which holds none of the method's arithmetic.
 *
 * Plain, slow, obviously correct: fp64 everywhere, one loop per definition,
 * no blocking or fusion.  OpenMP only splits independent output rows.
 *
 * Sources (the web pages this method is described on):
 *   [SDN]  SD.Next ("automatic") commit log, modules/attention/sparse:
 *          "selector" paragraph (mean-pool, score, keep within budget, no scale
 *          or softmax, diagonal kept, dense when the budget covers all),
 *          "layout" paragraph (image/video sparsifiable; text, conditioning,
 *          audio, unknown pin rows and columns; padding dropped; straddling
 *          tile pins), "radial" paragraph (band around the diagonal at the
 *          selector's density, same pins), "host sync" paragraph (ranking
 *          instead of a host-sized top-k; density read back on demand).
 *   [HS]   haagenti_sparse crate docs and lib.rs: AttentionMask (which heads
 *          to compute), MIN_ACTIVE_HEADS = 4.
 *   [GLO]  inferensys glossary "Sparse Attention": sliding window (W tokens
 *          left and right), dilated (i +- r, i +- 2r, ...), global tokens
 *          (attend to all, attended by all), block-sparse (only connected
 *          block pairs computed).
 *
 * Readings where the pages are silent (the CUDA library takes the same ones):
 *   budget k = clamp(floor(rho*C + 1e-4), 1, C) with C the sparsifiable
 *   candidates; the diagonal is forced and counts in k; ties break to the
 *   lower block index; -0 ranks as +0; lists are emitted in ascending block
 *   order; pinned rows are dense over non-dropped columns; dropped rows and
 *   skipped heads give count 0 and O = 0; softmax scale 1/sqrt(d); kept tiles
 *   are computed whole (no token mask inside a tile).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_SEG_TEXT = 0, OR_SEG_PAD = 1, OR_SEG_IMAGE = 2, OR_SEG_OTHER = 3 };
enum { OR_PIN = 0, OR_SPARSE = 1, OR_DROP = 2 };
enum { OR_PAT_RADIAL = 0, OR_PAT_WINDOW_GLOBAL = 1, OR_PAT_DILATED = 2, OR_PAT_RANDOM = 3 };

static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * Block classes from token segments [SDN "layout" paragraph].
 * A block whose tokens are all image/video is SPARSE; all padding is DROP;
 * anything else (text, other, or a mix of kinds: a straddling tile) is PIN.
 * With no segments the whole sequence is image [SDN: "without a layout the
 * whole sequence is sparsified"].  Returns 0 on success, -1 on bad segments
 * (not tiling [0, N) in order, or an unknown kind).
 */
int oracle_layout(const int32_t* segs, int nseg, int N, int block, uint8_t* cls) {
  if (N <= 0 || block <= 0 || N % block) return -1;
  int nB = N / block;
  int* kind = (int*)malloc(sizeof(int) * (size_t)N);
  if (!kind) return -1;
  if (nseg == 0) {
    for (int n = 0; n < N; ++n) kind[n] = OR_SEG_IMAGE;
  } else {
    int pos = 0;
    for (int s = 0; s < nseg; ++s) {
      int k = segs[3 * s], st = segs[3 * s + 1], len = segs[3 * s + 2];
      if (k < 0 || k > 3 || st != pos || len <= 0 || st + len > N) { free(kind); return -1; }
      for (int n = st; n < st + len; ++n) kind[n] = k;
      pos += len;
    }
    if (pos != N) { free(kind); return -1; }
  }
  for (int b = 0; b < nB; ++b) {
    int n_img = 0, n_pad = 0;
    for (int n = b * block; n < (b + 1) * block; ++n) {
      if (kind[n] == OR_SEG_IMAGE) ++n_img;
      if (kind[n] == OR_SEG_PAD) ++n_pad;
    }
    if (n_img == block) cls[b] = OR_SPARSE;
    else if (n_pad == block) cls[b] = OR_DROP;
    else cls[b] = OR_PIN;
  }
  free(kind);
  return 0;
}

/*
 * Mean of each block of rows [SDN "selector": "mean-pools query and key
 * tiles"].  X is bf16 bits, [BH][N][d]; out is [BH][nB][d] fp64.
 */
void oracle_pool(const uint16_t* X, int BH, int N, int d, int block, double* out) {
  int nB = N / block;
#pragma omp parallel for schedule(static)
  for (int bh = 0; bh < BH; ++bh)
    for (int i = 0; i < nB; ++i)
      for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int r = 0; r < block; ++r)
          s += bf16_to_double(X[((size_t)bh * N + (size_t)i * block + r) * d + c]);
        out[((size_t)bh * nB + i) * d + c] = s / block;
      }
}

/*
 * The key/value head that query head bh = b*H + h reads when H query heads
 * share Hkv key/value heads [SDN "selector": scoring runs on query heads, so
 * grouped attention needs no key expansion]: consecutive groups of H/Hkv
 * query heads share one, b*Hkv + h / (H/Hkv).  Hkv = H is plain multi-head.
 */
static int kv_head(int bh, int H, int Hkv) { return (bh / H) * Hkv + (bh % H) / (H / Hkv); }

/*
 * Tile-pair scores s[i][j] = qbar_i . kbar_j, no scale and no softmax
 * [SDN "selector": top-k is invariant under both], on query heads: qbar is
 * [BH][nB][d] (BH = B*H), kbar [B*Hkv][nB][d], s [BH][nB][nB] fp64.
 */
void oracle_scores(const double* qbar, const double* kbar, int BH, int H, int Hkv, int nB, int d, double* s) {
#pragma omp parallel for schedule(static)
  for (int bh = 0; bh < BH; ++bh) {
    int kh = kv_head(bh, H, Hkv);
    for (int i = 0; i < nB; ++i)
      for (int j = 0; j < nB; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c)
          acc += qbar[((size_t)bh * nB + i) * d + c] * kbar[((size_t)kh * nB + j) * d + c];
        s[((size_t)bh * nB + i) * nB + j] = acc;
      }
  }
}

/* Budget in candidates [SDN "selector": a fraction of the sparsifiable candidates]. */
int oracle_budget(float density, int C) {
  if (C <= 0) return 0;
  long k = (long)floor((double)density * (double)C + 1e-4);
  if (k < 1) k = 1;
  if (k > C) k = C;
  return (int)k;
}

typedef struct { double key; int j; } cand_t;
static int cand_cmp(const void* a, const void* b) {
  const cand_t* x = (const cand_t*)a;
  const cand_t* y = (const cand_t*)b;
  if (x->key > y->key) return -1;   /* higher score first */
  if (x->key < y->key) return 1;
  return (x->j < y->j) ? -1 : (x->j > y->j);  /* then lower block index */
}

/* Emit the kept columns of one row in ascending block order. */
static int emit_row(const uint8_t* keep, int nB, int32_t* row_idx) {
  int c = 0;
  for (int j = 0; j < nB; ++j)
    if (keep[j]) row_idx[c++] = j;
  return c;
}

/* Pinned rows are dense over non-dropped columns; dropped rows are empty. */
static int fixed_row(const uint8_t* cls, int nB, int i, uint8_t* keep) {
  memset(keep, 0, (size_t)nB);
  if (cls[i] == OR_DROP) return 1;
  if (cls[i] == OR_PIN) {
    for (int j = 0; j < nB; ++j) keep[j] = (cls[j] != OR_DROP);
    return 1;
  }
  for (int j = 0; j < nB; ++j) keep[j] = (cls[j] == OR_PIN);  /* pinned columns of a sparse row */
  return 0;
}

/*
 * Rank-select [SDN "selector" + "layout"].  scores [BH][nB][nB] (the GPU's
 * fp32 scores widened exactly, or the oracle's own fp64 scores).  For each
 * active head and sparse row: the diagonal is forced first, the remaining
 * k-1 slots go to the highest-scoring sparse candidates (stable sort by
 * score descending, block index ascending), pinned columns are added,
 * dropped columns never appear.  head_mask [H] (NULL = all heads), heads of
 * bh are bh % H.  idx [BH][nB][cap], counts [BH][nB].
 */
void oracle_select(const double* scores, const uint8_t* cls, int BH, int H, int nB, float density,
                   const uint8_t* head_mask, int cap, int32_t* idx, int32_t* counts) {
  int C = 0;
  for (int j = 0; j < nB; ++j) C += (cls[j] == OR_SPARSE);
  int k = oracle_budget(density, C);
#pragma omp parallel
  {
    uint8_t* keep = (uint8_t*)malloc((size_t)nB);
    cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nB > 0 ? nB : 1));
#pragma omp for schedule(static)
    for (int bh = 0; bh < BH; ++bh) {
      int active = head_mask ? head_mask[bh % H] != 0 : 1;
      for (int i = 0; i < nB; ++i) {
        int32_t* row_idx = idx + ((size_t)bh * nB + i) * cap;
        if (!active) { counts[(size_t)bh * nB + i] = 0; continue; }
        if (!fixed_row(cls, nB, i, keep)) {
          int nc = 0;
          for (int j = 0; j < nB; ++j) {
            if (cls[j] != OR_SPARSE) continue;
            double s = scores[((size_t)bh * nB + i) * nB + j];
            if (s == 0.0) s = 0.0;                /* -0 ranks as +0 */
            cand[nc].key = (j == i) ? INFINITY : s;  /* diagonal forced */
            cand[nc].j = j;
            ++nc;
          }
          qsort(cand, (size_t)nc, sizeof(cand_t), cand_cmp);
          for (int r = 0; r < k && r < nc; ++r) keep[cand[r].j] = 1;
        }
        counts[(size_t)bh * nB + i] = emit_row(keep, nB, row_idx);
      }
    }
    free(keep);
    free(cand);
  }
}

/* Smallest |q - key| over q in block I and key in block J (block cover test). */
static long block_gap(int i, int j, int block) {
  long lo = (long)(j - i) * block - (block - 1);
  long hi = (long)(j - i) * block + (block - 1);
  if (lo <= 0 && hi >= 0) return 0;
  return lo > 0 ? lo : -hi;
}

/* True when some q in block I and key in J have key - q = delta, |delta| <= W, delta % r == 0. */
static int dilated_cover(int i, int j, int block, int W, int r) {
  long lo = (long)(j - i) * block - (block - 1);
  long hi = (long)(j - i) * block + (block - 1);
  if (lo < -W) lo = -W;
  if (hi > W) hi = W;
  for (long delta = lo; delta <= hi; ++delta)
    if (delta % r == 0) return 1;
  return 0;
}

/*
 * Control patterns at the same pins and drops [SDN "radial" paragraph;
 * GLO sliding window, dilated, global].  kind 0 RADIAL: the selector's k,
 * candidates ranked by |i - j| then j.  kind 1 WINDOW_GLOBAL: block cover
 * of |q - key| <= W plus the first G sparse blocks as global rows and
 * columns.  kind 2 DILATED: block cover of {key : |q - key| <= W,
 * (q - key) % r == 0}, plus G globals when G > 0.
 */
/*
 * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014): output number n >= 1 of the generator seeded
 * with `seed`.  The state advances by the odd constant 0x9E3779B97F4A7C15 per
 * output; an output is the state after its advance, put through the mix
 * (xor-shift 30, multiply, xor-shift 27, multiply, xor-shift 31).
 */
static uint64_t splitmix64_nth(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

int oracle_pattern(const uint8_t* cls, int nB, int block, int kind, int W, int G, int r, float density,
                   int BH, int H, const uint8_t* head_mask, int cap, int32_t* idx, int32_t* counts,
                   uint64_t seed) {
  if (kind < 0 || kind > 3) return -1;
  if (kind == OR_PAT_DILATED && r <= 0) return -1;
  int C = 0;
  for (int j = 0; j < nB; ++j) C += (cls[j] == OR_SPARSE);
  int k = oracle_budget(density, C);
  uint8_t* global = (uint8_t*)calloc((size_t)nB, 1);
  int g = 0;
  for (int j = 0; j < nB && g < G && kind != OR_PAT_RADIAL && kind != OR_PAT_RANDOM; ++j)
    if (cls[j] == OR_SPARSE) { global[j] = 1; ++g; }
  uint8_t* keep = (uint8_t*)malloc((size_t)nB);
  cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nB > 0 ? nB : 1));
  for (int bh = 0; bh < BH; ++bh) {
    int active = head_mask ? head_mask[bh % H] != 0 : 1;
    for (int i = 0; i < nB; ++i) {
      int32_t* row_idx = idx + ((size_t)bh * nB + i) * cap;
      if (!active) { counts[(size_t)bh * nB + i] = 0; continue; }
      if (!fixed_row(cls, nB, i, keep)) {
        if (kind == OR_PAT_RADIAL) {
          int nc = 0;
          for (int j = 0; j < nB; ++j) {
            if (cls[j] != OR_SPARSE) continue;
            cand[nc].key = -(double)abs(i - j);   /* nearer first */
            cand[nc].j = j;
            ++nc;
          }
          qsort(cand, (size_t)nc, sizeof(cand_t), cand_cmp);
          for (int q = 0; q < k && q < nc; ++q) keep[cand[q].j] = 1;
        } else if (kind == OR_PAT_RANDOM) {
          /* [GLO random: each query attends to a fixed set of keys sampled
           * uniformly at random]: the diagonal, then the k - 1 other sparse
           * blocks ranked by the top 21 bits of output i*nB + j + 1, larger
           * first (ties: lower block), the same for every head */
          int nc = 0;
          for (int j = 0; j < nB; ++j) {
            if (cls[j] != OR_SPARSE) continue;
            cand[nc].key = (j == i) ? INFINITY
                                    : (double)(splitmix64_nth(seed, (uint64_t)i * (uint64_t)nB + (uint64_t)j + 1) >> 43);
            cand[nc].j = j;
            ++nc;
          }
          qsort(cand, (size_t)nc, sizeof(cand_t), cand_cmp);
          for (int q = 0; q < k && q < nc; ++q) keep[cand[q].j] = 1;
        } else if (global[i]) {
          for (int j = 0; j < nB; ++j) keep[j] = (cls[j] != OR_DROP);
        } else {
          for (int j = 0; j < nB; ++j) {
            if (cls[j] != OR_SPARSE) continue;
            int in = global[j];
            if (kind == OR_PAT_WINDOW_GLOBAL) in |= block_gap(i, j, block) <= W;
            else in |= dilated_cover(i, j, block, W, r);
            if (in) keep[j] = 1;
          }
        }
      }
      counts[(size_t)bh * nB + i] = emit_row(keep, nB, row_idx);
    }
  }
  free(global);
  free(keep);
  free(cand);
  return 0;
}

/*
 * Attention over the selected tiles [GLO block-sparse; SDN flex consumer:
 * every selected tile computed in full].  For each requested query row:
 * S = q . K^T * scale, -inf outside the kept tiles, softmax, times V.
 * Rows whose list is empty, and skipped heads, give O = 0.  Q is bf16 bits
 * [BH][N][d]; K and V are [B*Hkv][N][d], query head bh reading key/value
 * head kv_head(bh); rows lists flat row ids bh*N + n (NULL = every row);
 * out is [nrows][d] fp64.
 * key_mask (NULL = none) is a token-level mask over keys, [B][N] bytes, 1 =
 * may be attended: a key inside a kept tile counts only where it is set
 * [SDN "masked_block": a backend takes the attention mask and the block
 * mask together].  A row none of whose kept keys is set gives O = 0.
 */
void oracle_attention(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int BH, int H, int Hkv, int N, int d,
                      int block, const int32_t* idx, const int32_t* counts, int cap, const uint8_t* head_mask,
                      const uint8_t* key_mask, double scale, const int64_t* rows, int64_t nrows, double* out) {
  int nB = N / block;
  if (!rows) nrows = (int64_t)BH * N;
#pragma omp parallel
  {
    uint8_t* keep = (uint8_t*)malloc((size_t)N);
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* q = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < nrows; ++t) {
      int64_t row = rows ? rows[t] : t;
      int bh = (int)(row / N), n = (int)(row % N), i = n / block, kh = kv_head(bh, H, Hkv);
      double* o = out + (size_t)t * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      int active = head_mask ? head_mask[bh % H] != 0 : 1;
      int cnt = active ? counts[(size_t)bh * nB + i] : 0;
      if (cnt <= 0) continue;
      memset(keep, 0, (size_t)N);
      const int32_t* li = idx + ((size_t)bh * nB + i) * cap;
      for (int e = 0; e < cnt; ++e)
        for (int r = 0; r < block; ++r) keep[(size_t)li[e] * block + r] = 1;
      if (key_mask) {
        const uint8_t* km = key_mask + (size_t)(bh / H) * N;
        int any = 0;
        for (int key = 0; key < N; ++key) {
          keep[key] = keep[key] && km[key];
          any |= keep[key];
        }
        if (!any) continue;
      }
      for (int c = 0; c < d; ++c) q[c] = bf16_to_double(Q[((size_t)bh * N + n) * d + c]);
      double mx = -INFINITY;
      for (int key = 0; key < N; ++key) {
        if (!keep[key]) { s[key] = -INFINITY; continue; }
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[c] * bf16_to_double(K[((size_t)kh * N + key) * d + c]);
        s[key] = acc * scale;
        if (s[key] > mx) mx = s[key];
      }
      double den = 0.0;
      for (int key = 0; key < N; ++key) {
        if (!keep[key]) continue;
        double p = exp(s[key] - mx);
        den += p;
        for (int c = 0; c < d; ++c) o[c] += p * bf16_to_double(V[((size_t)kh * N + key) * d + c]);
      }
      for (int c = 0; c < d; ++c) o[c] /= den;
    }
    free(keep);
    free(s);
    free(q);
  }
}

/* Realized tile density [SDN "host sync": density read back only on demand]. */
void oracle_density(const int32_t* counts, int BH, int H, int nB, const uint8_t* head_mask,
                    double* over_active, double* over_all) {
  double tiles = 0.0;
  int active_bh = 0;
  for (int bh = 0; bh < BH; ++bh) {
    int active = head_mask ? head_mask[bh % H] != 0 : 1;
    if (!active) continue;
    ++active_bh;
    for (int i = 0; i < nB; ++i) tiles += counts[(size_t)bh * nB + i];
  }
  *over_active = active_bh ? tiles / ((double)active_bh * nB * nB) : 0.0;
  *over_all = BH ? tiles / ((double)BH * nB * nB) : 0.0;
}
