/*
 * oracle.c -- plain, slow, fp64 CPU oracle for paged decode attention and the
 * two cache-maintenance operations. TEST INFRASTRUCTURE ONLY: the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg call it; the
 * product path never does. It shares no code with the CUDA library.
 *
 * What it computes, and where the pages say so:
 *
 *  oracle_gather      Rebuild one sequence's contiguous K (or V) from the pool
 *                     through its block table and cut it to the sequence
 *                     length: token i lives in physical block table[i / bs] at
 *                     row i % bs.  "17. vLLM PagedAttention" (datawhalechina),
 *                     Step 4, get_physical_cache (concatenate the table's
 *                     blocks, keep the first seq_len rows); "五十三：vLLM-
 *                     PagedAttention" section 8 (the kernel finds the history
 *                     through the block table).
 *  oracle_decode      For each (sequence b, query head hq): gather K and V of
 *                     KV head hq / (Hq / Hkv), then textbook softmax attention
 *                     of the one query vector over the ctx_b cached tokens:
 *                     s_i = scale * q . k_i, m = max s, w_i = exp(s_i - m),
 *                     o = sum_i w_i v_i / sum_i w_i.  "17. vLLM PagedAttention"
 *                     Step 2 (gather the scattered blocks, attention dot
 *                     product with the current query); "vLLM 与 LLM 推理部署实战"
 *                     section 2.3 (FlashAttention reading non-contiguous
 *                     blocks: the result is ordinary attention).
 *                     The pages give no formula; this is the plain reading.
 *                     GQA grouping hq / G (contiguous groups) and scale
 *                     1/sqrt(D) are readings too: the pages are silent.
 *  oracle_decode_partitioned
 *                     The same attention cut into contiguous partitions of
 *                     partition_size tokens from token 0. Each partition j
 *                     yields m_j, l_j = sum exp(s_i - m_j), acc_j = sum
 *                     exp(s_i - m_j) v_i; the merge takes M = max m_j,
 *                     L = sum l_j exp(m_j - M), o = sum exp(m_j - M) acc_j / L,
 *                     skipping empty partitions. Not on the pages; it is the
 *                     exact algebra of splitting a softmax sum.
 *  oracle_reshape_and_cache
 *                     Scatter each new token's K and V row to its slot:
 *                     block slot / bs, row slot % bs; negative slot = skip.
 *                     "17. vLLM PagedAttention" Step 4, allocate_for_decode
 *                     (the new token goes into the sequence's current block).
 *  oracle_copy_blocks Copy-on-write: every (src, dst) pair copies the whole
 *                     src block (all rows, all heads) of K and V to dst, all
 *                     sources read before any write. "vLLM 与 LLM 推理部署实战"
 *                     section 2.2 (a write to a shared block copies it whole).
 *
 * Inputs are read exactly: f32 as is; f16 and bf16 are widened to double from
 * their bit patterns by the IEEE-754 definitions of those formats.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2 };
enum { OR_OK = 0, OR_ERR_ARG = 1, OR_ERR_BLOCK = 2, OR_ERR_SLOT = 3, OR_ERR_PAIR = 4,
       OR_ERR_NOMEM = 5 };

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
static double f16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1, e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);                 /* subnormal: f * 2^(1-15-10) */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(f | 0x400), e - 25);    /* (1.f) * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16: the upper half of a binary32 pattern */
static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float x;
  memcpy(&x, &u, sizeof x);
  return (double)x;
}

static int esize_of(int dtype) { return dtype == OR_F32 ? 4 : 2; }

static double elem(const void* base, size_t i, int dtype) {
  if (dtype == OR_F32) return (double)((const float*)base)[i];
  uint16_t h = ((const uint16_t*)base)[i];
  return dtype == OR_F16 ? f16_to_double(h) : bf16_to_double(h);
}

/* out[i, d] = pool[table[i / bs], i % bs, h, d] for i < ctx (one KV head). */
static int gather_head(double* out, const void* pool, int dtype, const int32_t* table,
                       int ctx, int Hkv, int h, int D, int bs, int num_blocks) {
  for (int i = 0; i < ctx; ++i) {
    int32_t blk = table[i / bs];
    if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;
    size_t row = (((size_t)blk * bs + (size_t)(i % bs)) * Hkv + h) * (size_t)D;
    for (int d = 0; d < D; ++d) out[(size_t)i * D + d] = elem(pool, row + d, dtype);
  }
  return OR_OK;
}

/* Whole-sequence gather, all heads: out [ctx, Hkv, D]. */
int oracle_gather(double* out, const void* pool, int dtype, const int32_t* table, int ctx,
                  int Hkv, int D, int bs, int num_blocks) {
  if (!out || !pool || !table || ctx < 0 || Hkv <= 0 || D <= 0 || bs <= 0) return OR_ERR_ARG;
  for (int i = 0; i < ctx; ++i) {
    int32_t blk = table[i / bs];
    if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;
    for (int h = 0; h < Hkv; ++h) {
      size_t src = (((size_t)blk * bs + (size_t)(i % bs)) * Hkv + h) * (size_t)D;
      for (int d = 0; d < D; ++d) out[((size_t)i * Hkv + h) * D + d] = elem(pool, src + d, dtype);
    }
  }
  return OR_OK;
}

/* One (b, hq) output row by the textbook two-pass softmax. */
static int attend_row(double* o, const void* q, const void* kpool, const void* vpool,
                      int dtype, const int32_t* table, int ctx, int Hq, int Hkv, int D,
                      int bs, int num_blocks, double scale, int b, int hq) {
  int G = Hq / Hkv, h = hq / G;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (ctx <= 0) return OR_OK;
  double* K = (double*)malloc(sizeof(double) * (size_t)ctx * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)ctx * D);
  double* s = (double*)malloc(sizeof(double) * (size_t)ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)D);
  int rc = OR_ERR_NOMEM;
  if (K && V && s && qv) {
    rc = gather_head(K, kpool, dtype, table, ctx, Hkv, h, D, bs, num_blocks);
    if (rc == OR_OK) rc = gather_head(V, vpool, dtype, table, ctx, Hkv, h, D, bs, num_blocks);
  }
  if (rc == OR_OK) {
    for (int d = 0; d < D; ++d) qv[d] = elem(q, ((size_t)b * Hq + hq) * D + d, dtype);
    double m = -INFINITY;
    for (int i = 0; i < ctx; ++i) {
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qv[d] * K[(size_t)i * D + d];
      s[i] = scale * dot;
      if (s[i] > m) m = s[i];
    }
    double l = 0.0;
    for (int i = 0; i < ctx; ++i) {
      double w = exp(s[i] - m);
      l += w;
      for (int d = 0; d < D; ++d) o[d] += w * V[(size_t)i * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
  }
  free(K); free(V); free(s); free(qv);
  return rc;
}

static int check_decode_args(const void* q, const void* kp, const void* vp, int dtype,
                             const int32_t* bt, int MB, const int32_t* cl, int B, int Hq,
                             int Hkv, int D, int bs) {
  if (!q || !kp || !vp || !bt || !cl) return OR_ERR_ARG;
  if (dtype < OR_F32 || dtype > OR_BF16 || B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0)
    return OR_ERR_ARG;
  if (Hq % Hkv) return OR_ERR_ARG;
  for (int b = 0; b < B; ++b)
    if (cl[b] < 0 || (long long)cl[b] > (long long)MB * bs) return OR_ERR_ARG;
  return OR_OK;
}

/*
 * out: [n_rows, D] (rows != NULL: rows holds n_rows (b, hq) pairs) or
 *      [B, Hq, D] (rows == NULL).
 * Returns OR_OK, or an error code (first error wins); n_threads <= 0 = all.
 */
int oracle_decode(double* out, const void* q, const void* kpool, const void* vpool, int dtype,
                  const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                  int B, int Hq, int Hkv, int D, int bs, int num_blocks, double scale,
                  const int32_t* rows, int n_rows, int n_threads) {
  int rc = check_decode_args(q, kpool, vpool, dtype, block_tables, max_blocks, context_lens,
                             B, Hq, Hkv, D, bs);
  if (rc != OR_OK || !out) return rc ? rc : OR_ERR_ARG;
  long long n = rows ? n_rows : (long long)B * Hq;
  int err = OR_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long r = 0; r < n; ++r) {
    int b = rows ? rows[2 * r] : (int)(r / Hq);
    int hq = rows ? rows[2 * r + 1] : (int)(r % Hq);
    int e;
    if (b < 0 || b >= B || hq < 0 || hq >= Hq) e = OR_ERR_ARG;
    else
      e = attend_row(out + r * D, q, kpool, vpool, dtype, block_tables + (size_t)b * max_blocks,
                     context_lens[b], Hq, Hkv, D, bs, num_blocks, scale, b, hq);
    if (e != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      { if (err == OR_OK) err = e; }
    }
  }
  return err;
}

/*
 * Split-context form. out [B, Hq, D] (merged); optional part_m / part_l
 * [B, Hq, P] and part_acc [B, Hq, P, D] receive each partition's (m_j, l_j,
 * acc_j) with P = ceil(max ctx / partition_size); empty partitions get
 * m = -inf, l = 0, acc = 0.
 */
int oracle_decode_partitioned(double* out, double* part_m, double* part_l, double* part_acc,
                              const void* q, const void* kpool, const void* vpool, int dtype,
                              const int32_t* block_tables, int max_blocks,
                              const int32_t* context_lens, int B, int Hq, int Hkv, int D,
                              int bs, int num_blocks, double scale, int partition_size,
                              int n_threads) {
  int rc = check_decode_args(q, kpool, vpool, dtype, block_tables, max_blocks, context_lens,
                             B, Hq, Hkv, D, bs);
  if (rc != OR_OK || !out) return rc ? rc : OR_ERR_ARG;
  if (partition_size <= 0) return OR_ERR_ARG;
  int maxc = 0;
  for (int b = 0; b < B; ++b) if (context_lens[b] > maxc) maxc = context_lens[b];
  int P = (maxc + partition_size - 1) / partition_size;
  int G = Hq / Hkv;
  int err = OR_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long r = 0; r < (long long)B * Hq; ++r) {
    int b = (int)(r / Hq), hq = (int)(r % Hq), h = hq / G, ctx = context_lens[b];
    const int32_t* table = block_tables + (size_t)b * max_blocks;
    double* K = (double*)malloc(sizeof(double) * ((size_t)ctx + 1) * D);
    double* V = (double*)malloc(sizeof(double) * ((size_t)ctx + 1) * D);
    double* qv = (double*)malloc(sizeof(double) * (size_t)D);
    double* mj = (double*)malloc(sizeof(double) * ((size_t)P + 1));
    double* lj = (double*)malloc(sizeof(double) * ((size_t)P + 1));
    double* aj = (double*)calloc(((size_t)P + 1) * D, sizeof(double));
    int e = (K && V && qv && mj && lj && aj) ? OR_OK : OR_ERR_NOMEM;
    if (e == OR_OK) e = gather_head(K, kpool, dtype, table, ctx, Hkv, h, D, bs, num_blocks);
    if (e == OR_OK) e = gather_head(V, vpool, dtype, table, ctx, Hkv, h, D, bs, num_blocks);
    if (e == OR_OK) {
      for (int d = 0; d < D; ++d) qv[d] = elem(q, ((size_t)b * Hq + hq) * D + d, dtype);
      for (int j = 0; j < P; ++j) {
        int lo = j * partition_size, hi = lo + partition_size < ctx ? lo + partition_size : ctx;
        mj[j] = -INFINITY;
        lj[j] = 0.0;
        for (int i = lo; i < hi; ++i) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qv[d] * K[(size_t)i * D + d];
          if (scale * dot > mj[j]) mj[j] = scale * dot;
        }
        for (int i = lo; i < hi; ++i) {
          double dot = 0.0;
          for (int d = 0; d < D; ++d) dot += qv[d] * K[(size_t)i * D + d];
          double w = exp(scale * dot - mj[j]);
          lj[j] += w;
          for (int d = 0; d < D; ++d) aj[(size_t)j * D + d] += w * V[(size_t)i * D + d];
        }
      }
      double M = -INFINITY;
      for (int j = 0; j < P; ++j) if (lj[j] > 0.0 && mj[j] > M) M = mj[j];
      double L = 0.0;
      double* o = out + r * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      for (int j = 0; j < P; ++j) {
        if (!(lj[j] > 0.0)) continue;
        double c = exp(mj[j] - M);
        L += lj[j] * c;
        for (int d = 0; d < D; ++d) o[d] += c * aj[(size_t)j * D + d];
      }
      if (L > 0.0)
        for (int d = 0; d < D; ++d) o[d] /= L;
      if (part_m && part_l)
        for (int j = 0; j < P; ++j) {
          part_m[r * P + j] = mj[j];
          part_l[r * P + j] = lj[j];
        }
      if (part_acc)
        for (int j = 0; j < P; ++j)
          for (int d = 0; d < D; ++d) part_acc[(r * P + j) * D + d] = aj[(size_t)j * D + d];
    }
    free(K); free(V); free(qv); free(mj); free(lj); free(aj);
    if (e != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      { if (err == OR_OK) err = e; }
    }
  }
  return err;
}

/* Sequential scatter of T new rows; validates every slot before writing any. */
int oracle_reshape_and_cache(void* kpool, void* vpool, const void* key, const void* value,
                             const int64_t* slot_mapping, int T, int Hkv, int D, int bs,
                             int num_blocks, int dtype) {
  if (!kpool || !vpool || (T > 0 && (!key || !value || !slot_mapping))) return OR_ERR_ARG;
  if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || num_blocks <= 0) return OR_ERR_ARG;
  size_t row = (size_t)Hkv * D * esize_of(dtype);
  long long nslots = (long long)num_blocks * bs;
  for (int t = 0; t < T; ++t)
    if (slot_mapping[t] >= nslots) return OR_ERR_SLOT;
  for (int t = 0; t < T; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    size_t blk = (size_t)(s / bs), off = (size_t)(s % bs);
    size_t dst = (blk * bs + off) * row;
    memcpy((char*)kpool + dst, (const char*)key + (size_t)t * row, row);
    memcpy((char*)vpool + dst, (const char*)value + (size_t)t * row, row);
  }
  return OR_OK;
}

/* Whole-block copies; all sources are snapshotted before the first write. */
int oracle_copy_blocks(void* kpool, void* vpool, const int64_t* block_mapping, int num_pairs,
                       int Hkv, int D, int bs, int num_blocks, int dtype) {
  if (!kpool || !vpool || num_pairs < 0 || (num_pairs > 0 && !block_mapping)) return OR_ERR_ARG;
  size_t blk = (size_t)bs * Hkv * D * esize_of(dtype);
  for (int p = 0; p < num_pairs; ++p) {
    int64_t s = block_mapping[2 * p], d = block_mapping[2 * p + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return OR_ERR_PAIR;
  }
  if (num_pairs == 0) return OR_OK;
  char* snap = (char*)malloc(2 * blk * (size_t)num_pairs);
  if (!snap) return OR_ERR_NOMEM;
  for (int p = 0; p < num_pairs; ++p) {
    size_t s = (size_t)block_mapping[2 * p];
    memcpy(snap + (2 * (size_t)p) * blk, (const char*)kpool + s * blk, blk);
    memcpy(snap + (2 * (size_t)p + 1) * blk, (const char*)vpool + s * blk, blk);
  }
  for (int p = 0; p < num_pairs; ++p) {
    size_t d = (size_t)block_mapping[2 * p + 1];
    memcpy((char*)kpool + d * blk, snap + (2 * (size_t)p) * blk, blk);
    memcpy((char*)vpool + d * blk, snap + (2 * (size_t)p + 1) * blk, blk);
  }
  free(snap);
  return OR_OK;
}

/* Exported widening, so tests can pin the f16 / bf16 decoding to a library. */
int oracle_widen(double* out, const void* src, long long n, int dtype) {
  if (!out || !src || n < 0) return OR_ERR_ARG;
  for (long long i = 0; i < n; ++i) out[i] = elem(src, (size_t)i, dtype);
  return OR_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
