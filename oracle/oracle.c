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
 *  oracle_prefill     Prompt (chunked-prefill) attention: new token i of
 *                     sequence b, at position p = ctx_b - n_b + i, attends the
 *                     cached tokens 0 .. p (causal) through the block table,
 *                     by the same two-pass softmax as oracle_decode.
 *                     "推理引擎内部机制——PagedAttention、连续批处理、分块预填充"
 *                     (chunked prefill: a long prompt's chunks attend the
 *                     paged cache). Causality is the plain reading of a
 *                     prompt's self-attention.
 *  oracle_swap_blocks The same whole-block copy between two different pools
 *                     (host and device memory): preemption by swapping moves
 *                     a sequence's blocks to CPU memory and back. "vLLM 与
 *                     LLM 推理部署实战" section 三 (preemption: the block
 *                     manager swaps blocks out to CPU memory).
 *  FP8 KV cache       The pools may hold 8-bit codes instead of 16/32-bit
 *                     values: halving the bytes per token is the stated
 *                     point ("vLLM 与 LLM 推理部署实战" section 6.2; "vLLM与
 *                     PagedAttention：大模型推理内存优化技术解析" section 6.1
 *                     names fp8 K with bf16 V). The pages fix no
 *                     format; the reading here is OCP FP8 E4M3 (bias 7, no
 *                     infinities, 448 the largest finite value) with one
 *                     float scale per pool: stored code = E4M3(x / scale),
 *                     the quotient taken in binary32 and rounded to nearest
 *                     even, saturating at +-448; value read = code * scale.
 *                     oracle_reshape_and_cache_fp8 quantises that way and
 *                     oracle_decode_kv reads the codes times their scale
 *                     (exact in double). The explainer's mixed configuration
 *                     (K in fp8, V in bf16) takes one element type per pool:
 *                     oracle_decode_mixed, oracle_prefill_mixed and
 *                     oracle_reshape_and_cache_mixed.
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

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_FP8 = 3 };
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

/* E4M3: 1 sign, 4 exponent (bias 7), 3 fraction bits; exponent 15 with
   fraction 7 is NaN, there are no infinities. */
static double e4m3_to_double(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, f = c & 7;
  double v;
  if (e == 15 && f == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)f, -9);                  /* subnormal: f/8 * 2^(1-7) */
  else
    v = ldexp((double)(8 + f), e - 10);        /* (1 + f/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* binary32 -> E4M3, round to nearest even on the E4M3 grid, saturating:
   |y| >= 448 (or rounding to above 448) gives +-448, NaN gives 0x7F. */
static uint8_t e4m3_from_float(float y) {
  if (isnan(y)) return 0x7F;
  uint8_t sign = signbit(y) ? 0x80 : 0;
  double a = fabs((double)y);
  if (a >= 448.0) return sign | 0x7E;
  int ex;
  frexp(a, &ex);                                /* a in [2^(ex-1), 2^ex) */
  int binade = ex - 1 < -6 ? -6 : ex - 1;       /* below 2^-6 the grid is uniform */
  double step = ldexp(1.0, binade - 3);         /* 3 fraction bits */
  double v = rint(a / step) * step;             /* ties to even (default mode) */
  if (v == 0.0) return sign;
  frexp(v, &ex);
  int be = ex - 1;
  if (be < -6) return sign | (uint8_t)(v / ldexp(1.0, -9));           /* subnormal */
  return sign | (uint8_t)((be + 7) << 3) | (uint8_t)((v / ldexp(1.0, be) - 1.0) * 8.0);
}

static int esize_of(int dtype) { return dtype == OR_F32 ? 4 : (dtype == OR_FP8 ? 1 : 2); }

static double elem(const void* base, size_t i, int dtype) {
  if (dtype == OR_F32) return (double)((const float*)base)[i];
  if (dtype == OR_FP8) return e4m3_to_double(((const uint8_t*)base)[i]);
  uint16_t h = ((const uint16_t*)base)[i];
  return dtype == OR_F16 ? f16_to_double(h) : bf16_to_double(h);
}

/* out[i, d] = pool[table[i / bs], i % bs, h, d] * pscale for i < ctx (one KV
   head); pscale is 1 for 16/32-bit pools, the pool's scale for FP8 codes. */
static int gather_head(double* out, const void* pool, int dtype, double pscale,
                       const int32_t* table, int ctx, int Hkv, int h, int D, int bs,
                       int num_blocks) {
  for (int i = 0; i < ctx; ++i) {
    int32_t blk = table[i / bs];
    if (blk < 0 || blk >= num_blocks) return OR_ERR_BLOCK;
    size_t row = (((size_t)blk * bs + (size_t)(i % bs)) * Hkv + h) * (size_t)D;
    for (int d = 0; d < D; ++d) out[(size_t)i * D + d] = elem(pool, row + d, dtype) * pscale;
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

/* One (b, hq) output row by the textbook two-pass softmax (K and V pools may
   hold different element types). */
static int attend_row(double* o, const void* q, int qdt, const void* kpool, int kdt,
                      double kscale, const void* vpool, int vdt, double vscale,
                      const int32_t* table, int ctx, int Hq, int Hkv, int D, int bs,
                      int num_blocks, double scale, int b, int hq) {
  int G = Hq / Hkv, h = hq / G;
  if (kdt != OR_FP8) kscale = 1.0;             /* a scale belongs to FP8 codes only */
  if (vdt != OR_FP8) vscale = 1.0;
  for (int d = 0; d < D; ++d) o[d] = 0.0;
  if (ctx <= 0) return OR_OK;
  double* K = (double*)malloc(sizeof(double) * (size_t)ctx * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)ctx * D);
  double* s = (double*)malloc(sizeof(double) * (size_t)ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)D);
  int rc = OR_ERR_NOMEM;
  if (K && V && s && qv) {
    rc = gather_head(K, kpool, kdt, kscale, table, ctx, Hkv, h, D, bs, num_blocks);
    if (rc == OR_OK)
      rc = gather_head(V, vpool, vdt, vscale, table, ctx, Hkv, h, D, bs, num_blocks);
  }
  if (rc == OR_OK) {
    for (int d = 0; d < D; ++d) qv[d] = elem(q, ((size_t)b * Hq + hq) * D + d, qdt);
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
  if (dtype < OR_F32 || dtype > OR_FP8 || B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0)
    return OR_ERR_ARG;
  if (Hq % Hkv) return OR_ERR_ARG;
  for (int b = 0; b < B; ++b)
    if (cl[b] < 0 || (long long)cl[b] > (long long)MB * bs) return OR_ERR_ARG;
  return OR_OK;
}

/*
 * out: [n_rows, D] (rows != NULL: rows holds n_rows (b, hq) pairs) or
 *      [B, Hq, D] (rows == NULL). The K pool holds k_dtype elements (read times
 * k_scale if they are FP8 codes), the V pool v_dtype elements (times v_scale
 * if FP8; 16/32-bit pools are read as stored): an FP8 K pool with a
 * 16-bit V pool is the mixed configuration of "vLLM与PagedAttention：大模型推理
 * 内存优化技术解析" section 6.1.
 * Returns OR_OK, or an error code (first error wins); n_threads <= 0 = all.
 */
int oracle_decode_mixed(double* out, const void* q, int q_dtype, const void* kpool, int k_dtype,
                        double k_scale, const void* vpool, int v_dtype, double v_scale,
                        const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                        int B, int Hq, int Hkv, int D, int bs, int num_blocks, double scale,
                        const int32_t* rows, int n_rows, int n_threads) {
  if (q_dtype < OR_F32 || q_dtype > OR_BF16) return OR_ERR_ARG;
  if (v_dtype < OR_F32 || v_dtype > OR_FP8) return OR_ERR_ARG;
  int rc = check_decode_args(q, kpool, vpool, k_dtype, block_tables, max_blocks, context_lens,
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
      e = attend_row(out + r * D, q, q_dtype, kpool, k_dtype, k_scale, vpool, v_dtype, v_scale,
                     block_tables + (size_t)b * max_blocks, context_lens[b], Hq, Hkv, D, bs,
                     num_blocks, scale, b, hq);
    if (e != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      { if (err == OR_OK) err = e; }
    }
  }
  return err;
}

/* Both pools of one element type (kv_dtype), the query of q_dtype. */
int oracle_decode_kv(double* out, const void* q, int q_dtype, const void* kpool,
                     const void* vpool, int kv_dtype, double k_scale, double v_scale,
                     const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                     int B, int Hq, int Hkv, int D, int bs, int num_blocks, double scale,
                     const int32_t* rows, int n_rows, int n_threads) {
  return oracle_decode_mixed(out, q, q_dtype, kpool, kv_dtype, k_scale, vpool, kv_dtype, v_scale,
                             block_tables, max_blocks, context_lens, B, Hq, Hkv, D, bs,
                             num_blocks, scale, rows, n_rows, n_threads);
}

/*
 * Causal prefill: out [T, Hq, D]; query [T, Hq, D] (packed new tokens, rows
 * query_start[b] .. query_start[b+1] of sequence b); context_lens after the chunk.
 */
int oracle_prefill_mixed(double* out, const void* q, int q_dtype, const void* kpool,
                         int k_dtype, double k_scale, const void* vpool, int v_dtype,
                         double v_scale, const int32_t* block_tables, int max_blocks,
                         const int32_t* context_lens, const int32_t* query_start, int B, int Hq,
                         int Hkv, int D, int bs, int num_blocks, double scale, int n_threads) {
  if (!out || !query_start) return OR_ERR_ARG;
  if (q_dtype < OR_F32 || q_dtype > OR_BF16 || v_dtype < OR_F32 || v_dtype > OR_FP8)
    return OR_ERR_ARG;
  int rc = check_decode_args(q, kpool, vpool, k_dtype, block_tables, max_blocks, context_lens, B,
                             Hq, Hkv, D, bs);
  if (rc != OR_OK) return rc;
  for (int b = 0; b < B; ++b) {
    int n = query_start[b + 1] - query_start[b];
    if (n < 0 || n > context_lens[b]) return OR_ERR_ARG;
  }
  long long T = query_start[B];
  int err = OR_OK;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (long long r = 0; r < T * Hq; ++r) {
    long long t = r / Hq;
    int hq = (int)(r % Hq), b = 0;
    while (query_start[b + 1] <= t) ++b;                /* the sequence of query row t */
    int n = query_start[b + 1] - query_start[b];
    int pos = context_lens[b] - n + (int)(t - query_start[b]);
    int e = attend_row(out + r * D, q, q_dtype, kpool, k_dtype, k_scale, vpool, v_dtype, v_scale,
                       block_tables + (size_t)b * max_blocks, pos + 1, Hq, Hkv, D, bs,
                       num_blocks, scale, (int)t, hq);
    if (e != OR_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
      { if (err == OR_OK) err = e; }
    }
  }
  return err;
}

/* One element type for the query and both pools (16/32-bit). */
int oracle_prefill(double* out, const void* q, const void* kpool, const void* vpool, int dtype,
                   const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                   const int32_t* query_start, int B, int Hq, int Hkv, int D, int bs,
                   int num_blocks, double scale, int n_threads) {
  if (dtype == OR_FP8) return OR_ERR_ARG;
  return oracle_prefill_mixed(out, q, dtype, kpool, dtype, 1.0, vpool, dtype, 1.0, block_tables,
                              max_blocks, context_lens, query_start, B, Hq, Hkv, D, bs,
                              num_blocks, scale, n_threads);
}

/* Same element type for q, K and V (16/32-bit pools). */
int oracle_decode(double* out, const void* q, const void* kpool, const void* vpool, int dtype,
                  const int32_t* block_tables, int max_blocks, const int32_t* context_lens,
                  int B, int Hq, int Hkv, int D, int bs, int num_blocks, double scale,
                  const int32_t* rows, int n_rows, int n_threads) {
  if (dtype == OR_FP8) return OR_ERR_ARG;
  return oracle_decode_kv(out, q, dtype, kpool, vpool, dtype, 1.0, 1.0, block_tables,
                          max_blocks, context_lens, B, Hq, Hkv, D, bs, num_blocks, scale, rows,
                          n_rows, n_threads);
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
  if (partition_size <= 0 || dtype == OR_FP8) return OR_ERR_ARG;
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
    if (e == OR_OK) e = gather_head(K, kpool, dtype, 1.0, table, ctx, Hkv, h, D, bs, num_blocks);
    if (e == OR_OK) e = gather_head(V, vpool, dtype, 1.0, table, ctx, Hkv, h, D, bs, num_blocks);
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

/* Scatter with quantisation to E4M3 codes: code = E4M3(float(x) / scale), the
   quotient in binary32 (x is exact in binary32 for every source type). */
int oracle_reshape_and_cache_fp8(uint8_t* kpool, uint8_t* vpool, const void* key,
                                 const void* value, int src_dtype, float k_scale, float v_scale,
                                 const int64_t* slot_mapping, int T, int Hkv, int D, int bs,
                                 int num_blocks) {
  if (!kpool || !vpool || (T > 0 && (!key || !value || !slot_mapping))) return OR_ERR_ARG;
  if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || num_blocks <= 0) return OR_ERR_ARG;
  if (src_dtype < OR_F32 || src_dtype > OR_BF16 || !(k_scale > 0.f) || !(v_scale > 0.f))
    return OR_ERR_ARG;
  size_t row = (size_t)Hkv * D;
  long long nslots = (long long)num_blocks * bs;
  for (int t = 0; t < T; ++t)
    if (slot_mapping[t] >= nslots) return OR_ERR_SLOT;
  for (int t = 0; t < T; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    for (size_t i = 0; i < row; ++i) {
      float kx = (float)elem(key, (size_t)t * row + i, src_dtype);
      float vx = (float)elem(value, (size_t)t * row + i, src_dtype);
      kpool[(size_t)s * row + i] = e4m3_from_float(kx / k_scale);
      vpool[(size_t)s * row + i] = e4m3_from_float(vx / v_scale);
    }
  }
  return OR_OK;
}

/* Scatter into pools of per-pool element types: a pool of the source type gets
   the row copied bit for bit, an FP8 pool gets codes E4M3(float(x) / scale)
   (the two cases above, one per pool). */
int oracle_reshape_and_cache_mixed(void* kpool, void* vpool, const void* key, const void* value,
                                   int src_dtype, int k_dtype, int v_dtype, float k_scale,
                                   float v_scale, const int64_t* slot_mapping, int T, int Hkv,
                                   int D, int bs, int num_blocks) {
  if (!kpool || !vpool || (T > 0 && (!key || !value || !slot_mapping))) return OR_ERR_ARG;
  if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || num_blocks <= 0) return OR_ERR_ARG;
  if (src_dtype < OR_F32 || src_dtype > OR_BF16) return OR_ERR_ARG;
  if ((k_dtype != src_dtype && k_dtype != OR_FP8) || (v_dtype != src_dtype && v_dtype != OR_FP8))
    return OR_ERR_ARG;
  if ((k_dtype == OR_FP8 && !(k_scale > 0.f)) || (v_dtype == OR_FP8 && !(v_scale > 0.f)))
    return OR_ERR_ARG;
  size_t row = (size_t)Hkv * D;
  long long nslots = (long long)num_blocks * bs;
  for (int t = 0; t < T; ++t)
    if (slot_mapping[t] >= nslots) return OR_ERR_SLOT;
  for (int t = 0; t < T; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    for (int which = 0; which < 2; ++which) {
      const void* src = which ? value : key;
      void* pool = which ? vpool : kpool;
      int pdt = which ? v_dtype : k_dtype;
      float sc = which ? v_scale : k_scale;
      if (pdt == OR_FP8) {
        for (size_t i = 0; i < row; ++i) {
          float x = (float)elem(src, (size_t)t * row + i, src_dtype);
          ((uint8_t*)pool)[(size_t)s * row + i] = e4m3_from_float(x / sc);
        }
      } else {
        size_t rb = row * esize_of(pdt);
        memcpy((char*)pool + (size_t)s * rb, (const char*)src + (size_t)t * rb, rb);
      }
    }
  }
  return OR_OK;
}

/* E4M3 codes of n binary32 values (the quantiser above, exported for pinning). */
int oracle_fp8_encode(uint8_t* out, const float* x, long long n) {
  if (!out || !x || n < 0) return OR_ERR_ARG;
  for (long long i = 0; i < n; ++i) out[i] = e4m3_from_float(x[i]);
  return OR_OK;
}

/* Block copies between two pools (src_pool -> dst_pool, pairs of block ids). */
int oracle_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                       const int64_t* block_mapping, int num_pairs, size_t block_bytes,
                       int src_blocks, int dst_blocks) {
  if (!dst_k || !dst_v || !src_k || !src_v || num_pairs < 0 || (num_pairs > 0 && !block_mapping))
    return OR_ERR_ARG;
  for (int p = 0; p < num_pairs; ++p) {
    int64_t s = block_mapping[2 * p], d = block_mapping[2 * p + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) return OR_ERR_PAIR;
  }
  for (int p = 0; p < num_pairs; ++p) {
    size_t s = (size_t)block_mapping[2 * p], d = (size_t)block_mapping[2 * p + 1];
    memcpy((char*)dst_k + d * block_bytes, (const char*)src_k + s * block_bytes, block_bytes);
    memcpy((char*)dst_v + d * block_bytes, (const char*)src_v + s * block_bytes, block_bytes);
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
