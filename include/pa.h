/*
 * pa.h -- C ABI of libpa.so: paged KV-cache decode attention for NVIDIA B200
 * (sm_100a), and the two kernels that keep the paged cache current.
 *
 * The problem, as the pages on PagedAttention state it: a pool of fixed-size
 * physical KV blocks, shaped [num_blocks, block_size, ...] ("17. vLLM
 * PagedAttention", Step 3: the physical block pool), and per sequence a block
 * table mapping logical block i to a physical block id, not contiguous
 * ("五十三：vLLM-PagedAttention" section 8; "vLLM 与 LLM 推理部署实战" section
 * 2.1). The attention kernel finds each sequence's history through its block
 * table and attends the current query to it ("17. vLLM PagedAttention",
 * Step 2; "vLLM 与 LLM 推理部署实战" section 2.3).
 *
 * Conventions shared by every entry point
 *  - All array arguments are DEVICE pointers owned by the caller; the library
 *    allocates no device memory. Arrays are dense, row-major, in the layouts
 *    written beside each argument, and 16-byte aligned (element arrays).
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream). The return value covers only what the host can see
 *    before launching: a nonzero pa_status means nothing was launched.
 *  - Errors that depend on device data (a block id or slot out of range, a
 *    context length beyond the table) never fault and never trap: the
 *    offending element is skipped and a bit is OR-ed into *err_flag (if
 *    err_flag is not NULL). err_flag is a device uint32 the caller zeroes and
 *    reads back when it wants to know.
 *  - Element types: PA_F32, PA_F16 (IEEE binary16), PA_BF16. Pools, queries
 *    and new K/V rows share one element type per call, except in the FP8
 *    entry points below, whose pools hold PA_FP8_E4M3 codes.
 *  - Shapes: head size D in {64, 128}; block_size in {16, 32}; Hq a multiple
 *    of Hkv with G = Hq / Hkv in {1, 2, 4, 8, 16}. Query head hq reads KV head
 *    hq / G (contiguous groups; the pages do not say, this is the usual GQA
 *    grouping).
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_NULL = 1,        /* a required pointer is NULL */
  PA_ERR_SHAPE = 2,       /* a size is negative or inconsistent */
  PA_ERR_DTYPE = 3,       /* unknown element type, or out_dtype not F32 / dtype */
  PA_ERR_UNSUPPORTED = 4, /* D, block_size or G outside the supported set */
  PA_ERR_WORKSPACE = 5,   /* workspace missing or smaller than pa_workspace_size() */
  PA_ERR_CUDA = 6,        /* a CUDA call failed (launch error, no device, ...) */
  PA_ERR_ALIGN = 7        /* an element array is not 16-byte aligned */
} pa_status;

/* Bits OR-ed into *err_flag by the kernels (never a trap). */
#define PA_DEV_BAD_BLOCK_ID 1u /* a needed block-table entry is outside [0, num_blocks):
                                  that block's tokens are left out of the softmax */
#define PA_DEV_BAD_CTX 2u      /* context_lens[b] < 0, > max_blocks_per_seq * block_size or
                                  > max_context_len: sequence b's output rows are zeros */
#define PA_DEV_BAD_SLOT 4u     /* slot >= num_blocks * block_size: that token is not written */
#define PA_DEV_BAD_PAIR 8u     /* src or dst outside [0, num_blocks): that pair is skipped */
#define PA_DEV_TIMEOUT 16u     /* a pipeline wait inside a tensor-core kernel gave up
                                  (bounded at 1 s): outputs of that launch are unspecified */

/*
 * pa_workspace_size -- bytes of scratch pa_decode needs for these sizes.
 *
 * Splitting one sequence's softmax sum over several workers needs scratch:
 * each part's running max m, exp-sum l and unnormalised output (fp32), which
 * are then combined: M = max m_j, L = sum l_j e^(m_j - M),
 * o = sum e^(m_j - M) o_j / L. This is not on the pages; it is the algebra of
 * splitting one softmax sum.
 *  - The CUDA-core kernel splits long contexts into partitions (of
 *    partition_size tokens: 0 = let the library choose, else a multiple of
 *    block_size, used as given) and a merge kernel combines them.
 *  - The tensor-core kernel (16-bit or FP8 pools, head size 128, Hq / Hkv in
 *    {4, 8}, Hkv a multiple of 4) divides all the work evenly over the SMs;
 *    a sequence cut between two of them is merged inside the kernel, through
 *    per-SM slots and one word per (sequence, group of 4 KV heads). It does
 *    not use partition_size. Its scratch (about 2.5 MB at G = 4, 5 MB at
 *    G = 8) is needed on those shapes whatever the context length.
 * Returns the larger of the two needs (0 when neither kernel needs any). Same
 * arguments as the pa_decode call it sizes; never fails (nonsense sizes give 0).
 */
size_t pa_workspace_size(int B, int Hq, int Hkv, int D, int max_context_len,
                         int partition_size);

/*
 * pa_decode -- one decode step of attention for B sequences, one new query
 * token each, against their paged KV history.
 *
 *   out[b, hq, :] = sum_i softmax_i(scale * q[b,hq,:] . K_b[i]) V_b[i],  i < context_lens[b]
 *   with K_b[i] = key_cache[block_tables[b, i / block_size], i % block_size, hq / G, :]
 *   and  V_b[i] likewise from value_cache.
 *
 * out           [B, Hq, D] of out_dtype (PA_F32, or the same type as dtype);
 *               written, rounded to nearest even from fp32.
 * query         [B, Hq, D] of dtype.
 * key_cache,
 * value_cache   [num_blocks, block_size, Hkv, D] of dtype; read only.
 * block_tables  [B, max_blocks_per_seq] int32; entries past
 *               ceil(context_lens[b] / block_size) are never read.
 * context_lens  [B] int32: tokens attended per sequence (0 gives a zero row).
 * scale         softmax scale (usually 1/sqrt(D)).
 * max_context_len  host-side upper bound of context_lens (no device read is
 *               needed to size the launch); a larger length is an error bit.
 * partition_size   0 = auto, else split into partitions of this many tokens
 *               (CUDA-core kernel; the tensor-core kernel splits its own way).
 * workspace     device scratch of at least pa_workspace_size(...) bytes, or
 *               NULL when that size is 0. Overwritten; the caller owns it; its
 *               initial contents do not matter.
 * err_flag      nullable device uint32, see PA_DEV_*.
 * stream        cudaStream_t.
 *
 * Arithmetic: products and sums in fp32, online softmax with exp2, fp32
 * accumulation; the GQA tensor-core path multiplies in the input type with
 * fp32 accumulators (tcgen05, TMEM).
 */
int pa_decode(void* out, int out_dtype, const void* query, const void* key_cache,
              const void* value_cache, int dtype, const int32_t* block_tables,
              int max_blocks_per_seq, const int32_t* context_lens, int B, int Hq, int Hkv,
              int D, int block_size, int num_blocks, float scale, int max_context_len,
              int partition_size, void* workspace, size_t workspace_bytes,
              uint32_t* err_flag, void* stream);

/*
 * pa_reshape_and_cache -- write the K and V rows of T new tokens into the
 * pool: key_cache[s / block_size, s % block_size, :, :] = key[t, :, :] with
 * s = slot_mapping[t] (the same for value). A negative slot means "no
 * token" (padding) and is skipped. This is the write the exercise page's
 * allocate_for_decode prepares ("17. vLLM PagedAttention", Step 4: the new
 * token goes into the sequence's current block, a new block when it is full).
 *
 * key, value    [T, Hkv, D] of dtype.
 * key_cache,
 * value_cache   [num_blocks, block_size, Hkv, D]; written in place.
 * slot_mapping  [T] int64. Two tokens naming the same slot is a caller
 *               error (which one lands is unspecified).
 * Bit-exact copy; no arithmetic on the values.
 */
int pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                         int dtype, const int64_t* slot_mapping, int T, int Hkv, int D,
                         int block_size, int num_blocks, uint32_t* err_flag, void* stream);

/*
 * pa_copy_blocks -- copy-on-write: for each pair p, copy the whole physical
 * block block_mapping[p][0] (all block_size rows, all Hkv heads) to block
 * block_mapping[p][1], in both pools. A write into a block that several
 * sequences share first copies that block whole ("vLLM 与 LLM 推理部署实战"
 * section 2.2; "五十三：vLLM-PagedAttention" sections 10 and 17).
 *
 * block_mapping [num_pairs, 2] int64 (src, dst). Destinations must be
 *               distinct and must not appear as a source in the same call
 *               (the block manager guarantees it: a fresh block is never
 *               shared); otherwise the result is unspecified.
 * dtype may also be PA_FP8_E4M3 (pools of codes). Bit-exact copy.
 */
int pa_copy_blocks(void* key_cache, void* value_cache, int dtype, const int64_t* block_mapping,
                   int num_pairs, int Hkv, int D, int block_size, int num_blocks,
                   uint32_t* err_flag, void* stream);

/*
 * pa_decode_static -- pa_decode without a workspace argument, for callers
 * that cannot allocate device memory (a plugin inside an engine that owns all
 * device memory, a program with a fixed device budget, a framework that
 * forbids allocation inside its step). The pages have no counterpart: this
 * entry point exists only for such callers.
 *
 * Same arguments, meaning and results as pa_decode, minus workspace and
 * workspace_bytes. The scratch is a device array of PA_STATIC_SCRATCH_BYTES
 * inside libpa.so: the library calls no allocator (no cudaMalloc, no cudaFree).
 *  - Sizes whose pa_workspace_size(...) exceeds PA_STATIC_SCRATCH_BYTES are
 *    rejected with PA_ERR_WORKSPACE before anything is launched.
 *  - Every GPU that loads the array keeps those bytes until the process exits.
 *  - The array's device address belongs to the CUDA context the library was
 *    loaded into. Each call looks it up in the context current at that call
 *    (so a second context on the device, or a device reset, gets its own
 *    array), except while `stream` is capturing: then the address found by
 *    the last call made outside capture in the same context is reused, and
 *    with none the call fails (PA_ERR_CUDA). Make a first call outside capture.
 *  - All calls in one context share the one array and it keeps the last
 *    call's contents (nothing in it needs to start at zero); calls that
 *    overlap on the GPU race on it, so order them (one stream, or events).
 * Returns a pa_status like pa_decode (PA_ERR_CUDA if the address lookup fails).
 */
#define PA_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)
int pa_decode_static(void* out, int out_dtype, const void* query, const void* key_cache,
                     const void* value_cache, int dtype, const int32_t* block_tables,
                     int max_blocks_per_seq, const int32_t* context_lens, int B, int Hq, int Hkv,
                     int D, int block_size, int num_blocks, float scale, int max_context_len,
                     int partition_size, uint32_t* err_flag, void* stream);

/*
 * FP8 KV cache. The pages give halving the bytes per cached token as the
 * reason to keep K and V in 8 bits ("vLLM 与 LLM 推理部署实战" section 6.2;
 * "vLLM与PagedAttention：大模型推理内存优化技术解析" section 6.1) and fix no
 * format. Here an FP8 pool holds OCP FP8 E4M3 codes, one byte per element
 * (sign, 4-bit exponent with bias 7, 3 fraction bits, no infinities, largest
 * finite value 448), with one float scale per pool: code c stands for
 * value(c) * scale.
 */
#define PA_FP8_E4M3 3 /* pool element type for the FP8 entry points, copy_blocks and swap_blocks */

/*
 * pa_reshape_and_cache_fp8 -- pa_reshape_and_cache into FP8 pools.
 * key, value    [T, Hkv, D] of src_dtype (PA_F32, PA_F16 or PA_BF16);
 * key_cache, value_cache
 *               [num_blocks, block_size, Hkv, D] uint8 E4M3 codes;
 * k_scale, v_scale
 *               positive finite scales: code = E4M3(float(x) / scale), the
 *               quotient rounded to binary32 (IEEE division) and then to the
 *               nearest E4M3 value, ties to even, saturating at +-448 (an
 *               infinite quotient gives +-448, a NaN one 0x7F);
 * slot_mapping, T, Hkv, D, block_size, num_blocks, err_flag, stream
 *               as pa_reshape_and_cache.
 * Returns PA_ERR_SHAPE for a scale that is not positive and finite, otherwise
 * as pa_reshape_and_cache.
 */
int pa_reshape_and_cache_fp8(const void* key, const void* value, int src_dtype, void* key_cache,
                             void* value_cache, float k_scale, float v_scale,
                             const int64_t* slot_mapping, int T, int Hkv, int D, int block_size,
                             int num_blocks, uint32_t* err_flag, void* stream);

/*
 * pa_decode_fp8 -- pa_decode over FP8 pools: each K element attended is
 * value(code) * k_scale and each V element value(code) * v_scale.
 * query         [B, Hq, D] of q_dtype (PA_F32, PA_F16 or PA_BF16);
 * out           [B, Hq, D] of out_dtype (PA_F32 or q_dtype);
 * key_cache, value_cache
 *               [num_blocks, block_size, Hkv, D] uint8 E4M3 codes;
 * k_scale, v_scale
 *               positive finite scales (else PA_ERR_SHAPE).
 * Every other argument, the workspace (sized by pa_workspace_size), the
 * supported shapes and the error behaviour are those of pa_decode. With a
 * 16-bit query on the tensor-core kernel's shapes the codes are widened to the
 * query's type on the chip (exactly) and the products run on the tensor cores;
 * every other call runs on the CUDA-core decode kernel.
 */
int pa_decode_fp8(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                  const void* value_cache, float k_scale, float v_scale,
                  const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, int B, int Hq, int Hkv, int D, int block_size,
                  int num_blocks, float scale, int max_context_len, int partition_size,
                  void* workspace, size_t workspace_bytes, uint32_t* err_flag, void* stream);

/*
 * Mixed pools: one element type per pool. The explainer configures the key
 * cache in fp8 and the value cache in bf16 ("vLLM与PagedAttention：大模型推理
 * 内存优化技术解析" section 6.1, mixed-precision configuration); the two
 * entry points below take each pool's type separately.
 *
 * pa_reshape_and_cache_kv -- pa_reshape_and_cache with per-pool types.
 * key, value    [T, Hkv, D] of src_dtype (PA_F32, PA_F16 or PA_BF16);
 * key_cache     [num_blocks, block_size, Hkv, D] of k_dtype: src_dtype (the
 *               rows are copied bit for bit) or PA_FP8_E4M3 (quantised as in
 *               pa_reshape_and_cache_fp8 with k_scale);
 * value_cache   likewise with v_dtype and v_scale;
 * a scale is checked (positive, finite) and used only for an FP8 pool.
 * Other arguments and errors as pa_reshape_and_cache.
 */
int pa_reshape_and_cache_kv(const void* key, const void* value, int src_dtype, void* key_cache,
                            int k_dtype, float k_scale, void* value_cache, int v_dtype,
                            float v_scale, const int64_t* slot_mapping, int T, int Hkv, int D,
                            int block_size, int num_blocks, uint32_t* err_flag, void* stream);

/*
 * pa_decode_kv -- pa_decode with per-pool types: each K element attended is
 * the K pool's value (times k_scale if it holds FP8 codes), each V element
 * likewise with v_scale.
 * query         [B, Hq, D] of q_dtype (PA_F32, PA_F16 or PA_BF16);
 * key_cache     of k_dtype, value_cache of v_dtype: each q_dtype or
 *               PA_FP8_E4M3; one FP8 pool beside one of the query's type needs
 *               a 16-bit query (otherwise PA_ERR_DTYPE);
 * k_scale, v_scale  positive finite scales of the FP8 pools (ignored for others).
 * Every other argument, the workspace (pa_workspace_size) and the errors are
 * pa_decode's. Calls with both pools of the query's type are pa_decode; calls
 * with an FP8 pool run on the CUDA-core decode kernel.
 */
int pa_decode_kv(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                 int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                 const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                 int B, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
                 int max_context_len, int partition_size, void* workspace,
                 size_t workspace_bytes, uint32_t* err_flag, void* stream);

/*
 * pa_swap_blocks -- preemption by swapping: copy whole blocks (K and V)
 * between two pools, typically the device pool and a pool in page-locked host
 * memory ("vLLM 与 LLM 推理部署实战" section 三: under memory pressure the
 * block manager moves blocks out to CPU memory, and back).
 * dst_key, dst_value  [dst_blocks, block_size, Hkv, D] destination pools;
 * src_key, src_value  [src_blocks, block_size, Hkv, D] source pools;
 *               each pool is device memory or page-locked host memory that
 *               the device can address (cudaHostAlloc, torch pin_memory);
 *               the kernel reads and writes both directly (one launch, no
 *               copy-engine calls). Source and destination pools must not
 *               overlap, and the dst ids must be distinct.
 * dtype         element type of both pools (PA_F32, PA_F16, PA_BF16 or
 *               PA_FP8_E4M3; only its size matters);
 * block_mapping [num_pairs, 2] int64 (src id, dst id), device or page-locked
 *               host memory; a pair with an id out of range is skipped and
 *               sets PA_DEV_BAD_PAIR.
 * Returns a pa_status like pa_copy_blocks.
 */
int pa_swap_blocks(void* dst_key, void* dst_value, const void* src_key, const void* src_value,
                   int dtype, const int64_t* block_mapping, int num_pairs, int Hkv, int D,
                   int block_size, int src_blocks, int dst_blocks, uint32_t* err_flag,
                   void* stream);

/*
 * pa_decode_shared_prefix -- pa_decode for a batch whose sequences come in
 * groups that share the leading blocks of their block tables: the sequences
 * forked from one prompt for parallel sampling share its blocks
 * ("五十三：vLLM-PagedAttention" section 17; the copy-on-write sharing of
 * "vLLM 与 LLM 推理部署实战" section 2.2). The shared blocks are read once per
 * group, for the queries of all its members together (tensor cores), each
 * sequence's own blocks once, and the two parts are merged (split-context
 * merge). The result is pa_decode's on the same arguments.
 *
 * Every argument of pa_decode, with the same meaning and layout, plus:
 * shared_blocks   [B] int32: the first shared_blocks[b] entries of sequence
 *                 b's table are its group's shared prefix (the same entries
 *                 in every member's table; 0 = nothing shared);
 * num_groups, group_offsets [num_groups + 1] int32, group_members [B] int32:
 *                 group g is group_members[group_offsets[g] ..
 *                 group_offsets[g + 1]); every sequence is in exactly one
 *                 group and all members of a group have the same
 *                 shared_blocks value (a lone sequence is a group of one);
 * max_group_size  the largest group (host-side bound, >= 1);
 * max_shared_blocks  the largest shared_blocks value (host-side bound);
 * workspace       of pa_shared_prefix_workspace_size(...) bytes.
 * Groups that break the contract give unspecified (finite) results. A
 * sequence whose shared blocks hold more tokens than its context length is a
 * bad context (PA_DEV_BAD_CTX, zero row). Element types other than f16 / bf16,
 * D = 64, or G > 64 (and max_shared_blocks = 0) run as plain pa_decode.
 */
size_t pa_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D, int max_context_len,
                                       int partition_size, int block_size,
                                       int max_shared_blocks);
int pa_decode_shared_prefix(void* out, int out_dtype, const void* query, const void* key_cache,
                            const void* value_cache, int dtype, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* context_lens,
                            const int32_t* shared_blocks, int num_groups,
                            const int32_t* group_offsets, const int32_t* group_members,
                            int max_group_size, int max_shared_blocks, int B, int Hq, int Hkv,
                            int D, int block_size, int num_blocks, float scale,
                            int max_context_len, int partition_size, void* workspace,
                            size_t workspace_bytes, uint32_t* err_flag, void* stream);

/*
 * pa_decode_shared_prefix_kv -- pa_decode_shared_prefix over pools of other
 * element types than the query's (FP8 E4M3 codes times k_scale / v_scale in
 * either pool or both; see pa_decode_kv): parallel sampling over an FP8 cache,
 * or over the explainer's mixed one, reads each group's shared blocks once.
 * Arguments as pa_decode_shared_prefix, with q_dtype, k_dtype / k_scale and
 * v_dtype / v_scale as in pa_decode_kv; the workspace is sized by
 * pa_shared_prefix_workspace_size. Shapes the prefix kernel does not take run
 * as pa_decode_kv.
 */
int pa_decode_shared_prefix_kv(void* out, int out_dtype, const void* query, int q_dtype,
                               const void* key_cache, int k_dtype, float k_scale,
                               const void* value_cache, int v_dtype, float v_scale,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, const int32_t* shared_blocks,
                               int num_groups, const int32_t* group_offsets,
                               const int32_t* group_members, int max_group_size,
                               int max_shared_blocks, int B, int Hq, int Hkv, int D,
                               int block_size, int num_blocks, float scale, int max_context_len,
                               int partition_size, void* workspace, size_t workspace_bytes,
                               uint32_t* err_flag, void* stream);

/*
 * pa_prefill -- paged prefill (prompt or chunked-prefill) attention: each new
 * query token attends, causally, to its sequence's cached tokens up to and
 * including itself. Long prompts are cut into chunks that run between decode
 * steps ("推理引擎内部机制——PagedAttention、连续批处理、分块预填充", chunked
 * prefill); a chunk's K/V rows are written into the pool first
 * (pa_reshape_and_cache), then its queries attend through the block table.
 *
 * query        [T, Hq, D] of dtype: the new tokens of all sequences, packed;
 *              sequence b's are rows [query_start[b], query_start[b + 1]);
 * query_start  [B + 1] int32, non-decreasing, query_start[B] = T;
 * context_lens [B] int32: tokens of sequence b in the pool after the chunk,
 *              its new tokens included; new token i of b (0-based) sits at
 *              position context_lens[b] - n_b + i and attends positions
 *              0 .. that position (n_b = query_start[b + 1] - query_start[b]);
 * max_query_len the largest n_b (host-side bound);
 * out          [T, Hq, D] of out_dtype (PA_F32 or dtype);
 * key_cache, value_cache, block_tables, max_blocks_per_seq, block_size,
 * num_blocks, scale, max_context_len, err_flag, stream: as pa_decode.
 * Supported: 16-bit K/V (PA_F16, PA_BF16), D = 128, the pa_decode block and
 * group sizes; otherwise PA_ERR_UNSUPPORTED. A sequence with n_b >
 * context_lens[b] (or a context the table cannot hold) sets PA_DEV_BAD_CTX and
 * its rows are not written. No workspace.
 */
int pa_prefill(void* out, int out_dtype, const void* query, const void* key_cache,
               const void* value_cache, int dtype, const int32_t* block_tables,
               int max_blocks_per_seq, const int32_t* context_lens, const int32_t* query_start,
               int B, int T, int max_query_len, int Hq, int Hkv, int D, int block_size,
               int num_blocks, float scale, int max_context_len, uint32_t* err_flag,
               void* stream);

/*
 * pa_prefill_kv -- pa_prefill over pools of other element types than the
 * query's: FP8 E4M3 codes (times k_scale / v_scale) in either pool or both, the
 * other pool of the query's 16-bit type. The FP8 KV cache and the mixed
 * configuration of the explainer ("vLLM与PagedAttention：大模型推理内存优化技术
 * 解析" section 6.1) hold the same tokens a prompt's chunks attend.
 * query        [T, Hq, D] of q_dtype (PA_F16 or PA_BF16);
 * key_cache    of k_dtype, value_cache of v_dtype: each q_dtype or PA_FP8_E4M3;
 * k_scale, v_scale  positive finite scales of the FP8 pools (ignored for others).
 * Every other argument and the errors are pa_prefill's. The codes are widened
 * to the query's type on the chip, exactly.
 */
int pa_prefill_kv(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                  int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                  const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, const int32_t* query_start, int B, int T,
                  int max_query_len, int Hq, int Hkv, int D, int block_size, int num_blocks,
                  float scale, int max_context_len, uint32_t* err_flag, void* stream);

/* Static text for a pa_status value. */
const char* pa_status_string(int status);

/*
 * pa_decode_plan -- what pa_decode will launch for these arguments, for
 * tools and tests (dtype = PA_FP8_E4M3 plans pa_decode_fp8 with a 16-bit
 * query; an fp32 query always takes the CUDA-core kernel): *kernel = 1
 * (CUDA-core path) or 2 (tcgen05 GQA path), *num_partitions = partitions per
 * sequence of the CUDA-core split pass (1 = no split; always 1 for the
 * tensor-core kernel, which splits the work over the SMs itself),
 * *partition_tokens = their length. Any pointer may be NULL. Returns a
 * pa_status (PA_ERR_UNSUPPORTED etc. for the same reasons pa_decode would).
 */
int pa_decode_plan(int dtype, int B, int Hq, int Hkv, int D, int block_size,
                   int max_context_len, int partition_size, int* kernel, int* num_partitions,
                   int* partition_tokens);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
