// pa_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_common.cuh"

namespace pa {

// Everything a decode launch needs, resolved by the host layer.
struct DecodeArgs {
  void* out;
  int out_dtype;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int B, Hq, Hkv, D, bs, num_blocks;
  float scale_log2;     // softmax scale * log2(e): scores live in the log2 domain
  int max_context_len;
  int P;                // partitions per sequence (grid extent); 1 = single pass
  int psize;            // tokens per partition (a multiple of bs)
  float* ws_acc;        // [B, P, Hq, D] unnormalised partial outputs (P > 1)
  float* ws_m;          // [B, P, Hq] partial max, log2 domain
  float* ws_l;          // [B, P, Hq] partial sum of exp2(s - m)
  float v_scale;        // value of one V unit (FP8 pools; 1 otherwise); K's is in scale_log2
  uint32_t* err_flag;
  // Shared-prefix (cascade) suffix pass: sequence b attends tokens
  // [start_blocks[b] * bs, ctx_b) only (start_blocks NULL = all tokens),
  // partition j goes to workspace slot slot_base + j, and with force_split
  // every partition is left as a partial for the merge (which then also
  // writes empty and bad rows).
  const int32_t* start_blocks;
  int slot_base;
  int force_split;
  // Tensor-core path (work split evenly over the CTAs): a (sequence, group of
  // 4 KV heads) whose tiles straddle CTAs is written as pieces, at most two
  // per CTA (slot 2 * cta for its first unit, 2 * cta + 1 for its last), and
  // the last piece to finish, chosen by a ticket per (sequence, group), merges
  // them. A ticket word is (epoch << 24 | count): a word from another call (or
  // uninitialised memory) has another epoch and counts as zero.
  float* sk_acc;                  // [2 * grid][4 * G][D] unnormalised piece outputs
  float* sk_m;                    // [2 * grid][4 * G] piece reference max (log2 domain)
  float* sk_l;                    // [2 * grid][4 * G] piece exp-sums
  unsigned long long* tickets;    // [B * (Hkv / 4)]
  unsigned long long epoch;       // this call's number (40 bits)
  unsigned long long wait_ns;     // limit of every pipeline wait of the tensor-core kernel
  int pair_cost;                  // work split: cost of a pair's start and end, in 1/16 of a
                                  // tile's (the CTAs take equal shares of tiles + pair costs)
  int test_withhold_q;            // timeout-path test only: the first unit's query is never
                                  // loaded, so the wait for it can only run out
};

// Shared-prefix decode: the prefix is cut into partitions of a multiple of
// kPrefixTile tokens (one tensor-core tile); a sequence's workspace slots
// [0, slot_base) hold its prefix partials, at most ceil(prefix / kPrefixTile).
constexpr int kPrefixTile = 128;

struct DecodePlan {
  int kernel;           // 1 = CUDA-core path, 2 = tcgen05 GQA path
  int P;
  int psize;
};

// Host planning shared by pa_workspace_size, pa_decode_plan and pa_decode.
DecodePlan plan_decode(int dtype, int B, int Hq, int Hkv, int D, int bs, int max_ctx,
                       int partition_size);
size_t workspace_bytes_for(int B, int Hq, int D, int P);
// Scratch a decode with this plan needs: the tensor-core kernel's pieces and
// tickets, or the CUDA-core split pass's partials (0 for a single pass).
size_t decode_scratch_bytes(const DecodePlan& p, int B, int Hq, int Hkv, int D);

int launch_decode_simt(const DecodeArgs& a, int dtype, cudaStream_t stream);
// Pools whose element types differ from the query's: both FP8 E4M3 (any query
// type), or one FP8 and the other of the query's 16-bit type.
int launch_decode_simt_kv(const DecodeArgs& a, int q_dtype, int k_dtype, int v_dtype,
                          cudaStream_t stream);
// dtype: the query's (16-bit) type; kv8: both pools hold FP8 E4M3 codes.
int launch_decode_tc(const DecodeArgs& a, int dtype, bool kv8, cudaStream_t stream);
bool tc_supported(int dtype, int Hq, int Hkv, int D, int bs);
// Shapes the tensor-core path can take for some 16-bit element type and block size.
bool tc_shape(int Hq, int Hkv, int D);
// Scratch of the tensor-core path (pieces and tickets), and its carve-up.
size_t tc_workspace_bytes(int B, int Hq, int Hkv, int D);
void tc_carve(DecodeArgs& a, char* base);
int sm_count_cached();
int launch_merge(const DecodeArgs& a, cudaStream_t stream);
bool prefix_tc_supported(int dtype, int Hq, int Hkv, int D, int bs);
int prefix_chunks(int max_group_size, int G);

// Paged prefill on the multi-query tensor-core kernel.
struct PrefillLaunch {
  void* out;
  int out_dtype;
  const void* q;                // [T, Hq, D]
  const void* k_cache;
  const void* v_cache;
  int dtype;                    // query type (16-bit)
  int k_dtype, v_dtype;         // pool types: dtype, or PA_FP8_E4M3 (codes times the scale)
  float v_scale;                // FP8 V pool's scale (K's is in scale_log2)
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;  // [B] tokens in the cache after the chunk
  const int32_t* query_start;   // [B + 1]
  int B, T, max_query_len, Hq, Hkv, bs, num_blocks;
  float scale_log2;
  int max_context_len;
  uint32_t* err_flag;
};
int launch_prefill_tc(const PrefillLaunch& p, cudaStream_t stream);
// Paged prefill with the query rows on the MMA's M (prefill_tc.cu).
bool prefill_fa_supported(int dtype, int Hq, int Hkv, int D, int bs);
int launch_prefill_fa(const PrefillLaunch& p, cudaStream_t stream);
// dtype: the query's (16-bit) type; k8 / v8: that pool holds FP8 E4M3 codes.
int launch_prefix_tc(const DecodeArgs& a, int dtype, const int32_t* group_offsets,
                     const int32_t* group_members, int num_groups, int max_group_size, int parts,
                     int part_tokens, cudaStream_t stream, bool k8 = false, bool v8 = false);

int launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                             void* value_cache, int esize, const int64_t* slot_mapping, int T,
                             int Hkv, int D, int block_size, int num_blocks, uint32_t* err_flag,
                             cudaStream_t stream);
int launch_copy_blocks(void* key_cache, void* value_cache, int esize,
                       const int64_t* block_mapping, int num_pairs, int Hkv, int D,
                       int block_size, int num_blocks, uint32_t* err_flag, cudaStream_t stream);
// Scatter with one element type per pool: a pool of the source type gets the
// row copied, an FP8 pool gets it quantised (code = E4M3(x / scale)).
int launch_reshape_and_cache_kv(const void* key, const void* value, int src_dtype,
                                void* key_cache, int k_fp8, float k_scale, void* value_cache,
                                int v_fp8, float v_scale, const int64_t* slot_mapping, int T,
                                int Hkv, int D, int block_size, int num_blocks,
                                uint32_t* err_flag, cudaStream_t stream);
int launch_swap_blocks(void* dst_key, void* dst_value, const void* src_key,
                       const void* src_value, int esize, const int64_t* block_mapping,
                       int num_pairs, int Hkv, int D, int block_size, int src_blocks,
                       int dst_blocks, uint32_t* err_flag, cudaStream_t stream);

}  // namespace pa
