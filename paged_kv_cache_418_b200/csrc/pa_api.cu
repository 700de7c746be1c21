// pa_api.cu -- the extern "C" boundary of libpa.so: argument checks, launch
// planning (split or not, which kernel), workspace carve-up, launches.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "pa_internal.h"

namespace pa {

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("PA_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

namespace {

constexpr int kDefaultPartition = 512;

bool supported_shape(int Hq, int Hkv, int D, int bs) {
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return (D == 64 || D == 128) && (bs == 16 || bs == 32) &&
         (G == 1 || G == 2 || G == 4 || G == 8 || G == 16);
}

int esize_of(int dtype) { return dtype == PA_F32 ? 4 : (dtype == PA_FP8_E4M3 ? 1 : 2); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Upper bound of the prefix partitions of a shared-prefix decode (one per tile).
int max_prefix_slots(int max_shared_blocks, int block_size) {
  return (max_shared_blocks * block_size + kPrefixTile - 1) / kPrefixTile;
}

// Kernel override for A/B measurements: PA_DECODE_KERNEL=simt|tc (unset = auto).
int kernel_override() {
  const char* s = std::getenv("PA_DECODE_KERNEL");
  if (!s) return 0;
  if (!std::strcmp(s, "simt")) return 1;
  if (!std::strcmp(s, "tc")) return 2;
  return 0;
}

// Limit of every pipeline wait of the tensor-core kernels, in ns (1 s; the
// environment variable PA_TC_WAIT_NS lowers it, for tests of the timeout path).
unsigned long long tc_wait_ns() {
  const char* s = std::getenv("PA_TC_WAIT_NS");
  if (!s || !*s) return 1000000000ull;
  char* end = nullptr;
  const unsigned long long v = std::strtoull(s, &end, 10);
  return (end && *end == 0 && v <= 1000000000ull) ? v : 1000000000ull;
}

// The timeout-path test's hook (PA_TC_TEST_WITHHOLD_Q=1): the tensor-core
// kernel leaves the first unit's query unloaded, so the wait for it runs out.
int tc_test_withhold_q() {
  const char* s = std::getenv("PA_TC_TEST_WITHHOLD_Q");
  return s && s[0] == '1' ? 1 : 0;
}

// Cost of a pair's start and end in the tensor-core kernel's work split, in
// 1/16 of a tile. Per-CTA timers on the Llama-3-70B-shaped batch put a unit's
// query load, first-tile reduction and epilogue at 1.2-1.5 tiles' time; a
// sweep of 0-60 on the GQA, FP8 GQA, long-context and shared-prefix batches
// was fastest at 28 or within 1.5% of it. PA_TC_PAIR_COST overrides it (0 =
// equal tile counts), for measurements.
constexpr int kPairCostDefault = 28;
int tc_pair_cost() {
  const char* s = std::getenv("PA_TC_PAIR_COST");
  if (!s || !*s) return kPairCostDefault;
  char* end = nullptr;
  const long v = std::strtol(s, &end, 10);
  return (end && *end == 0 && v >= 0 && v <= 4096) ? (int)v : kPairCostDefault;
}

// A number per call of the tensor-core path (40 bits; its tickets carry it).
unsigned long long next_epoch() {
  static std::atomic<unsigned long long> n{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 2654435761ull};
  return (n.fetch_add(1) + 1) & ((1ull << 40) - 1);
}

}  // namespace

// SM count of the current device (148 on B200; also the fallback with no device).
int sm_count_cached() {
  static int n = 0;
  if (n <= 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return kSMs;                       // not cached: a device may appear later
    }
    n = v;
  }
  return n;
}

DecodePlan plan_decode(int dtype, int B, int Hq, int Hkv, int D, int bs, int max_ctx,
                       int partition_size) {
  DecodePlan p{1, 1, 0};
  int psize = partition_size;
  if (psize <= 0) {
    // Auto: one pass when every context fits one default partition; else
    // fixed partitions, so no CTA streams more than 512 tokens and the tail
    // of a ragged batch stays short.
    psize = kDefaultPartition;
  }
  const int mc = max_ctx > 0 ? max_ctx : 1;
  p.P = (mc + psize - 1) / psize;
  if (p.P <= 1) {
    p.P = 1;
    p.psize = ((mc + bs - 1) / bs) * bs;
  } else {
    p.psize = psize;
  }
  const int ov = kernel_override();
  const bool tc = tc_supported(dtype, Hq, Hkv, D, bs);
  p.kernel = ov == 1 ? 1 : (ov == 2 ? (tc ? 2 : 1) : (tc ? 2 : 1));
  if (p.kernel == 2) {
    // the tensor-core kernel splits the work evenly over the SMs itself (pieces
    // merged in the kernel): no fixed partitions, no merge launch
    p.P = 1;
    p.psize = ((mc + bs - 1) / bs) * bs;
  }
  (void)B;
  return p;
}

size_t workspace_bytes_for(int B, int Hq, int D, int P) {
  if (P <= 1 || B <= 0) return 0;
  const size_t rows = (size_t)B * Hq * P;
  // acc [rows, D] then m [rows] then l [rows], each 256-byte aligned
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up(rows * D * 4) + up(rows * 4) + up(rows * 4);
}

size_t decode_scratch_bytes(const DecodePlan& p, int B, int Hq, int Hkv, int D) {
  return p.kernel == 2 ? tc_workspace_bytes(B, Hq, Hkv, D) : workspace_bytes_for(B, Hq, D, p.P);
}

}  // namespace pa

using namespace pa;

extern "C" {

size_t pa_workspace_size(int B, int Hq, int Hkv, int D, int max_context_len, int partition_size) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_context_len <= 0 || partition_size < 0)
    return 0;
  // enough for either kernel: the CUDA-core split pass, or the tensor-core
  // kernel's pieces and tickets (shapes it can take in a 16-bit type)
  DecodePlan p = plan_decode(PA_F32, B, Hq, Hkv, D, 16, max_context_len, partition_size);
  return std::max(workspace_bytes_for(B, Hq, D, p.P), tc_workspace_bytes(B, Hq, Hkv, D));
}

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_NULL: return "a required pointer is NULL";
    case PA_ERR_SHAPE: return "a size is negative or inconsistent";
    case PA_ERR_DTYPE: return "unsupported element type or output type";
    case PA_ERR_UNSUPPORTED: return "head size, block size or group size not supported";
    case PA_ERR_WORKSPACE: return "workspace missing or too small";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_ALIGN: return "element array not 16-byte aligned";
  }
  return "unknown status";
}

int pa_decode_plan(int dtype, int B, int Hq, int Hkv, int D, int block_size, int max_context_len,
                   int partition_size, int* kernel, int* num_partitions, int* partition_tokens) {
  if (dtype < PA_F32 || dtype > PA_FP8_E4M3) return PA_ERR_DTYPE;
  if (B < 0 || max_context_len < 0 || partition_size < 0) return PA_ERR_SHAPE;
  if (!supported_shape(Hq, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (partition_size > 0 && partition_size % block_size) return PA_ERR_SHAPE;
  DecodePlan p = plan_decode(dtype, B, Hq, Hkv, D, block_size, max_context_len, partition_size);
  if (kernel) *kernel = p.kernel;
  if (num_partitions) *num_partitions = p.P;
  if (partition_tokens) *partition_tokens = p.psize;
  return PA_OK;
}

}  // extern "C"

namespace {

bool scale_ok(float x) { return std::isfinite(x) && x > 0.f; }

// Pool element types a decode takes for a query of q_dtype: both the query's
// type; both FP8; or, for a 16-bit query, one FP8 pool and one of its type.
bool pool_types_ok(int q_dtype, int k_dtype, int v_dtype) {
  const bool kf = k_dtype == PA_FP8_E4M3, vf = v_dtype == PA_FP8_E4M3;
  if (!kf && k_dtype != q_dtype) return false;
  if (!vf && v_dtype != q_dtype) return false;
  if (kf != vf && q_dtype == PA_F32) return false;
  return true;
}

// Shared body of the decode entry points. q_dtype: query element type;
// k_dtype / v_dtype: pool element types (q_dtype, or PA_FP8_E4M3 read times
// k_scale / v_scale; a scale is used only by an FP8 pool).
int decode_impl(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                int B, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
                int max_context_len, int partition_size, void* workspace,
                size_t workspace_bytes, uint32_t* err_flag, void* stream) {
  if (q_dtype < PA_F32 || q_dtype > PA_BF16) return PA_ERR_DTYPE;
  if (!pool_types_ok(q_dtype, k_dtype, v_dtype)) return PA_ERR_DTYPE;
  const bool k_fp8 = k_dtype == PA_FP8_E4M3, v_fp8 = v_dtype == PA_FP8_E4M3;
  if (!k_fp8) k_scale = 1.f;
  if (!v_fp8) v_scale = 1.f;
  if (out_dtype != PA_F32 && out_dtype != q_dtype) return PA_ERR_DTYPE;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0)
    return PA_ERR_SHAPE;
  if (!supported_shape(Hq, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (partition_size > 0 && partition_size % block_size) return PA_ERR_SHAPE;
  if (!std::isfinite(scale) || !scale_ok(k_scale) || !scale_ok(v_scale)) return PA_ERR_SHAPE;
  if (B > 65535 || Hkv > 65535) return PA_ERR_UNSUPPORTED;
  if (B == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens)
    return PA_ERR_NULL;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;

  // pools of another type than the query's run on the CUDA-core kernel, except
  // FP8 K and V with a 16-bit query (the tensor-core kernel widens the codes)
  DecodePlan p = plan_decode(k_fp8 || v_fp8 ? PA_FP8_E4M3 : q_dtype, B, Hq, Hkv, D, block_size,
                             max_context_len, partition_size);
  if (p.kernel == 2 && (k_fp8 != v_fp8 || (k_fp8 && q_dtype == PA_F32)))
    p = plan_decode(PA_F32, B, Hq, Hkv, D, block_size, max_context_len, partition_size);
  DecodeArgs a{};
  a.out = out; a.out_dtype = out_dtype; a.q = query;
  a.k_cache = key_cache; a.v_cache = value_cache;
  a.block_tables = block_tables; a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.bs = block_size; a.num_blocks = num_blocks;
  a.scale_log2 = scale * kLog2e * k_scale;      // k_scale = 1 unless K holds FP8 codes
  a.v_scale = v_scale;
  a.max_context_len = max_context_len;
  a.P = p.P; a.psize = p.psize;
  a.err_flag = err_flag;
  const bool tc_path = p.kernel == 2;
  if (tc_path) {
    const size_t need = decode_scratch_bytes(p, B, Hq, Hkv, D);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return PA_ERR_WORKSPACE;
    tc_carve(a, static_cast<char*>(workspace));
    a.epoch = next_epoch();
    a.wait_ns = tc_wait_ns();
    a.pair_cost = tc_pair_cost();
    a.test_withhold_q = tc_test_withhold_q();
  } else if (p.P > 1) {
    const size_t need = decode_scratch_bytes(p, B, Hq, Hkv, D);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return PA_ERR_WORKSPACE;
    const size_t rows = (size_t)B * Hq * p.P;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    char* w = static_cast<char*>(workspace);
    a.ws_acc = reinterpret_cast<float*>(w);
    a.ws_m = reinterpret_cast<float*>(w + up(rows * D * 4));
    a.ws_l = reinterpret_cast<float*>(w + up(rows * D * 4) + up(rows * 4));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc;
  if (p.kernel == 2) rc = launch_decode_tc(a, q_dtype, k_fp8, s);
  else if (k_fp8 || v_fp8) rc = launch_decode_simt_kv(a, q_dtype, k_dtype, v_dtype, s);
  else rc = launch_decode_simt(a, q_dtype, s);
  if (rc == PA_OK && p.P > 1) rc = launch_merge(a, s);
  return rc;
}

}  // namespace

extern "C" {

int pa_decode(void* out, int out_dtype, const void* query, const void* key_cache,
              const void* value_cache, int dtype, const int32_t* block_tables,
              int max_blocks_per_seq, const int32_t* context_lens, int B, int Hq, int Hkv, int D,
              int block_size, int num_blocks, float scale, int max_context_len,
              int partition_size, void* workspace, size_t workspace_bytes, uint32_t* err_flag,
              void* stream) {
  if (dtype < PA_F32 || dtype > PA_BF16) return PA_ERR_DTYPE;
  return decode_impl(out, out_dtype, query, dtype, key_cache, dtype, 1.f, value_cache, dtype, 1.f,
                     block_tables, max_blocks_per_seq, context_lens, B, Hq, Hkv, D, block_size,
                     num_blocks, scale, max_context_len, partition_size, workspace,
                     workspace_bytes, err_flag, stream);
}

int pa_decode_fp8(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                  const void* value_cache, float k_scale, float v_scale,
                  const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, int B, int Hq, int Hkv, int D, int block_size,
                  int num_blocks, float scale, int max_context_len, int partition_size,
                  void* workspace, size_t workspace_bytes, uint32_t* err_flag, void* stream) {
  return decode_impl(out, out_dtype, query, q_dtype, key_cache, PA_FP8_E4M3, k_scale, value_cache,
                     PA_FP8_E4M3, v_scale, block_tables, max_blocks_per_seq, context_lens, B, Hq,
                     Hkv, D, block_size, num_blocks, scale, max_context_len, partition_size,
                     workspace, workspace_bytes, err_flag, stream);
}

int pa_decode_kv(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                 int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                 const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                 int B, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
                 int max_context_len, int partition_size, void* workspace,
                 size_t workspace_bytes, uint32_t* err_flag, void* stream) {
  if (k_dtype < PA_F32 || k_dtype > PA_FP8_E4M3 || v_dtype < PA_F32 || v_dtype > PA_FP8_E4M3)
    return PA_ERR_DTYPE;
  return decode_impl(out, out_dtype, query, q_dtype, key_cache, k_dtype, k_scale, value_cache,
                     v_dtype, v_scale, block_tables, max_blocks_per_seq, context_lens, B, Hq, Hkv,
                     D, block_size, num_blocks, scale, max_context_len, partition_size, workspace,
                     workspace_bytes, err_flag, stream);
}

int pa_reshape_and_cache_fp8(const void* key, const void* value, int src_dtype, void* key_cache,
                             void* value_cache, float k_scale, float v_scale,
                             const int64_t* slot_mapping, int T, int Hkv, int D, int block_size,
                             int num_blocks, uint32_t* err_flag, void* stream) {
  if (src_dtype < PA_F32 || src_dtype > PA_BF16) return PA_ERR_DTYPE;
  if (T < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0) return PA_ERR_SHAPE;
  if (!scale_ok(k_scale) || !scale_ok(v_scale)) return PA_ERR_SHAPE;
  if (!supported_shape(Hkv, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (T == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;
  return launch_reshape_and_cache_kv(key, value, src_dtype, key_cache, 1, k_scale, value_cache, 1,
                                      v_scale, slot_mapping, T, Hkv, D, block_size, num_blocks,
                                      err_flag, static_cast<cudaStream_t>(stream));
}

int pa_reshape_and_cache_kv(const void* key, const void* value, int src_dtype, void* key_cache,
                            int k_dtype, float k_scale, void* value_cache, int v_dtype,
                            float v_scale, const int64_t* slot_mapping, int T, int Hkv, int D,
                            int block_size, int num_blocks, uint32_t* err_flag, void* stream) {
  if (src_dtype < PA_F32 || src_dtype > PA_BF16) return PA_ERR_DTYPE;
  const bool kf = k_dtype == PA_FP8_E4M3, vf = v_dtype == PA_FP8_E4M3;
  if ((!kf && k_dtype != src_dtype) || (!vf && v_dtype != src_dtype)) return PA_ERR_DTYPE;
  if (T < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0) return PA_ERR_SHAPE;
  if ((kf && !scale_ok(k_scale)) || (vf && !scale_ok(v_scale))) return PA_ERR_SHAPE;
  if (!supported_shape(Hkv, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (T == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;
  return launch_reshape_and_cache_kv(key, value, src_dtype, key_cache, kf, k_scale, value_cache,
                                     vf, v_scale, slot_mapping, T, Hkv, D, block_size, num_blocks,
                                     err_flag, static_cast<cudaStream_t>(stream));
}

size_t pa_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D, int max_context_len,
                                        int partition_size, int block_size,
                                        int max_shared_blocks) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_context_len <= 0 || partition_size < 0 ||
      block_size <= 0 || max_shared_blocks < 0)
    return 0;
  if (max_shared_blocks == 0) return pa_workspace_size(B, Hq, Hkv, D, max_context_len, partition_size);
  DecodePlan p = plan_decode(PA_F32, B, Hq, Hkv, D, block_size, max_context_len, partition_size);
  // partial slots of the prefix and suffix passes, then the tensor-core suffix
  // pass's pieces and tickets
  return workspace_bytes_for(B, Hq, D, max_prefix_slots(max_shared_blocks, block_size) + p.P) +
         tc_workspace_bytes(B, Hq, Hkv, D);
}

}  // extern "C"

namespace {

// Shared body of pa_decode_shared_prefix and pa_decode_shared_prefix_kv.
int shared_prefix_impl(void* out, int out_dtype, const void* query, int q_dtype,
                       const void* key_cache, int k_dtype, float k_scale, const void* value_cache,
                       int v_dtype, float v_scale, const int32_t* block_tables,
                       int max_blocks_per_seq, const int32_t* context_lens,
                       const int32_t* shared_blocks, int num_groups, const int32_t* group_offsets,
                       const int32_t* group_members, int max_group_size, int max_shared_blocks,
                       int B, int Hq, int Hkv, int D, int block_size, int num_blocks, float scale,
                       int max_context_len, int partition_size, void* workspace,
                       size_t workspace_bytes, uint32_t* err_flag, void* stream) {
  if (q_dtype < PA_F32 || q_dtype > PA_BF16) return PA_ERR_DTYPE;
  if (!pool_types_ok(q_dtype, k_dtype, v_dtype)) return PA_ERR_DTYPE;
  const bool k8 = k_dtype == PA_FP8_E4M3, v8 = v_dtype == PA_FP8_E4M3;
  if (num_groups < 0 || max_group_size < 0 || max_shared_blocks < 0) return PA_ERR_SHAPE;
  if (max_shared_blocks > max_blocks_per_seq) return PA_ERR_SHAPE;
  const bool share = max_shared_blocks > 0 && num_groups > 0 && B > 0 &&
                     prefix_tc_supported(q_dtype, Hq, Hkv, D, block_size);
  if (!share)   // nothing shared, or a shape the prefix kernel does not take: plain decode
    return decode_impl(out, out_dtype, query, q_dtype, key_cache, k_dtype, k_scale, value_cache,
                       v_dtype, v_scale, block_tables, max_blocks_per_seq, context_lens, B, Hq,
                       Hkv, D, block_size, num_blocks, scale, max_context_len, partition_size,
                       workspace, workspace_bytes, err_flag, stream);
  if (out_dtype != PA_F32 && out_dtype != q_dtype) return PA_ERR_DTYPE;
  if (Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0 ||
      max_blocks_per_seq <= 0 || max_context_len < 0 || partition_size < 0 || max_group_size < 1)
    return PA_ERR_SHAPE;
  if (!supported_shape(Hq, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (partition_size > 0 && partition_size % block_size) return PA_ERR_SHAPE;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  if ((k8 && !scale_ok(k_scale)) || (v8 && !scale_ok(v_scale))) return PA_ERR_SHAPE;
  if (B > 65535 || Hkv > 65535) return PA_ERR_UNSUPPORTED;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens ||
      !shared_blocks || !group_offsets || !group_members)
    return PA_ERR_NULL;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;

  // the suffix pass runs on the kernel pa_decode_kv would take
  DecodePlan p = plan_decode(k8 || v8 ? PA_FP8_E4M3 : q_dtype, B, Hq, Hkv, D, block_size,
                             max_context_len, partition_size);
  if (p.kernel == 2 && k8 != v8)
    p = plan_decode(PA_F32, B, Hq, Hkv, D, block_size, max_context_len, partition_size);
  // Prefix partitions: as many as keep every (group, member chunk, KV head)
  // unit of all of them in one wave over the SMs, at least one tile each.
  const int tiles = max_prefix_slots(max_shared_blocks, block_size);
  const long long per_part =
      (long long)num_groups * prefix_chunks(max_group_size, Hq / Hkv) * Hkv;
  int parts = (int)std::max(1LL, std::min<long long>(tiles, sm_count_cached() / std::max(1LL, per_part)));
  const int part_tokens = (tiles + parts - 1) / parts * kPrefixTile;
  parts = (max_shared_blocks * block_size + part_tokens - 1) / part_tokens;
  DecodeArgs a{};
  a.out = out; a.out_dtype = out_dtype; a.q = query;
  a.k_cache = key_cache; a.v_cache = value_cache;
  a.block_tables = block_tables; a.max_blocks = max_blocks_per_seq;
  a.context_lens = context_lens;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.bs = block_size; a.num_blocks = num_blocks;
  a.scale_log2 = scale * kLog2e * (k8 ? k_scale : 1.f);
  a.v_scale = v8 ? v_scale : 1.f;
  a.max_context_len = max_context_len;
  a.P = tiles + p.P; a.psize = p.psize;    // slot stride as sized by the workspace query
  a.err_flag = err_flag;
  a.start_blocks = shared_blocks;        // the suffix pass starts after the shared blocks
  a.slot_base = parts;                   // slots [0, parts) hold the prefix partials
  a.force_split = 1;
  const size_t part_bytes = workspace_bytes_for(B, Hq, D, a.P);
  const size_t need = part_bytes + (p.kernel == 2 ? tc_workspace_bytes(B, Hq, Hkv, D) : 0);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return PA_ERR_WORKSPACE;
  const size_t rows = (size_t)B * Hq * a.P;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* w = static_cast<char*>(workspace);
  a.ws_acc = reinterpret_cast<float*>(w);
  a.ws_m = reinterpret_cast<float*>(w + up(rows * D * 4));
  a.ws_l = reinterpret_cast<float*>(w + up(rows * D * 4) + up(rows * 4));
  if (p.kernel == 2) {
    tc_carve(a, w + part_bytes);
    a.epoch = next_epoch();
    a.wait_ns = tc_wait_ns();
    a.pair_cost = tc_pair_cost();
    a.test_withhold_q = tc_test_withhold_q();
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc;
  if (p.kernel == 2) rc = launch_decode_tc(a, q_dtype, k8, st);
  else if (k8 || v8) rc = launch_decode_simt_kv(a, q_dtype, k_dtype, v_dtype, st);
  else rc = launch_decode_simt(a, q_dtype, st);
  if (rc == PA_OK)
    rc = launch_prefix_tc(a, q_dtype, group_offsets, group_members, num_groups, max_group_size,
                          parts, part_tokens, st, k8, v8);
  if (rc == PA_OK) rc = launch_merge(a, st);
  return rc;
}

}  // namespace

extern "C" {

int pa_decode_shared_prefix(void* out, int out_dtype, const void* query, const void* key_cache,
                            const void* value_cache, int dtype, const int32_t* block_tables,
                            int max_blocks_per_seq, const int32_t* context_lens,
                            const int32_t* shared_blocks, int num_groups,
                            const int32_t* group_offsets, const int32_t* group_members,
                            int max_group_size, int max_shared_blocks, int B, int Hq, int Hkv,
                            int D, int block_size, int num_blocks, float scale,
                            int max_context_len, int partition_size, void* workspace,
                            size_t workspace_bytes, uint32_t* err_flag, void* stream) {
  if (dtype < PA_F32 || dtype > PA_BF16) return PA_ERR_DTYPE;
  return shared_prefix_impl(out, out_dtype, query, dtype, key_cache, dtype, 1.f, value_cache,
                            dtype, 1.f, block_tables, max_blocks_per_seq, context_lens,
                            shared_blocks, num_groups, group_offsets, group_members,
                            max_group_size, max_shared_blocks, B, Hq, Hkv, D, block_size,
                            num_blocks, scale, max_context_len, partition_size, workspace,
                            workspace_bytes, err_flag, stream);
}

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
                               uint32_t* err_flag, void* stream) {
  if (k_dtype < PA_F32 || k_dtype > PA_FP8_E4M3 || v_dtype < PA_F32 || v_dtype > PA_FP8_E4M3)
    return PA_ERR_DTYPE;
  return shared_prefix_impl(out, out_dtype, query, q_dtype, key_cache, k_dtype, k_scale,
                            value_cache, v_dtype, v_scale, block_tables, max_blocks_per_seq,
                            context_lens, shared_blocks, num_groups, group_offsets,
                            group_members, max_group_size, max_shared_blocks, B, Hq, Hkv, D,
                            block_size, num_blocks, scale, max_context_len, partition_size,
                            workspace, workspace_bytes, err_flag, stream);
}

}  // extern "C"

namespace {

// Shared body of pa_prefill and pa_prefill_kv.
int prefill_impl(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                 int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                 const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                 const int32_t* query_start, int B, int T, int max_query_len, int Hq, int Hkv,
                 int D, int block_size, int num_blocks, float scale, int max_context_len,
                 uint32_t* err_flag, void* stream) {
  if (q_dtype < PA_F32 || q_dtype > PA_BF16) return PA_ERR_DTYPE;
  if (out_dtype != PA_F32 && out_dtype != q_dtype) return PA_ERR_DTYPE;
  const bool k8 = k_dtype == PA_FP8_E4M3, v8 = v_dtype == PA_FP8_E4M3;
  if ((!k8 && k_dtype != q_dtype) || (!v8 && v_dtype != q_dtype)) return PA_ERR_DTYPE;
  if (B < 0 || T < 0 || max_query_len < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 ||
      num_blocks < 0 || max_blocks_per_seq <= 0 || max_context_len < 0)
    return PA_ERR_SHAPE;
  if (!supported_shape(Hq, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (!prefix_tc_supported(q_dtype, Hq, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  if ((k8 && !scale_ok(k_scale)) || (v8 && !scale_ok(v_scale))) return PA_ERR_SHAPE;
  // the kernel with the query rows on the MMA's M, unless PA_PREFILL_KERNEL=mq
  // asks for the multi-query kernel (for measurements; 16-bit pools only)
  const char* ov = std::getenv("PA_PREFILL_KERNEL");
  const bool mq = ov && !std::strcmp(ov, "mq");
  const bool fa = prefill_fa_supported(q_dtype, Hq, Hkv, D, block_size) && !(mq && !k8 && !v8);
  if ((k8 || v8) && !fa) return PA_ERR_UNSUPPORTED;
  if (B == 0 || T == 0 || max_query_len == 0) return PA_OK;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens ||
      !query_start)
    return PA_ERR_NULL;
  if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;
  PrefillLaunch p{};
  p.out = out; p.out_dtype = out_dtype; p.q = query;
  p.k_cache = key_cache; p.v_cache = value_cache; p.dtype = q_dtype;
  p.k_dtype = k8 ? PA_FP8_E4M3 : q_dtype;
  p.v_dtype = v8 ? PA_FP8_E4M3 : q_dtype;
  p.v_scale = v8 ? v_scale : 1.f;
  p.block_tables = block_tables; p.max_blocks = max_blocks_per_seq;
  p.context_lens = context_lens; p.query_start = query_start;
  p.B = B; p.T = T; p.max_query_len = max_query_len; p.Hq = Hq; p.Hkv = Hkv; p.bs = block_size;
  p.num_blocks = num_blocks;
  p.scale_log2 = scale * kLog2e * (k8 ? k_scale : 1.f);
  p.max_context_len = max_context_len;
  p.err_flag = err_flag;
  if (fa) return launch_prefill_fa(p, static_cast<cudaStream_t>(stream));
  return launch_prefill_tc(p, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int pa_prefill(void* out, int out_dtype, const void* query, const void* key_cache,
               const void* value_cache, int dtype, const int32_t* block_tables,
               int max_blocks_per_seq, const int32_t* context_lens, const int32_t* query_start,
               int B, int T, int max_query_len, int Hq, int Hkv, int D, int block_size,
               int num_blocks, float scale, int max_context_len, uint32_t* err_flag,
               void* stream) {
  if (dtype < PA_F32 || dtype > PA_BF16) return PA_ERR_DTYPE;
  return prefill_impl(out, out_dtype, query, dtype, key_cache, dtype, 1.f, value_cache, dtype, 1.f,
                      block_tables, max_blocks_per_seq, context_lens, query_start, B, T,
                      max_query_len, Hq, Hkv, D, block_size, num_blocks, scale, max_context_len,
                      err_flag, stream);
}

int pa_prefill_kv(void* out, int out_dtype, const void* query, int q_dtype, const void* key_cache,
                  int k_dtype, float k_scale, const void* value_cache, int v_dtype, float v_scale,
                  const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, const int32_t* query_start, int B, int T,
                  int max_query_len, int Hq, int Hkv, int D, int block_size, int num_blocks,
                  float scale, int max_context_len, uint32_t* err_flag, void* stream) {
  if (k_dtype < PA_F32 || k_dtype > PA_FP8_E4M3 || v_dtype < PA_F32 || v_dtype > PA_FP8_E4M3)
    return PA_ERR_DTYPE;
  return prefill_impl(out, out_dtype, query, q_dtype, key_cache, k_dtype, k_scale, value_cache,
                      v_dtype, v_scale, block_tables, max_blocks_per_seq, context_lens,
                      query_start, B, T, max_query_len, Hq, Hkv, D, block_size, num_blocks,
                      scale, max_context_len, err_flag, stream);
}

int pa_swap_blocks(void* dst_key, void* dst_value, const void* src_key, const void* src_value,
                   int dtype, const int64_t* block_mapping, int num_pairs, int Hkv, int D,
                   int block_size, int src_blocks, int dst_blocks, uint32_t* err_flag,
                   void* stream) {
  if (dtype < PA_F32 || dtype > PA_FP8_E4M3) return PA_ERR_DTYPE;
  if (num_pairs < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || src_blocks < 0 ||
      dst_blocks < 0)
    return PA_ERR_SHAPE;
  if (!supported_shape(Hkv, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!dst_key || !dst_value || !src_key || !src_value || !block_mapping) return PA_ERR_NULL;
  if (!aligned16(dst_key) || !aligned16(dst_value) || !aligned16(src_key) || !aligned16(src_value))
    return PA_ERR_ALIGN;
  return launch_swap_blocks(dst_key, dst_value, src_key, src_value, esize_of(dtype),
                            block_mapping, num_pairs, Hkv, D, block_size, src_blocks, dst_blocks,
                            err_flag, static_cast<cudaStream_t>(stream));
}

int pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                         int dtype, const int64_t* slot_mapping, int T, int Hkv, int D,
                         int block_size, int num_blocks, uint32_t* err_flag, void* stream) {
  if (dtype < PA_F32 || dtype > PA_BF16) return PA_ERR_DTYPE;
  if (T < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0) return PA_ERR_SHAPE;
  if (!supported_shape(Hkv, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (T == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
    return PA_ERR_ALIGN;
  return launch_reshape_and_cache(key, value, key_cache, value_cache, esize_of(dtype),
                                  slot_mapping, T, Hkv, D, block_size, num_blocks, err_flag,
                                  static_cast<cudaStream_t>(stream));
}

int pa_copy_blocks(void* key_cache, void* value_cache, int dtype, const int64_t* block_mapping,
                   int num_pairs, int Hkv, int D, int block_size, int num_blocks,
                   uint32_t* err_flag, void* stream) {
  if (dtype < PA_F32 || dtype > PA_FP8_E4M3) return PA_ERR_DTYPE;
  if (num_pairs < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks < 0)
    return PA_ERR_SHAPE;
  if (!supported_shape(Hkv, Hkv, D, block_size)) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_mapping) return PA_ERR_NULL;
  if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_ALIGN;
  return launch_copy_blocks(key_cache, value_cache, esize_of(dtype), block_mapping, num_pairs,
                            Hkv, D, block_size, num_blocks, err_flag,
                            static_cast<cudaStream_t>(stream));
}

}  // extern "C"
