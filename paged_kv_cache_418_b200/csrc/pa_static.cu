// pa_static.cu -- pa_decode_static: paged decode attention for callers that
// cannot allocate device memory.
//
// Some callers are handed only their input and output device buffers and may
// not allocate anything themselves: a plugin inside an engine that owns every
// byte of device memory, a C program whose device memory is fixed at start,
// or a host framework that forbids allocation inside its step. pa_decode
// asks such callers for a workspace they cannot provide when contexts are
// split. This entry point takes the same inputs and outputs but no workspace:
// the scratch is a file-scope device array of PA_STATIC_SCRATCH_BYTES that
// lives in this library's module, so the library calls no allocator at all.
//
// Costs and rules of that choice:
//  - every GPU that loads this module holds the array until the process exits;
//  - all calls in one CUDA context share one array; nothing in it needs to
//    start at zero (every scratch value the kernels read is written earlier in
//    the same call), and it keeps the last call's partial results;
//  - two calls that overlap on the GPU (other streams, other threads) race on
//    the array: order them on one stream or with events;
//  - the array's device address belongs to the CUDA context the module was
//    loaded in. A call whose stream is not capturing looks it up afresh in the
//    context current at that call (a second context on the same device, or a
//    device reset, therefore gets its own address). A call whose stream is
//    capturing cannot do that lookup safely and reuses the address found by
//    an earlier non-capturing call in the same context; with none, it fails
//    with PA_ERR_CUDA. So make one call outside capture first.
#include <mutex>

#include "pa_internal.h"

namespace {

// The scratch itself. In host code this name is only a stand-in for the
// device object: its address must come from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

// Addresses found by non-capturing calls, per CUDA context (for capturing calls).
struct CtxAddr {
  void* ctx;
  void* addr;
};
constexpr int kMaxContexts = 64;
CtxAddr g_seen[kMaxContexts] = {};
int g_nseen = 0;
std::mutex g_mu;

using CtxGetCurrentFn = int (*)(void**);   // CUresult cuCtxGetCurrent(CUcontext*)

// The driver's current context (no link dependency on libcuda: the runtime
// hands out the driver entry point).
bool current_context(void** ctx) {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  *ctx = nullptr;
  return fn && fn(ctx) == 0 && *ctx != nullptr;
}

// Device address of the scratch in the current context.
int scratch_address(cudaStream_t stream, void** addr) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) { cudaGetLastError(); return PA_ERR_CUDA; }
  void* p = nullptr;
  if (cs == cudaStreamCaptureStatusNone) {
    // the lookup also makes the runtime set up its context if it has none yet
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
  }
  void* ctx = nullptr;
  if (!current_context(&ctx)) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  int slot = -1;
  for (int i = 0; i < g_nseen; ++i)
    if (g_seen[i].ctx == ctx) slot = i;
  if (cs != cudaStreamCaptureStatusNone) {
    if (slot < 0) return PA_ERR_CUDA;       // no lookup outside capture in this context yet
    *addr = g_seen[slot].addr;
    return PA_OK;
  }
  if (slot < 0) {
    slot = g_nseen < kMaxContexts ? g_nseen++ : (int)(reinterpret_cast<uintptr_t>(ctx) % kMaxContexts);
    g_seen[slot].ctx = ctx;
  }
  g_seen[slot].addr = p;
  *addr = p;
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_static(void* out, int out_dtype, const void* query,
                                const void* key_cache, const void* value_cache, int dtype,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int B, int Hq, int Hkv, int D,
                                int block_size, int num_blocks, float scale, int max_context_len,
                                int partition_size, uint32_t* err_flag, void* stream) {
  // the scratch bytes of the very plan pa_decode will make for these arguments
  // (argument errors are left to pa_decode, which reports them before any launch)
  size_t need = 0;
  if (B > 0 && Hq > 0 && D > 0 && block_size > 0 && max_context_len >= 0 && partition_size >= 0) {
    const pa::DecodePlan p =
        pa::plan_decode(dtype, B, Hq, Hkv, D, block_size, max_context_len, partition_size);
    need = pa::decode_scratch_bytes(p, B, Hq, Hkv, D);
  }
  if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
  if (rc != PA_OK) return rc;
  return pa_decode(out, out_dtype, query, key_cache, value_cache, dtype, block_tables,
                   max_blocks_per_seq, context_lens, B, Hq, Hkv, D, block_size, num_blocks, scale,
                   max_context_len, partition_size, need ? scratch : nullptr,
                   need ? (size_t)PA_STATIC_SCRATCH_BYTES : 0, err_flag, stream);
}
