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
//  - all calls on a device share one array; nothing in it needs to start at
//    zero (every scratch value the kernels read is written earlier in the same
//    call), and it keeps the last call's partial results;
//  - two calls that overlap on the GPU (other streams, other threads) race on
//    the array: order them on one stream or with events;
//  - the device address of the array is looked up once per device, by the
//    first call made with that device current; make that first call before
//    any stream capture.
#include <mutex>

#include "pa_internal.h"

namespace {

// The scratch itself. In host code this name is only a stand-in for the
// device object: its address must come from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_static_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch for the current device (set up on first use).
int scratch_for_current_device(void** addr) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return PA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_static(void* out, int out_dtype, const void* query,
                                const void* key_cache, const void* value_cache, int dtype,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int B, int Hq, int Hkv, int D,
                                int block_size, int num_blocks, float scale, int max_context_len,
                                int partition_size, uint32_t* err_flag, void* stream) {
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc != PA_OK) return rc;
  const size_t need = pa_workspace_size(B, Hq, Hkv, D, max_context_len, partition_size);
  if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
  return pa_decode(out, out_dtype, query, key_cache, value_cache, dtype, block_tables,
                   max_blocks_per_seq, context_lens, B, Hq, Hkv, D, block_size, num_blocks, scale,
                   max_context_len, partition_size, need ? scratch : nullptr,
                   need ? (size_t)PA_STATIC_SCRATCH_BYTES : 0, err_flag, stream);
}
