// cache_ops.cu -- reshape_and_cache (scatter new tokens to their slots) and
// copy_blocks (copy-on-write of whole physical blocks).
//
// Both are pure byte movement, so both work in 16-byte vectors regardless of
// the element type: one physical row of a token is Hkv * D * esize bytes
// (a multiple of 16 for every supported shape), one physical block is
// block_size such rows. Both are tiny (a decode step writes one row per
// sequence and copies at most a few blocks) and launch-bound; the launch
// shapes below aim at few, short-lived CTAs.
#include "pa_internal.h"

namespace pa {

// One thread moves one 16-byte chunk of one token's K row and the same chunk
// of its V row. row16 = chunks per token row.
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ key,
                                         const uint4* __restrict__ value,
                                         uint4* __restrict__ key_cache,
                                         uint4* __restrict__ value_cache,
                                         const int64_t* __restrict__ slot_mapping, int T,
                                         int row16, long long num_slots, uint32_t* err_flag) {
  pdl_trigger();
  pdl_wait();
  long long n = (long long)T * row16;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    int t = (int)(i / row16);
    int c = (int)(i - (long long)t * row16);
    int64_t s = slot_mapping[t];
    if (s < 0) continue;                      // padding token
    if (s >= num_slots) {                     // never write outside the pool
      if (c == 0) flag_error(err_flag, PA_DEV_BAD_SLOT);
      continue;
    }
    // slot s is row s of the [num_blocks * block_size, Hkv * D] view of the pool
    size_t dst = (size_t)s * row16 + c;
    size_t src = (size_t)t * row16 + c;
    key_cache[dst] = key[src];
    value_cache[dst] = value[src];
  }
}

// blockIdx.x = pair, blockIdx.z = 0 (K) / 1 (V); y-blocks stride the block.
__global__ void copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                                   const int64_t* __restrict__ block_mapping, int block16,
                                   int num_blocks, uint32_t* err_flag) {
  pdl_trigger();
  pdl_wait();
  int p = blockIdx.x;
  int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(err_flag, PA_DEV_BAD_PAIR);
    return;
  }
  uint4* pool = blockIdx.z == 0 ? key_cache : value_cache;
  const uint4* s = pool + (size_t)src * block16;
  uint4* d = pool + (size_t)dst * block16;
  for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < block16; i += gridDim.y * blockDim.x)
    d[i] = s[i];
}

int launch_reshape_and_cache(const void* key, const void* value, void* key_cache,
                             void* value_cache, int esize, const int64_t* slot_mapping, int T,
                             int Hkv, int D, int block_size, int num_blocks, uint32_t* err_flag,
                             cudaStream_t stream) {
  if (T == 0) return PA_OK;
  int row16 = Hkv * D * esize / 16;
  long long n = (long long)T * row16;
  int threads = 256;
  long long blocks = (n + threads - 1) / threads;
  if (blocks > 8 * kSMs) blocks = 8 * kSMs;
  const cudaError_t e = launch_k(
      reshape_and_cache_kernel, dim3((unsigned)blocks), dim3(threads), 0, stream,
      (const uint4*)key, (const uint4*)value, (uint4*)key_cache, (uint4*)value_cache,
      slot_mapping, T, row16, (long long)num_blocks * block_size, err_flag);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_copy_blocks(void* key_cache, void* value_cache, int esize,
                       const int64_t* block_mapping, int num_pairs, int Hkv, int D,
                       int block_size, int num_blocks, uint32_t* err_flag, cudaStream_t stream) {
  if (num_pairs == 0) return PA_OK;
  int block16 = block_size * Hkv * D * esize / 16;
  int threads = 256;
  int yb = (block16 + threads * 4 - 1) / (threads * 4);   // ~4 vectors per thread
  if (yb < 1) yb = 1;
  dim3 grid(num_pairs, yb, 2);
  const cudaError_t e = launch_k(copy_blocks_kernel, grid, dim3(threads), 0, stream,
                                 (uint4*)key_cache, (uint4*)value_cache, block_mapping, block16,
                                 num_blocks, err_flag);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
