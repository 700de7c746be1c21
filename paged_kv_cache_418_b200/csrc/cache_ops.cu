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

// reshape_and_cache into pools of per-pool element types: one thread takes 16
// consecutive elements of one token's K row and the same 16 of its V row. A
// pool marked FP8 (KQ / VQ) receives codes: each element (TS = f32, f16 or
// bf16, exact in fp32) is divided by the pool's scale (IEEE division) and
// rounded to E4M3, nearest even, saturating; the other pool receives the 16
// elements bit for bit.
__device__ __forceinline__ uint4 quantise16(const float* f, float scale) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_fp8x2_storage_t c0 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(f[4 * k], scale), __fdiv_rn(f[4 * k + 1], scale)), __NV_SATFINITE,
        __NV_E4M3);
    const __nv_fp8x2_storage_t c1 = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(f[4 * k + 2], scale), __fdiv_rn(f[4 * k + 3], scale)),
        __NV_SATFINITE, __NV_E4M3);
    w[k] = (uint32_t)c0 | ((uint32_t)c1 << 16);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename TS, bool KQ, bool VQ>
__global__ void reshape_and_cache_kv_kernel(const TS* __restrict__ key,
                                            const TS* __restrict__ value, void* __restrict__ key_cache,
                                            void* __restrict__ value_cache, float k_scale,
                                            float v_scale, const int64_t* __restrict__ slot_mapping,
                                            int T, int row16, long long num_slots,
                                            uint32_t* err_flag) {
  pdl_trigger();
  pdl_wait();
  constexpr int N = Vec<TS>::N;                  // source elements per 16-byte load
  long long n = (long long)T * row16;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    int t = (int)(i / row16);
    int c = (int)(i - (long long)t * row16);
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    if (s >= num_slots) {
      if (c == 0) flag_error(err_flag, PA_DEV_BAD_SLOT);
      continue;
    }
    const size_t src = ((size_t)t * row16 + c) * 16;   // first of this thread's 16 elements
    const size_t dst = ((size_t)s * row16 + c) * 16;   // the same element of the pool row
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      const TS* in = which ? value : key;
      const bool q = which ? VQ : KQ;
      void* pool = which ? value_cache : key_cache;
      if (q) {
        float f[16];
#pragma unroll
        for (int k = 0; k < 16 / N; ++k)
          widen16<TS>(*reinterpret_cast<const uint4*>(in + src + k * N), f + k * N);
        *reinterpret_cast<uint4*>(static_cast<uint8_t*>(pool) + dst) =
            quantise16(f, which ? v_scale : k_scale);
      } else {
#pragma unroll
        for (int k = 0; k < 16 / N; ++k)
          reinterpret_cast<uint4*>(static_cast<TS*>(pool) + dst)[k] =
              *reinterpret_cast<const uint4*>(in + src + k * N);
      }
    }
  }
}

// Whole-block copies between two pools (swap out / swap in): blockIdx.x =
// pair, blockIdx.z = 0 (K) / 1 (V); y-blocks stride the block. Either pool
// may be page-locked host memory, read or written over the host link.
__global__ void swap_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                   const uint4* __restrict__ src_k,
                                   const uint4* __restrict__ src_v,
                                   const int64_t* __restrict__ block_mapping, int block16,
                                   int src_blocks, int dst_blocks, uint32_t* err_flag) {
  pdl_trigger();
  pdl_wait();
  int p = blockIdx.x;
  int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) flag_error(err_flag, PA_DEV_BAD_PAIR);
    return;
  }
  const uint4* s = (blockIdx.z == 0 ? src_k : src_v) + (size_t)src * block16;
  uint4* d = (blockIdx.z == 0 ? dst_k : dst_v) + (size_t)dst * block16;
  for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < block16; i += gridDim.y * blockDim.x)
    d[i] = s[i];
}

template <typename TS>
int launch_rac_kv(const void* key, const void* value, void* key_cache, int k_fp8, float k_scale,
                  void* value_cache, int v_fp8, float v_scale, const int64_t* slot_mapping, int T,
                  int row16, long long slots, uint32_t* err_flag, cudaStream_t stream) {
  long long n = (long long)T * row16;
  int threads = 256;
  long long blocks = (n + threads - 1) / threads;
  if (blocks > 8 * kSMs) blocks = 8 * kSMs;
  const TS* k = static_cast<const TS*>(key);
  const TS* v = static_cast<const TS*>(value);
  auto go = [&](auto kern) {
    return launch_k(kern, dim3((unsigned)blocks), dim3(threads), 0, stream, k, v, key_cache,
                    value_cache, k_scale, v_scale, slot_mapping, T, row16, slots, err_flag);
  };
  cudaError_t e;
  if (k_fp8 && v_fp8) e = go(reshape_and_cache_kv_kernel<TS, true, true>);
  else if (k_fp8) e = go(reshape_and_cache_kv_kernel<TS, true, false>);
  else if (v_fp8) e = go(reshape_and_cache_kv_kernel<TS, false, true>);
  else e = go(reshape_and_cache_kv_kernel<TS, false, false>);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int launch_reshape_and_cache_kv(const void* key, const void* value, int src_dtype,
                                void* key_cache, int k_fp8, float k_scale, void* value_cache,
                                int v_fp8, float v_scale, const int64_t* slot_mapping, int T,
                                int Hkv, int D, int block_size, int num_blocks,
                                uint32_t* err_flag, cudaStream_t stream) {
  if (T == 0) return PA_OK;
  const int row16 = Hkv * D / 16;                // 16-element groups per token row
  const long long slots = (long long)num_blocks * block_size;
  switch (src_dtype) {
    case PA_F32:
      return launch_rac_kv<float>(key, value, key_cache, k_fp8, k_scale, value_cache, v_fp8,
                                  v_scale, slot_mapping, T, row16, slots, err_flag, stream);
    case PA_F16:
      return launch_rac_kv<__half>(key, value, key_cache, k_fp8, k_scale, value_cache, v_fp8,
                                   v_scale, slot_mapping, T, row16, slots, err_flag, stream);
    case PA_BF16:
      return launch_rac_kv<__nv_bfloat16>(key, value, key_cache, k_fp8, k_scale, value_cache,
                                          v_fp8, v_scale, slot_mapping, T, row16, slots, err_flag,
                                          stream);
  }
  return PA_ERR_DTYPE;
}

int launch_swap_blocks(void* dst_key, void* dst_value, const void* src_key,
                       const void* src_value, int esize, const int64_t* block_mapping,
                       int num_pairs, int Hkv, int D, int block_size, int src_blocks,
                       int dst_blocks, uint32_t* err_flag, cudaStream_t stream) {
  if (num_pairs == 0) return PA_OK;
  int block16 = block_size * Hkv * D * esize / 16;
  int threads = 256;
  int yb = (block16 + threads * 4 - 1) / (threads * 4);
  if (yb < 1) yb = 1;
  dim3 grid(num_pairs, yb, 2);
  const cudaError_t e = launch_k(swap_blocks_kernel, grid, dim3(threads), 0, stream,
                                 (uint4*)dst_key, (uint4*)dst_value, (const uint4*)src_key,
                                 (const uint4*)src_value, block_mapping, block16, src_blocks,
                                 dst_blocks, err_flag);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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
