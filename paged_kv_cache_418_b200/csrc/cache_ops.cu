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

// FP8 form of reshape_and_cache: one thread writes 16 codes (one 16-byte
// vector) of one token's K row and the same 16 of its V row. The source
// elements (TS = f32, f16 or bf16) are exact in fp32; each is divided by the
// pool's scale (IEEE division) and rounded to E4M3, nearest even, saturating.
template <typename TS>
__global__ void reshape_and_cache_fp8_kernel(const TS* __restrict__ key, const TS* __restrict__ value,
                                             uint4* __restrict__ key_cache,
                                             uint4* __restrict__ value_cache, float k_scale,
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
    float kf[16], vf[16];
#pragma unroll
    for (int k = 0; k < 16 / N; ++k) {
      widen16<TS>(*reinterpret_cast<const uint4*>(key + src + k * N), kf + k * N);
      widen16<TS>(*reinterpret_cast<const uint4*>(value + src + k * N), vf + k * N);
    }
    uint32_t kw[4], vw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_fp8x2_storage_t k0 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(kf[4 * k], k_scale), __fdiv_rn(kf[4 * k + 1], k_scale)),
          __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t k1 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(kf[4 * k + 2], k_scale), __fdiv_rn(kf[4 * k + 3], k_scale)),
          __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t v0 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(vf[4 * k], v_scale), __fdiv_rn(vf[4 * k + 1], v_scale)),
          __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t v1 = __nv_cvt_float2_to_fp8x2(
          make_float2(__fdiv_rn(vf[4 * k + 2], v_scale), __fdiv_rn(vf[4 * k + 3], v_scale)),
          __NV_SATFINITE, __NV_E4M3);
      kw[k] = (uint32_t)k0 | ((uint32_t)k1 << 16);
      vw[k] = (uint32_t)v0 | ((uint32_t)v1 << 16);
    }
    const size_t dst = (size_t)s * row16 + c;
    key_cache[dst] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
    value_cache[dst] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
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

int launch_reshape_and_cache_fp8(const void* key, const void* value, int src_dtype,
                                 void* key_cache, void* value_cache, float k_scale,
                                 float v_scale, const int64_t* slot_mapping, int T, int Hkv,
                                 int D, int block_size, int num_blocks, uint32_t* err_flag,
                                 cudaStream_t stream) {
  if (T == 0) return PA_OK;
  int row16 = Hkv * D / 16;                      // 16-code vectors per token row
  long long n = (long long)T * row16;
  int threads = 256;
  long long blocks = (n + threads - 1) / threads;
  if (blocks > 8 * kSMs) blocks = 8 * kSMs;
  const long long slots = (long long)num_blocks * block_size;
  cudaError_t e;
  switch (src_dtype) {
    case PA_F32:
      e = launch_k(reshape_and_cache_fp8_kernel<float>, dim3((unsigned)blocks), dim3(threads), 0,
                   stream, (const float*)key, (const float*)value, (uint4*)key_cache,
                   (uint4*)value_cache, k_scale, v_scale, slot_mapping, T, row16, slots, err_flag);
      break;
    case PA_F16:
      e = launch_k(reshape_and_cache_fp8_kernel<__half>, dim3((unsigned)blocks), dim3(threads), 0,
                   stream, (const __half*)key, (const __half*)value, (uint4*)key_cache,
                   (uint4*)value_cache, k_scale, v_scale, slot_mapping, T, row16, slots, err_flag);
      break;
    case PA_BF16:
      e = launch_k(reshape_and_cache_fp8_kernel<__nv_bfloat16>, dim3((unsigned)blocks),
                   dim3(threads), 0, stream, (const __nv_bfloat16*)key,
                   (const __nv_bfloat16*)value, (uint4*)key_cache, (uint4*)value_cache, k_scale,
                   v_scale, slot_mapping, T, row16, slots, err_flag);
      break;
    default:
      return PA_ERR_DTYPE;
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
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
