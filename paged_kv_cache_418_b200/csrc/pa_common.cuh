// pa_common.cuh -- element types, 16-byte vector helpers and device error bits
// shared by the libpa kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

constexpr int kSMs = 148;           // B200: 2 dies x 74 SMs
constexpr float kLog2e = 1.4426950408889634f;

// Number of T elements in one 16-byte vector.
template <typename T> struct Vec { static constexpr int N = 16 / sizeof(T); };

// Widen the 16-byte vector `v` (N elements of T) to fp32.
template <typename T> __device__ __forceinline__ void widen16(const uint4& v, float* f);

template <> __device__ __forceinline__ void widen16<float>(const uint4& v, float* f) {
  f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void widen16<__half>(const uint4& v, float* f) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __half22float2(h[i]);
    f[2 * i] = t.x; f[2 * i + 1] = t.y;
  }
}
template <> __device__ __forceinline__ void widen16<__nv_bfloat16>(const uint4& v, float* f) {
  // bf16 -> fp32 is exact: the bf16 pattern is the top half of the fp32 one.
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <> __device__ __forceinline__ void widen16<__nv_fp8_e4m3>(const uint4& v, float* f) {
  // E4M3 -> binary16 is exact (every E4M3 value, subnormals included, is a
  // normal or subnormal half), and half -> fp32 is exact.
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * k)) & 0xffffu), __NV_E4M3);
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&h));
      f[4 * i + 2 * k] = t.x;
      f[4 * i + 2 * k + 1] = t.y;
    }
  }
}

// One lane's slice of a K or V row: 8 or 16 bytes, loaded in one instruction.
template <int NB> struct Raw;
template <> struct Raw<16> { using T = uint4; };
template <> struct Raw<8> { using T = uint2; };

template <int NB> __device__ __forceinline__ typename Raw<NB>::T raw_zero();
template <> __device__ __forceinline__ uint4 raw_zero<16>() { return make_uint4(0, 0, 0, 0); }
template <> __device__ __forceinline__ uint2 raw_zero<8>() { return make_uint2(0, 0); }

// Widen E elements of type T held in E * sizeof(T) raw bytes to fp32.
template <typename T, int E>
__device__ __forceinline__ void widen_raw(const typename Raw<E * (int)sizeof(T)>::T& v, float* f) {
  if constexpr (E * sizeof(T) == 16) {
    widen16<T>(v, f);
  } else {
    static_assert(sizeof(T) == 1 && E == 8, "8-byte slices hold 8 FP8 codes");
    const uint32_t w[2] = {v.x, v.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * k)) & 0xffffu), __NV_E4M3);
        const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&h));
        f[4 * i + 2 * k] = t.x;
        f[4 * i + 2 * k + 1] = t.y;
      }
    }
  }
}

// Round fp32 to the output type (round to nearest even) and store.
__device__ __forceinline__ void store_out(void* base, size_t i, float x, int out_dtype) {
  if (out_dtype == PA_F32) reinterpret_cast<float*>(base)[i] = x;
  else if (out_dtype == PA_F16) reinterpret_cast<__half*>(base)[i] = __float2half_rn(x);
  else reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
}

// Streaming 16-byte load of data read exactly once (K/V rows): keep L1 clean.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
template <int NB> __device__ __forceinline__ typename Raw<NB>::T ld_stream(const void* p) {
  if constexpr (NB == 16) return ld_stream16(p);
  else return ld_stream8(p);
}

__device__ __forceinline__ void flag_error(uint32_t* err_flag, uint32_t bit) {
  if (err_flag) atomicOr(err_flag, bit);
}

// Programmatic dependent launch. Every kernel of the library lets the next
// kernel in its stream be scheduled as soon as all of its own CTAs are running
// (pdl_trigger), and touches global memory only after the previous kernel has
// completed and its writes are visible (pdl_wait). Without the launch
// attribute both are no-ops and the stream serialises as usual.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with the programmatic-stream-serialisation attribute (unless the
// environment sets PA_PDL=0).
bool pdl_enabled();
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

}  // namespace pa
