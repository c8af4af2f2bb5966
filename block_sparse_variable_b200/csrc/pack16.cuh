// pack16.cuh -- small device helpers shared by the kernels: the shared-memory
// window address of a pointer, fp32 <-> 16-bit pair packing (round to nearest
// even) for bf16 and fp16, and the hardware base-2 exponential.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace bsa {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// two fp32 values as one 32-bit word of 16-bit T (lo in the low half)
template <typename T>
struct Pack2;

template <>
struct Pack2<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t x) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&x);
    return __bfloat1622float2(v);
  }
};

template <>
struct Pack2<__half> {
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
  static __device__ __forceinline__ float2 unpack(uint32_t x) {
    __half2 v = *reinterpret_cast<__half2 *>(&x);
    return __half22float2(v);
  }
};

// hardware base-2 exponential (MUFU), flush-to-zero; ex2(-inf) = +0
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace bsa
