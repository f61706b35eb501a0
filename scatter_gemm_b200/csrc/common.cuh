// common.cuh -- element types and small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lora {

// Element-type traits: bf16 / fp16 stored as 16-bit words, widened to fp32
// for arithmetic and rounded once (to nearest even) on the way out.
struct Bf16 {
  using T = __nv_bfloat16;
  static __device__ __forceinline__ float to_f32(T v) { return __bfloat162float(v); }
  static __device__ __forceinline__ T from_f32(float v) { return __float2bfloat16_rn(v); }
  static __device__ __forceinline__ float bits_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
  }
  static __device__ __forceinline__ uint16_t f32_to_bits(float v) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
  // two packed elements <-> float2
  static __device__ __forceinline__ float2 u32_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  static __device__ __forceinline__ uint32_t f2_to_u32(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

struct Fp16 {
  using T = __half;
  static __device__ __forceinline__ float to_f32(T v) { return __half2float(v); }
  static __device__ __forceinline__ T from_f32(float v) { return __float2half_rn(v); }
  static __device__ __forceinline__ float bits_to_f32(uint16_t b) {
    return __half2float(__ushort_as_half(b));
  }
  static __device__ __forceinline__ uint16_t f32_to_bits(float v) {
    return __half_as_ushort(__float2half_rn(v));
  }
  static __device__ __forceinline__ float2 u32_to_f2(uint32_t w) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
  }
  static __device__ __forceinline__ uint32_t f2_to_u32(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Slice offsets travel by value in the kernel parameters (no device table,
// no host sync).
struct SliceTable {
  int32_t off[9];  // S+1 entries, S <= 8
  int S;
};

// Stores to global memory by explicit global-space instructions.  A store
// through a generic pointer might alias shared memory, so shared-memory loads
// issued after it wait behind it; these stores cannot alias it.
__device__ __forceinline__ void stg128(void* p, uint4 v) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(__cvta_generic_to_global(p)),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void stg64(void* p, uint2 v) {
  asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(__cvta_generic_to_global(p)), "r"(v.x),
               "r"(v.y)
               : "memory");
}

__device__ __forceinline__ void stg32(void* p, uint32_t v) {
  asm volatile("st.global.b32 [%0], %1;" ::"l"(__cvta_generic_to_global(p)), "r"(v) : "memory");
}

__device__ __forceinline__ void stg16(void* p, uint16_t v) {
  asm volatile("st.global.b16 [%0], %1;" ::"l"(__cvta_generic_to_global(p)), "h"(v) : "memory");
}

// Column c (global base-output column) -> its slice q.
__device__ __forceinline__ int slice_of(const SliceTable& st, int c) {
  int q = 0;
#pragma unroll
  for (int k = 1; k < 8; ++k)
    if (k < st.S && c >= st.off[k]) q = k;
  return q;
}

}  // namespace lora
