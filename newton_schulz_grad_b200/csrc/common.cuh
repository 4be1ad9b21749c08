// Device helpers shared by the elementwise and FFMA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bounds.cuh"

namespace dmuon {


template <typename T>
struct Elt;

template <>
struct Elt<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};

template <>
struct Elt<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  // round to nearest even
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// Load 8 consecutive elements starting at p into fp32 (vectorised when `vec`;
// otherwise element by element, only the first `valid` ones, the rest 0).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8], bool vec, int valid);

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8], bool vec, int valid) {
  if (vec) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (i < valid) ? p[i] : 0.f;
  }
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8], bool vec,
                                                     int valid) {
  if (vec) {
    uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (i < valid) ? __bfloat162float(p[i]) : 0.f;
  }
}

// Store 8 fp32 values as T (already representable in T when T is bf16 and
// the caller rounded; conversion here rounds to nearest even otherwise).
template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&v)[8], bool vec, int valid);

template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&v)[8], bool vec, int valid) {
  if (vec) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < valid) p[i] = v[i];
  }
}

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8], bool vec,
                                                      int valid) {
  if (vec) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = raw;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < valid) p[i] = __float2bfloat16_rn(v[i]);
  }
}

template <typename T>
__device__ __forceinline__ float round_to(float v) {
  return Elt<T>::to_f(Elt<T>::from_f(v));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace dmuon
