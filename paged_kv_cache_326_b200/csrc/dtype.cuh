// fp16 / bf16 <-> fp32 helpers on 16-byte vectors of 8 elements.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace pa {

template <typename T>
struct Elem;

template <>
struct Elem<__half> {
  __device__ __forceinline__ static float2 to_float2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
  __device__ __forceinline__ static uint32_t from_float2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <>
struct Elem<__nv_bfloat16> {
  // bf16 is the top half of an fp32: widening is exact bit placement.
  __device__ __forceinline__ static float2 to_float2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  __device__ __forceinline__ static uint32_t from_float2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  float2 a = Elem<T>::to_float2(v.x), b = Elem<T>::to_float2(v.y);
  float2 c = Elem<T>::to_float2(v.z), d = Elem<T>::to_float2(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 v;
  v.x = Elem<T>::from_float2(f[0], f[1]);
  v.y = Elem<T>::from_float2(f[2], f[3]);
  v.z = Elem<T>::from_float2(f[4], f[5]);
  v.w = Elem<T>::from_float2(f[6], f[7]);
  return v;
}

}  // namespace pa
