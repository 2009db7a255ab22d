// Device helpers shared by the libdsv4 kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsv4.h"

namespace dsv4 {

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Two adjacent channels (d, d+1), d even.
template <typename T>
__device__ __forceinline__ float2 load2(const T* p);
template <>
__device__ __forceinline__ float2 load2<float>(const float* p) { return *reinterpret_cast<const float2*>(p); }
template <>
__device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
template <typename T>
__device__ __forceinline__ void store2(T* p, float a, float b);
template <>
__device__ __forceinline__ void store2<float>(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
template <>
__device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}

// Rotation of interleaved pair k (of R/2) at integer position p: angle = p * theta^(-2k/R).
// The angle is formed and reduced in double precision so that positions up to 2^20 keep
// full float accuracy in cos/sin.
__device__ __forceinline__ void rope_cos_sin(int64_t p, int k, int R, float theta, float* c, float* s) {
  const double inv = pow((double)theta, -2.0 * (double)k / (double)R);
  const double ang = (double)p * inv;
  double sd, cd;
  sincos(ang, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Cache index of query (b, s): q_index[b,s], or s when the caller passes NULL (prefill).
__device__ __forceinline__ int query_cache_index(const int32_t* q_index, int64_t row, int s) {
  return q_index ? q_index[row] : s;
}

// Pool entries visible to a query at cache index t: an entry is ready once its window closed.
__device__ __forceinline__ int visible_entries(int t, int m, int P_cap) {
  const int v = (t + 1) / m;
  return v < P_cap ? v : P_cap;
}

}  // namespace dsv4
