// side_mean.cuh -- one row of the Transient-Global block means ("LongT5 长序列模型完全指南",
// Transient-Global: the tokens of each block are summed and normalised into one
// global token; 源码级证据: padding tokens belong to no block, a trailing partial
// block joins the block before it).  Shared by the standalone aggregation kernel
// and the band kernel's fused prologue, so that both give the same bits.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace swa {

template <typename T>
__device__ __forceinline__ float side_to_f(T x);
template <>
__device__ __forceinline__ float side_to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float side_to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T side_from_f(float x);
template <>
__device__ __forceinline__ float side_from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 side_from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// VEC = 16 bytes of T: columns [cg*VEC, cg*VEC + VEC) of side row s of plane bh,
// from x [planes, n, D] into out [planes, S, D], S = n / kb, V the valid length.
// The sum runs over the block's rows in ascending order in fp32, then one division.
template <typename T>
__device__ __forceinline__ void side_mean_vec(const T* __restrict__ x, T* __restrict__ out, size_t bh,
                                              int s, int cg, int n, int D, int kb, int V) {
  constexpr int VEC = 16 / sizeof(T);
  const int S = n / kb;
  const int lo = s * kb;
  const int hi = min((s == S - 1) ? n : lo + kb, V);
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  for (int j = lo; j < hi; ++j) {
    const uint4 raw = *reinterpret_cast<const uint4*>(x + (bh * n + j) * D + cg * VEC);
    const T* vals = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += side_to_f<T>(vals[e]);
  }
  const int cnt = hi > lo ? hi - lo : 0;
  uint4 res;
  T* o = reinterpret_cast<T*>(&res);
#pragma unroll
  for (int e = 0; e < VEC; ++e) o[e] = side_from_f<T>(cnt ? acc[e] / (float)cnt : 0.f);
  *reinterpret_cast<uint4*>(out + (bh * S + s) * D + cg * VEC) = res;
}

}  // namespace swa
