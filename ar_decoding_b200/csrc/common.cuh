// common.cuh -- small device helpers shared by the libtidar kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tidar.h"

namespace tidar {

// Device error word: kernels OR bits into *err; tidar_get_device_status reads it.
__device__ __forceinline__ void raise_error(unsigned int* err, unsigned int bits) {
  atomicOr(err, bits);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load N consecutive elements (N*sizeof(T) is 8 or 16 bytes, aligned) as fp32.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[N]) {
  static_assert(N * sizeof(T) == 16 || N * sizeof(T) == 8 || N * sizeof(T) == 4, "vector width");
  if constexpr (sizeof(T) == 4) {
    if constexpr (N == 4) {
      float4 x = *reinterpret_cast<const float4*>(p);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else if constexpr (N == 2) {
      float2 x = *reinterpret_cast<const float2*>(p);
      v[0] = x.x; v[1] = x.y;
    } else {
      v[0] = p[0];
    }
  } else {
    if constexpr (N == 8) {
      uint4 x = *reinterpret_cast<const uint4*>(p);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int i = 0; i < 4; ++i) { float2 f = __bfloat1622float2(h[i]); v[2 * i] = f.x; v[2 * i + 1] = f.y; }
    } else if constexpr (N == 4) {
      uint2 x = *reinterpret_cast<const uint2*>(p);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int i = 0; i < 2; ++i) { float2 f = __bfloat1622float2(h[i]); v[2 * i] = f.x; v[2 * i + 1] = f.y; }
    } else {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(p);
      float2 f = __bfloat1622float2(h);
      v[0] = f.x; v[1] = f.y;
    }
  }
}

template <typename T, int N>
__device__ __forceinline__ void store_vec(T* p, const float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) p[i] = from_f32<T>(v[i]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// Structured-mask predicate on step keys (zone-relative indices only).
// Row rho < k: draft row, sees step keys 0..rho.  Row in block j (1-based):
// sees step keys 0..j-1 and its own block [k + (j-1)k, k + jk).  k = 0: key 0.
// Returned as the two half-open intervals [0, e1) and [b0, b1) of visible keys.
struct StepVis {
  int e1, b0, b1;
};
__host__ __device__ __forceinline__ StepVis step_visibility(int k, int rho) {
  StepVis v;
  if (k == 0) { v.e1 = 1; v.b0 = 0; v.b1 = 0; return v; }
  if (rho < k) { v.e1 = rho + 1; v.b0 = 0; v.b1 = 0; return v; }
  int j = (rho - k) / k + 1;
  v.e1 = j;
  v.b0 = k + (j - 1) * k;
  v.b1 = v.b0 + k;
  return v;
}
__host__ __device__ __forceinline__ bool step_visible(const StepVis& v, int key) {
  return key < v.e1 || (key >= v.b0 && key < v.b1);
}

__host__ __device__ __forceinline__ int rows_per_seq(int k) { return k == 0 ? 1 : k + k * k; }

}  // namespace tidar
