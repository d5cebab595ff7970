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

// Thread-block clusters: the verification and commit kernels exchange their
// partial results over distributed shared memory inside one cluster.
constexpr int kMaxCluster = 16;

// Largest cluster (16 CTAs if this device schedules non-portable 16-CTA
// clusters of `kernel` with `threads` threads, else the portable 8).  The
// answer is cached per device in `cache`, so the first call -- which also sets
// the kernel's non-portable-cluster attribute -- should come before any
// stream capture.
template <typename Kernel>
inline int cluster_limit(Kernel kernel, int threads, int (&cache)[64], size_t smem = 0) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 8;
  if (cache[dev]) return cache[dev];
  int limit = 8;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxCluster, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kMaxCluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && n > 0) limit = kMaxCluster;
  }
  cudaGetLastError();   // a refused query leaves no sticky error behind
  cache[dev] = limit;
  return limit;
}

// Programmatic dependent launch.  Every library kernel is launched so that it
// may start while the previous kernel on the stream is finishing; it runs its
// own prologue, then pdl_wait() -- which returns once every earlier grid on
// the stream has completed and its memory is visible -- before it touches any
// global data, and pdl_trigger() lets the next kernel launch early.  Both
// are no-ops when there is no such dependency.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Order of a ragged batch over the grid: the CTAs of grid row r (rows are
// dispatched roughly in order) take the sequence with the r-th longest
// prefix (ties: the lower index first), so that the longest work starts
// first and the launch ends with a short tail instead of a long sequence
// started last.  Batches of 2..32 sequences (identity otherwise).  Called by
// whole warps after the dependency wait (the lengths may come from the
// previous kernel); every lane returns the same sequence.
__device__ __forceinline__ int longest_first(const int32_t* seq_lens, int B, int r) {
  if (B <= 1 || B > 32) return r;
  const int lane = (int)threadIdx.x & 31;
  const int len = lane < B ? seq_lens[lane] : 0;
  int rank = 0;
  for (int j = 0; j < B; ++j) {
    const int lj = __shfl_sync(0xffffffffu, len, j);
    rank += (lj > len || (lj == len && j < lane)) ? 1 : 0;
  }
  const unsigned m = __ballot_sync(0xffffffffu, lane < B && rank == r);
  return m ? __ffs(m) - 1 : r;
}

// Relaxed load at device scope: served by L2 (the point of coherence), never
// by a stale L1 line.  For data read before pdl_wait() that kernels further
// back on the stream wrote.
__device__ __forceinline__ int ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Launch `kernel` on `grid` with clusters of `cluster` CTAs (none if the
// cluster is 1x1x1), as a programmatic dependent of the previous kernel.
template <typename Kernel, typename... Args>
inline cudaError_t launch_clustered(Kernel kernel, dim3 grid, dim3 cluster, int threads, size_t smem,
                                    cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  int na = 0;
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster.x * cluster.y * cluster.z > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = cluster.x;
    at[na].val.clusterDim.y = cluster.y;
    at[na].val.clusterDim.z = cluster.z;
    ++na;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Plain grid, programmatic dependent of the previous kernel.
template <typename Kernel, typename... Args>
inline cudaError_t launch_pdl(Kernel kernel, dim3 grid, int threads, size_t smem, cudaStream_t s,
                              Args... args) {
  return launch_clustered(kernel, grid, dim3(1, 1, 1), threads, smem, s, args...);
}

// Launch `kernel` on grid (cx, gy) with clusters of (cx, 1, 1).
template <typename Kernel, typename... Args>
inline cudaError_t launch_cluster(Kernel kernel, int cx, int gy, int threads, size_t smem,
                                  cudaStream_t s, Args... args) {
  return launch_clustered(kernel, dim3(cx, gy, 1), dim3(cx, 1, 1), threads, smem, s, args...);
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
