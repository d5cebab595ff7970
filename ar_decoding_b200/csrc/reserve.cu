// reserve.cu -- pages for a step's draft rows, from a device stack of free pages.
//
// A step writes its draft rows P..P+n-1 into the cache, and the commit evicts
// the rejected ones and releases their pages (nodesdaily.com (fr), paragraph
// on the three zones: the settled cache is reused, rejected entries are
// evicted).  This call closes that loop on the device: the ids the last commit
// released are pushed on a stack of free pages, then every page-table entry
// that the step's draft rows need and that holds no prefix row, if it is -1,
// pops the stack in (sequence, page index) order.  With the commit's release
// list as input, reserve -> step attention -> verify -> commit repeats with no
// host round-trip (one CUDA graph for many steps).
//
// One CTA (the work is a few loads per sequence):
//   1. thread 0 reads the stack count and the number of returned ids; if they
//      do not fit in the capacity nothing changes (TIDAR_DEVERR_POOL);
//   2. the returned ids are copied on top of the stack;
//   3. one thread per sequence classifies it (skipped with BAD_LEN / BAD_PAGE,
//      else how many entries need a page) into a byte of shared memory, and a
//      block-wide sum gives the total; if the stack is too short no entry
//      changes (TIDAR_DEVERR_POOL);
//   4. a block-wide exclusive scan of the counts, chunk by chunk, gives each
//      sequence the position of its first pop; the t-th pop takes stack slot
//      count-1-t, read from the returned list when that slot was just pushed
//      (no read-after-write through global memory inside the kernel).
// No waits besides __syncthreads.
#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

constexpr int kRThreads = 1024;
constexpr int kRWarps = kRThreads / 32;

// -1: skipped (error bit raised when `report`); else entries that need a page.
__device__ int classify(const ReserveArgs& a, int b, bool report) {
  const int P = a.seq_lens[b];
  const int ps = a.page_size;
  if (P < 0 || P > a.max_prefix || (P + a.n + ps - 1) / ps > a.max_pages) {
    if (report) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    return -1;
  }
  const int lo = P / ps, settled = (P + ps - 1) / ps, hi = (P + a.n + ps - 1) / ps;
  int need = 0;
  for (int i = lo; i < hi; ++i) {
    const int e = a.page_table[(size_t)b * a.max_pages + i];
    if (e >= 0 && e < a.num_pages) continue;
    if (e == -1 && i >= settled) { ++need; continue; }
    if (report) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
    return -1;
  }
  return need;
}

// Exclusive scan of v over the block; *total receives the block's sum.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int w = s_warp[lane];
    int z = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, z, o);
      if (lane >= o) z += y;
    }
    s_warp[lane] = z - w;                       // exclusive warp offsets
    if (lane == 31) s_warp[32] = z;
  }
  __syncthreads();
  const int r = s_warp[wid] + x - v;
  *total = s_warp[32];
  __syncthreads();                              // s_warp is reused by the next call
  return r;
}

__global__ void __launch_bounds__(kRThreads) reserve_kernel(ReserveArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ signed char s_need[];       // [B]
  __shared__ int s_warp[kRWarps + 1];
  __shared__ int s_count, s_ret;

  // 1. stack count and returned ids
  if (threadIdx.x == 0) {
    const int c = *a.free_count;
    const int m = a.returned ? *a.num_returned : 0;
    const bool fits = c >= 0 && c <= a.capacity && m >= 0 && (long long)c + m <= a.capacity;
    if (!fits) raise_error(a.err, TIDAR_DEVERR_POOL);
    s_count = fits ? c : -1;
    s_ret = m;
  }
  __syncthreads();
  const int c0 = s_count, m = s_ret;
  if (c0 < 0) return;

  // 2. push
  for (int t = threadIdx.x; t < m; t += kRThreads) a.free_pages[c0 + t] = a.returned[t];
  const int count = c0 + m;

  // 3. classify and count
  int total = 0;
  for (int base = 0; base < a.B; base += kRThreads) {
    const int b = base + threadIdx.x;
    int need = 0;
    if (b < a.B) {
      need = classify(a, b, true);
      s_need[b] = (signed char)need;
    }
    int part = 0;
    block_exclusive_scan(need > 0 ? need : 0, s_warp, &part);
    total += part;
  }
  if (total > count) {
    if (threadIdx.x == 0) {
      raise_error(a.err, TIDAR_DEVERR_POOL);
      *a.free_count = count;                    // the push stands
    }
    return;
  }

  // 4. pop in (b, i) order
  int done = 0;
  for (int base = 0; base < a.B; base += kRThreads) {
    const int b = base + threadIdx.x;
    const int need = b < a.B ? (int)s_need[b] : 0;
    int part = 0;
    const int off = done + block_exclusive_scan(need > 0 ? need : 0, s_warp, &part);
    if (need > 0) {
      const int P = a.seq_lens[b], ps = a.page_size;
      int t = off;
      for (int i = (P + ps - 1) / ps; i < (P + a.n + ps - 1) / ps; ++i) {
        int32_t* e = &a.page_table[(size_t)b * a.max_pages + i];
        if (*e != -1) continue;
        const int slot = count - 1 - t++;
        *e = slot >= c0 ? a.returned[slot - c0] : a.free_pages[slot];
      }
    }
    done += part;
  }
  if (threadIdx.x == 0) *a.free_count = count - total;
}

}  // namespace

bool reserve_batch_ok(int B) { return B <= kReserveMaxBatch; }

cudaError_t launch_reserve(const ReserveArgs& a, cudaStream_t s) {
  static bool smem_set[64];
  const size_t smem = (size_t)a.B;
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && dev >= 0 && dev < 64 && !smem_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(reserve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kReserveMaxBatch);
    if (e != cudaSuccess) return e;
    smem_set[dev] = true;
  }
  return launch_pdl(reserve_kernel, dim3(1), kRThreads, smem, s, a);
}

}  // namespace tidar
