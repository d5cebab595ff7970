// commit.cu -- in-place KV commit / evict after verification.
//
// The settled cache is reused and rejected entries are evicted
// (nodesdaily.com (fr), paragraph on the three zones; mauroscia.it "KV Cache";
// exact KV cache in the paper's abstract on fugumt.com).  The accepted drafts
// are always a prefix of the draft zone, so no row moves: rows P+c..P+n-1 are
// zeroed, the length advances to P+c and pages that held only rejected rows
// are released.
//
// Two launches, no device-side waits:
//   scrub   grid (B): sequence b validates its own (P, c, pages), zeroes its
//           rejected rows with 16-byte stores, clears its released page-table
//           entries and writes their ids to its fixed slot range
//           released[b*S .. b*S+S) (-1 padded), then advances seq_lens[b].
//   compact grid (1): stable in-place compaction of `released` to (b, i) order
//           and the count.
#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

__global__ void __launch_bounds__(256) scrub_kernel(CommitArgs a, int slots) {
  const int b = blockIdx.x;
  __shared__ int sP, sc, sok;
  if (threadIdx.x == 0) {
    const int P = a.seq_lens[b], c = a.accept_count[b];
    int ok = 1;
    if (c < 0 || c > a.n) { raise_error(a.err, TIDAR_DEVERR_BAD_COUNT); ok = 0; }
    if (ok && P < 0) { raise_error(a.err, TIDAR_DEVERR_BAD_LEN); ok = 0; }
    if (ok && (P + a.n + a.page_size - 1) / a.page_size > a.max_pages) {
      raise_error(a.err, TIDAR_DEVERR_BAD_LEN); ok = 0;
    }
    for (int r = 0; ok && r < a.n; ++r) {
      const int page = a.page_table[(size_t)b * a.max_pages + (P + r) / a.page_size];
      if (page < 0 || page >= a.num_pages) { raise_error(a.err, TIDAR_DEVERR_BAD_PAGE); ok = 0; }
    }
    sP = P; sc = c; sok = ok;
  }
  __syncthreads();
  int32_t* rel = a.released + (size_t)b * slots;
  if (!sok) {
    for (int i = threadIdx.x; i < slots; i += blockDim.x) rel[i] = -1;
    return;
  }
  const int P = sP, c = sc;
  // zero rows P+c .. P+n-1 of every KV head, K and V (16-byte chunks)
  const int row_chunks = a.D * a.elem_bytes / 16;
  const int per_row = 2 * a.Hkv * row_chunks;
  const int total = (a.n - c) * per_row;
  for (int t = threadIdx.x; t < total; t += blockDim.x) {
    const int r = c + t / per_row;
    const int rem = t % per_row;
    const int which = rem / (a.Hkv * row_chunks);
    const int g = (rem / row_chunks) % a.Hkv;
    const int ch = rem % row_chunks;
    const int pos = P + r;
    const int page = a.page_table[(size_t)b * a.max_pages + pos / a.page_size];
    char* base = static_cast<char*>(which ? a.v_pages : a.k_pages);
    const size_t off = (((size_t)page * a.Hkv + g) * a.page_size + pos % a.page_size) * a.D * a.elem_bytes;
    reinterpret_cast<uint4*>(base + off)[ch] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();   // every thread has read the page table before it changes
  if (threadIdx.x == 0) {
    const int first = (P + c + a.page_size - 1) / a.page_size;
    const int last = (P + a.n + a.page_size - 1) / a.page_size;
    int cnt = 0;
    for (int i = first; i < last; ++i) {
      int32_t* ent = a.page_table + (size_t)b * a.max_pages + i;
      if (*ent >= 0) { rel[cnt++] = *ent; *ent = -1; }
    }
    for (; cnt < slots; ++cnt) rel[cnt] = -1;
    a.seq_lens[b] = P + c;
  }
}

__global__ void __launch_bounds__(1024) compact_kernel(int32_t* released, int total, int32_t* num_released) {
  __shared__ int s_warp[32];
  __shared__ int s_base;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int start = 0; start < total; start += blockDim.x) {
    const int i = start + threadIdx.x;
    const int v = i < total ? released[i] : -1;
    const int keep = v >= 0;
    const unsigned ball = __ballot_sync(0xffffffffu, keep);
    const int before = __popc(ball & ((1u << lane) - 1));
    if (lane == 0) s_warp[w] = __popc(ball);
    __syncthreads();
    int off = 0;
    for (int k = 0; k < w; ++k) off += s_warp[k];
    int chunk_total = 0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) chunk_total += s_warp[k];
    const int base = s_base;
    __syncthreads();                      // all reads of this chunk are done
    if (keep) released[base + off + before] = v;   // destination <= source index
    __syncthreads();
    if (threadIdx.x == 0) s_base = base + chunk_total;
    __syncthreads();
  }
  const int count = s_base;
  for (int i = count + threadIdx.x; i < total; i += blockDim.x) released[i] = -1;
  if (threadIdx.x == 0) *num_released = count;
}

}  // namespace

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t s) {
  const int slots = (a.n + a.page_size - 1) / a.page_size + 1;
  scrub_kernel<<<a.B, 256, 0, s>>>(a, slots);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  compact_kernel<<<1, 1024, 0, s>>>(a.released, a.B * slots, a.num_released);
  return cudaGetLastError();
}

}  // namespace tidar
