// commit.cu -- in-place KV commit / evict after verification.
//
// The settled cache is reused and rejected entries are evicted
// (nodesdaily.com (fr), paragraph on the three zones; mauroscia.it "KV Cache";
// exact KV cache in the paper's abstract on fugumt.com).  The accepted drafts
// are always a prefix of the draft zone, so no row moves: rows P+c..P+n-1 are
// zeroed, the length advances to P+c and pages that held only rejected rows
// are released.
//
// One launch: a single thread-block cluster of C <= 16 CTAs (one per 16 KB
// of rows to zero; one CTA up to 32 KB); CTA r owns the contiguous sequences
// [r*per, (r+1)*per) (with fewer sequences than CTAs, the zeroing of step 3
// is shared by the whole cluster).
//   1. every CTA validates its own sequences (one warp per sequence, the
//      page-table entries loaded by parallel lanes) and counts the pages each
//      releases (-1: invalid, left untouched), then an exclusive scan of the
//      counts over its own range;
//   2. cluster barrier; each CTA reads the other CTAs' totals over distributed
//      shared memory, which gives its base in the (b, i)-ordered release list
//      and the grand total; a second cluster barrier ends all remote reads;
//   3. each CTA zeroes the rejected rows of its sequences with 16-byte stores,
//      writes their released page ids at their final positions, clears those
//      page-table entries and advances seq_lens; the tail of the list is -1.
// No device-side waits besides the two hardware cluster barriers.
#include <cooperative_groups.h>

#include <algorithm>

#include "accept.cuh"
#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace cg = cooperative_groups;

namespace {

constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;

// Shared-memory record of one owned sequence: P, c, release count (-1 =
// invalid), exclusive prefix within the CTA, then the npm page ids that hold
// rows P .. P+n-1 (npm = min(n, ceil(n/ps) + 1)).
struct SeqRec { int P, c, cnt, off; };

// Optional timeline of CTA 0 (build with -DTIDAR_TRACE; absent from normal
// builds): [0] start, [1] after the wait on the previous kernel, [2] validated,
// [3] past the cluster barriers, [4] end.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_commit_trace[8];
#define COMMIT_TRACE(slot) do { if (blockIdx.x == 0 && threadIdx.x == 0) { unsigned long long t_; \
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)); g_commit_trace[(slot)] = t_; } } while (0)
#else
#define COMMIT_TRACE(slot) do {} while (0)
#endif

// kFused: the accept counts are not read but computed here from the chunk
// statistics of a greedy verification (`f`), whose outputs the owner of each
// sequence also writes (tidar_verify_commit).
template <bool kFused>
__global__ void __launch_bounds__(kCThreads) commit_cluster_kernel(CommitArgs a, int slots, int per, int npm,
                                                                    GreedyAcceptArgs f) {
  __shared__ int s_g[kFused ? kCWarps : 1][kFused ? 16 * 16 : 1];   // per-warp block guesses
  COMMIT_TRACE(0);
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  extern __shared__ int s_dyn[];
  SeqRec* s_rec = reinterpret_cast<SeqRec*>(s_dyn);
  int* s_pg = s_dyn + 4 * per;                      // [per][npm]
  // With fewer sequences than CTAs every CTA also keeps a record of every
  // sequence (read in step 1, before any CTA advances a length), so that the
  // whole cluster zeroes the rejected rows instead of their owners alone.
  const bool spread = a.B < C;
  SeqRec* s_all = reinterpret_cast<SeqRec*>(s_pg + per * npm);   // [B] when spread
  int* s_allpg = s_pg + per * npm + 4 * (spread ? a.B : 0);      // [B][npm] when spread
  __shared__ int s_total, s_base, s_grand;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int b0 = rank * per;
  const int nown = max(0, min(a.B, b0 + per) - b0);
  const int ps = a.page_size;
  // Fused with a greedy verification, the kernel before this one is the
  // verification's statistics, which write neither lengths nor page tables;
  // and that kernel passed its own dependency wait before this one could
  // start, so everything earlier on the stream is complete.  The lengths and
  // the page-table entries of the draft rows are therefore read before the
  // wait (relaxed loads, so no stale L1 copy is used), overlapping the
  // statistics' tail.
  const bool early = kFused;
  if (early) {
    // own sequences (spread: every sequence, into the all-sequence records)
    for (int i = wid; i < (spread ? a.B : nown); i += kCWarps) {
      const int b = spread ? i : b0 + i;
      int* pgs = spread ? s_allpg + i * npm : s_pg + i * npm;
      const int P = ld_relaxed(a.seq_lens + b);
      if (P >= 0 && (P + a.n + ps - 1) / ps <= a.max_pages) {
        const int p0 = P / ps, np = (P + a.n - 1) / ps - p0 + 1;
        if (lane < np) pgs[lane] = ld_relaxed(a.page_table + (size_t)b * a.max_pages + p0 + lane);
      }
      if (lane == 0) (spread ? s_all : s_rec)[i].P = P;
    }
    __syncwarp();
  }
  pdl_wait();
  pdl_trigger();
  COMMIT_TRACE(1);

  // 1. validate, count, keep the pages: one warp per sequence (its own
  //    sequences; with `spread`, every sequence -- the loop below)
  for (int i = wid; i < (spread ? 0 : nown); i += kCWarps) {
    const int b = b0 + i;
    const int P = early ? s_rec[i].P : a.seq_lens[b];
    const int c = kFused ? greedy_accept_warp(f, a.n, a.k, b, s_g[kFused ? wid : 0], true) : a.accept_count[b];
    COMMIT_TRACE(5);
    int ok = 1;
    if (c < 0 || c > a.n) { ok = 0; if (lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_COUNT); }
    if (ok && (P < 0 || (P + a.n + ps - 1) / ps > a.max_pages)) {
      ok = 0;
      if (lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    }
    if (ok) {
      const int p0 = P / ps, np = (P + a.n - 1) / ps - p0 + 1;   // np <= npm <= 16
      bool bad = false;
      if (lane < np) {
        const int page = early ? s_pg[i * npm + lane] : a.page_table[(size_t)b * a.max_pages + p0 + lane];
        bad = page < 0 || page >= a.num_pages;
        s_pg[i * npm + lane] = page;
      }
      if (__any_sync(0xffffffffu, bad)) {
        ok = 0;
        if (lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
      }
    }
    if (lane == 0) {
      SeqRec r;
      r.P = P; r.c = c; r.off = 0;
      r.cnt = ok ? (P + a.n + ps - 1) / ps - (P + c + ps - 1) / ps : -1;
      s_rec[i] = r;
    }
  }
  if (spread) {
    // the same per sequence, in every CTA; the owner (CTA b / per) reports the
    // errors and, fused, writes the verification outputs
    for (int b = wid; b < a.B; b += kCWarps) {
      const bool owner = b / per == rank;
      const int P = early ? s_all[b].P : a.seq_lens[b];
      const int c = kFused ? greedy_accept_warp(f, a.n, a.k, b, s_g[kFused ? wid : 0], owner) : a.accept_count[b];
      bool ok = true;
      if (c < 0 || c > a.n) { ok = false; if (owner && lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_COUNT); }
      if (ok && (P < 0 || (P + a.n + ps - 1) / ps > a.max_pages)) {
        ok = false;
        if (owner && lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
      }
      if (ok) {
        const int p0 = P / ps, np = (P + a.n - 1) / ps - p0 + 1;
        bool bad = false;
        if (lane < np) {
          const int page = early ? s_allpg[b * npm + lane] : a.page_table[(size_t)b * a.max_pages + p0 + lane];
          bad = page < 0 || page >= a.num_pages;
          s_allpg[b * npm + lane] = page;
        }
        ok = !__any_sync(0xffffffffu, bad);
        if (!ok && owner && lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
      }
      if (lane == 0) {
        SeqRec r;
        r.P = P; r.c = c; r.off = 0;
        r.cnt = ok ? (P + a.n + ps - 1) / ps - (P + c + ps - 1) / ps : -1;
        s_all[b] = r;
      }
    }
  }
  __syncthreads();
  COMMIT_TRACE(2);
  if (spread) {
    // Every CTA holds every sequence's record: the release-list offsets and
    // the total come from a local scan, and one cluster barrier orders every
    // CTA's reads of the lengths and tables before the owners' writes.
    if (wid == 0) {
      const int v = lane < a.B ? max(s_all[lane].cnt, 0) : 0;      // B < C <= 16 <= 32
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane < a.B) s_all[lane].off = x - v;
      if (lane == 31) s_grand = x;
      if (lane == 0) s_base = 0;
    }
    cl.sync();
  } else if (wid == 0) {
    int run = 0;
    for (int s0 = 0; s0 < nown; s0 += 32) {
      const int i = s0 + lane;
      const int v = i < nown ? max(s_rec[i].cnt, 0) : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < nown) s_rec[i].off = run + x - v;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_total = run;
  }

  // 2. bases across the cluster (one CTA: its own totals, no cluster barrier)
  if (C == 1) {
    __syncthreads();
    if (threadIdx.x == 0) { s_base = 0; s_grand = s_total; }
    __syncthreads();
  }
  if (!spread && C > 1) cl.sync();
  if (!spread && C > 1 && wid == 0) {
    int t = 0;
    if (lane < C) t = *cl.map_shared_rank(&s_total, lane);
    int sb = lane < rank ? t : 0, sg = t;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, o);
      sg += __shfl_xor_sync(0xffffffffu, sg, o);
    }
    if (lane == 0) { s_base = sb; s_grand = sg; }
  }
  if (!spread && C > 1) cl.sync();
  COMMIT_TRACE(3);

  // 3. release and advance (one warp per sequence), then scrub (whole CTA);
  //    no page-table reads from here on
  const int base = s_base;
  for (int i = wid; i < nown; i += kCWarps) {
    const int b = b0 + i;
    const SeqRec r = spread ? s_all[b] : s_rec[i];
    if (r.cnt < 0) continue;                        // invalid: left untouched
    const int p0 = r.P / ps, first = (r.P + r.c + ps - 1) / ps;
    const int* pg = spread ? s_allpg + b * npm : s_pg + i * npm;
    if (lane < r.cnt) {
      a.released[base + r.off + lane] = pg[first - p0 + lane];
      a.page_table[(size_t)b * a.max_pages + first + lane] = -1;
    }
    if (lane == 0) a.seq_lens[b] = r.P + r.c;
  }
  const int row_chunks = a.D * a.elem_bytes / 16;
  const int head_chunks = a.Hkv * row_chunks;       // one row of one of K / V, all heads
  const int cols = 2 * head_chunks;                  // 16-byte pieces of one cache row, K and V
  const int nscrub = spread ? a.B : nown;
  const int t0 = spread ? rank * kCThreads + (int)threadIdx.x : (int)threadIdx.x;
  const int tstep = spread ? C * kCThreads : kCThreads;
  const size_t row_bytes = (size_t)a.D * a.elem_bytes;
  if (tstep % cols == 0) {
    // Each thread keeps one 16-byte column (K or V, head, piece) and walks
    // the rejected rows tstep / cols apart: the column's decomposition is
    // computed once, each store costs a page lookup.
    const int col = t0 % cols, rstep = tstep / cols;
    const int which = col >= head_chunks;
    const int hc = col - which * head_chunks;
    const int g = hc / row_chunks, ch = hc - g * row_chunks;
    char* dbase = static_cast<char*>(which ? a.v_pages : a.k_pages) + (size_t)g * ps * row_bytes + (size_t)ch * 16;
    const size_t page_bytes = (size_t)a.Hkv * ps * row_bytes;
    for (int i = 0; i < nscrub; ++i) {
      const SeqRec r = spread ? s_all[i] : s_rec[i];
      const int* pg = spread ? s_allpg + i * npm : s_pg + i * npm;
      if (r.cnt < 0) continue;
      const int p0 = r.P / ps;
      for (int rr = t0 / cols; rr < a.n - r.c; rr += rstep) {
        const int pos = r.P + r.c + rr;
        const int pq = pos / ps;
        *reinterpret_cast<uint4*>(dbase + (size_t)pg[pq - p0] * page_bytes + (size_t)(pos - pq * ps) * row_bytes) =
            make_uint4(0, 0, 0, 0);
      }
    }
  } else {
    for (int i = 0; i < nscrub; ++i) {
      const SeqRec r = spread ? s_all[i] : s_rec[i];
      const int* pg = spread ? s_allpg + i * npm : s_pg + i * npm;
      if (r.cnt < 0) continue;
      const int p0 = r.P / ps;
      const int total = (a.n - r.c) * cols;
      for (int t = t0; t < total; t += tstep) {
        const int rr = t / cols;
        const int rem = t - rr * cols;
        const int which = rem >= head_chunks;
        const int hc = rem - which * head_chunks;
        const int g = hc / row_chunks, ch = hc - g * row_chunks;
        const int pos = r.P + r.c + rr;
        const int page = pg[pos / ps - p0];
        char* dst = static_cast<char*>(which ? a.v_pages : a.k_pages);
        const size_t off = (((size_t)page * a.Hkv + g) * ps + pos % ps) * row_bytes;
        reinterpret_cast<uint4*>(dst + off)[ch] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  const int grand = s_grand;
  for (int i = grand + rank * kCThreads + (int)threadIdx.x; i < a.B * slots; i += C * kCThreads)
    a.released[i] = -1;
  if (rank == 0 && threadIdx.x == 0) *a.num_released = grand;
  COMMIT_TRACE(4);
}

int commit_npm(int n, int ps) { return min(n, (n + ps - 1) / ps + 1); }

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_commit_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_commit_trace, bytes);
}
#endif

// Per owned sequence: a 4-int record and up to 16 page ids, in the dynamic
// shared memory of the portable cluster of 8 (the worst case) within 200 KB.
constexpr size_t kCommitSmemMax = 200 * 1024;
size_t commit_smem(int per, int npm) { return (size_t)per * (4 + npm) * sizeof(int); }

bool commit_batch_ok(int B, int k, int page_size) {
  const int n = k > 0 ? k : 1;
  return commit_smem((B + 7) / 8, commit_npm(n, page_size)) <= kCommitSmemMax;
}

template <bool kFused>
cudaError_t launch_commit_t(const CommitArgs& a, const GreedyAcceptArgs& f, cudaStream_t s) {
  static int limit_cache[64];
  static bool smem_set[64];
  const int slots = (a.n + a.page_size - 1) / a.page_size + 1;
  // One CTA per 16 KB of rows to zero (at most 32 KB: one CTA, which stores
  // them faster than a cluster barrier takes), up to the largest cluster: with
  // a small batch the CTAs share the zeroing, and a small cluster finds its
  // SMs free while the previous kernel's CTAs still hold most of the others.
  const size_t scrub = (size_t)a.B * a.n * 2 * a.Hkv * a.D * a.elem_bytes;
  const int C = scrub <= (32u << 10)
                    ? 1
                    : (int)std::min<size_t>(cluster_limit(commit_cluster_kernel<kFused>, kCThreads, limit_cache),
                                            (scrub + (16u << 10) - 1) >> 14);
  const int per = (a.B + C - 1) / C;
  const int npm = commit_npm(a.n, a.page_size);
  const size_t smem = commit_smem(per + (a.B < C ? a.B : 0), npm);
  if (smem > kCommitSmemMax) return cudaErrorNotSupported;
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && dev >= 0 && dev < 64 && !smem_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(commit_cluster_kernel<kFused>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCommitSmemMax);
    if (e != cudaSuccess) return e;
    smem_set[dev] = true;
  }
  return launch_cluster(commit_cluster_kernel<kFused>, C, 1, kCThreads, smem, s, a, slots, per, npm, f);
}

cudaError_t launch_commit(const CommitArgs& a, const GreedyAcceptArgs* fused, cudaStream_t s) {
  if (fused) return launch_commit_t<true>(a, *fused, s);
  return launch_commit_t<false>(a, GreedyAcceptArgs{}, s);
}

}  // namespace tidar
