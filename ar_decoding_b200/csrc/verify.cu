// verify.cu -- fused verification / acceptance / block selection over vocab rows.
//
// "Talk in Autoregression": the carried drafts are scored strictly left to
// right under the AR distribution (nodesdaily.com (fr), paragraph on betting
// on every outcome; mauroscia.it section 1: a good draft is accepted, a bad
// one corrected), so the emitted text follows plain AR sampling exactly
// (engineer-news.pages.dev, section "TiDAR 在做什麼").  The rejection rule is
// the speculative-sampling rule of TiDAR's lineage (Leviathan et al., Chen et
// al., listed on the mauroscia.it page).  The same scan picks the pre-drafted
// mask block that matches the accept count.
//
// Layout of the work (vocab rows are HBM/latency bound; nothing here is a
// contraction):
//   stats:     grid (chunks, rows).  One CTA sweeps CHUNK logits of one row with
//              16-byte loads: exact max / argmax (lowest index on ties) and,
//              for rejection, the fp64 sum of exp(x - chunk max).
//   greedy:    one warp per sequence.  Merges the chunk argmaxes, scans, writes
//              the outputs.
//   rejection: residual (grid (chunks, B)) recomputes the row normalisers from
//              the chunk stats, runs the accept scan (fp64), and sums the
//              sampling weights of its chunk; select (grid (B)) locates the
//              inverse-CDF chunk, scans it in fp64 and writes outputs.
#include <climits>
#include <math.h>

#include <mutex>

#include <cooperative_groups.h>

#include "common.cuh"
#include "accept.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tidar {

namespace cg = cooperative_groups;

namespace {

constexpr int kChunk = 4096;
constexpr int kThreads = 256;
constexpr int kPer = kChunk / kThreads;   // 16 elements per thread

template <typename T>
__device__ __forceinline__ float ld(const T* p, int i) { return to_f32(p[i]); }

// Logit row of q_i (i = 1..k-1: the distribution draft d_{i+1} was drawn
// from) for sequence b.  With draft_block the rows are read in place from the
// previous step's mask-block logits: the selected block j supplied the drafts
// [t*, g_{j,2}, .., g_{j,k}], so d_{i+1} came from slot i+1 of block j.
template <typename T>
__device__ __forceinline__ const T* q_row(const VerifyArgs& a, int b, int i) {
  const T* base = static_cast<const T*>(a.draft_logits);
  if (!a.draft_block) return base + ((size_t)b * (a.k - 1) + (i - 1)) * a.V;
  int j = a.draft_block[b];
  if (j < 1 || j > a.k) j = 1;
  return base + (((size_t)b * a.k + (j - 1)) * a.k + i) * a.V;
}

// Exact argmax merge: larger value wins, equal values -> lower index.
__device__ __forceinline__ void amax_merge(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}

// Loads this thread's kChunk / TH elements of the chunk (runs of one 16-byte
// vector, run r of thread t at c0 + (r * TH + t) * (16 / sizeof(T)), when the
// row is vector aligned; else single elements strided by TH).
template <typename T, int TH = kThreads>
__device__ __forceinline__ int load_chunk(const T* row, int V, int c0, float (&x)[kChunk / TH],
                                          int (&ix)[kChunk / TH], bool vec_ok) {
  constexpr int kPer = kChunk / TH, kThreads = TH;
  constexpr int kVec = 16 / sizeof(T);
  static_assert(kPer % kVec == 0, "whole vectors per thread");
  int cnt = 0;
  if (vec_ok) {
    // the 16-byte loads first, so they are in flight together
    uint4 raw[kPer / kVec];
#pragma unroll
    for (int it = 0; it < kPer / kVec; ++it) {
      const int base = c0 + (it * kThreads + threadIdx.x) * kVec;
      raw[it] = base + kVec <= V ? __ldg(reinterpret_cast<const uint4*>(row + base)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int it = 0; it < kPer / kVec; ++it) {
      const int base = c0 + (it * kThreads + threadIdx.x) * kVec;
      if (base + kVec <= V) {
        float v[kVec];
        load_vec<T, kVec>(reinterpret_cast<const T*>(&raw[it]), v);
#pragma unroll
        for (int e = 0; e < kVec; ++e) { x[it * kVec + e] = v[e]; ix[it * kVec + e] = base + e; }
      } else {
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
          const int id = base + e;
          x[it * kVec + e] = id < V ? ld(row, id) : -INFINITY;
          ix[it * kVec + e] = id < V ? id : INT_MAX;
        }
      }
    }
    cnt = kPer;
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int id = c0 + e * kThreads + threadIdx.x;
      x[e] = id < V ? ld(row, id) : -INFINITY;
      ix[e] = id < V ? id : INT_MAX;
    }
    cnt = kPer;
  }
  return cnt;
}

// Optional timeline (build with -DTIDAR_TRACE; absent from normal builds):
// statistics CTA (0, 0) [0] start, [1] after the wait on the previous kernel,
// [2] end; acceptance warp of sequence 0 [8] start, [9] after the wait, [10]
// end.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_verify_trace[16 * 8];
#define VERIFY_TRACE(cond, slot) do { if (cond) { unsigned long long t_; \
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)); g_verify_trace[(slot)] = t_; } } while (0)
#else
#define VERIFY_TRACE(cond, slot) do {} while (0)
#endif

// One 16-byte vector of the chunk per thread: 1024 threads for fp32 logits,
// 512 for bf16 (the fp64 exponentials of the weights are latency bound at
// fewer threads; one run per thread also makes the inverse CDF one block scan).
template <typename T>
constexpr int rej_threads() { return kChunk / (16 / (int)sizeof(T)); }

// TH threads per chunk: 256 for greedy (no exponentials); rejection uses
// rej_threads<T>() (fp64 exponentials, latency bound at fewer threads).
template <typename T, int TH = kThreads>
__global__ void __launch_bounds__(TH) stats_kernel(VerifyArgs a, ChunkStat* stats, int nchunk,
                                                   bool vec_ok) {
  constexpr int kThreads = TH, kPer = kChunk / TH;
  [[maybe_unused]] const bool tr = blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0;
  VERIFY_TRACE(tr, 0);
  {
    // this CTA's chunk of its row into L2 while the previous kernel ends (a
    // hint: for a q row read through draft_block, the block index is read
    // ahead of the dependency wait with a relaxed load and clamped, so a
    // stale value only prefetches another row of the same tensor)
    const int lo = (int)blockIdx.x * kChunk, hi = min(a.V, lo + kChunk);
    const T* row = nullptr;
    const int prow = a.B * a.n;
    if ((int)blockIdx.y < prow) {
      row = static_cast<const T*>(a.logits) + (size_t)blockIdx.y * a.V;
    } else if (a.mode == TIDAR_REJECTION && a.k > 1) {
      const int qb = ((int)blockIdx.y - prow) / (a.k - 1), qi = ((int)blockIdx.y - prow) % (a.k - 1) + 1;
      const T* base = static_cast<const T*>(a.draft_logits);
      if (!a.draft_block) {
        row = base + ((size_t)qb * (a.k - 1) + (qi - 1)) * a.V;
      } else {
        int jb;
        asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(jb) : "l"(a.draft_block + qb));
        if (jb < 1 || jb > a.k) jb = 1;
        row = base + (((size_t)qb * a.k + (jb - 1)) * a.k + qi) * a.V;
      }
    }
    if (row && hi > lo) prefetch_l2(row + lo, (size_t)(hi - lo) * sizeof(T), (int)threadIdx.x, kThreads);
  }
  pdl_wait();
  pdl_trigger();
  VERIFY_TRACE(tr, 1);
  const int c = blockIdx.x, rr = blockIdx.y;
  const int prow = a.B * a.n;
  const T* row = rr < prow ? static_cast<const T*>(a.logits) + (size_t)rr * a.V
                           : q_row<T>(a, (rr - prow) / (a.k - 1), (rr - prow) % (a.k - 1) + 1);
  float x[kPer];
  int ix[kPer];
  load_chunk<T, TH>(row, a.V, c * kChunk, x, ix, vec_ok);
  float bv = -INFINITY;
  int bi = INT_MAX;
#pragma unroll
  for (int e = 0; e < kPer; ++e) amax_merge(bv, bi, x[e], ix[e]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
    amax_merge(bv, bi, v2, i2);
  }
  __shared__ float sv[kThreads / 32];
  __shared__ int si[kThreads / 32];
  __shared__ double sd[kThreads / 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[w] = bv; si[w] = bi; }
  __syncthreads();
  if constexpr (kThreads / 32 <= 8) {
    if (threadIdx.x == 0) {
      for (int i = 1; i < kThreads / 32; ++i) amax_merge(bv, bi, sv[i], si[i]);
      sv[0] = bv; si[0] = bi;
    }
  } else if (threadIdx.x < 32) {             // many warps: one more exact butterfly
    bv = lane < kThreads / 32 ? sv[lane] : -INFINITY;
    bi = lane < kThreads / 32 ? si[lane] : INT_MAX;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
      amax_merge(bv, bi, v2, i2);
    }
    __syncwarp();
    if (lane == 0) { sv[0] = bv; si[0] = bi; }
  }
  __syncthreads();
  const float cmax = sv[0];
  const int carg = si[0];
  double sum = 0.0;
  if (a.mode == TIDAR_REJECTION) {
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (ix[e] != INT_MAX) sum += exp((double)x[e] - (double)cmax);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) sd[w] = sum;
    __syncthreads();
    if constexpr (kThreads / 32 <= 8) {
      if (threadIdx.x == 0) {
        sum = 0.0;
        for (int i = 0; i < kThreads / 32; ++i) sum += sd[i];
      }
    } else if (threadIdx.x < 32) {
      sum = lane < kThreads / 32 ? sd[lane] : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
  }
  if (threadIdx.x == 0) {
    ChunkStat st;
    st.max = cmax; st.arg = carg; st.sum = sum;
    stats[(size_t)rr * nchunk + c] = st;
  }
  VERIFY_TRACE(tr, 2);
}

// Greedy acceptance from the chunk statistics (one warp per sequence b,
// `greedy_accept_warp`).  The statistics kernel has left an exact
// (max, argmax) per 4096-wide chunk of every logits row -- that sweep runs on
// as many CTAs as there are chunks, since a single SM pulls only some tens of
// GB/s.
constexpr int kAccWarps = 4;
__global__ void __launch_bounds__(kAccWarps * 32) greedy_accept_kernel(VerifyArgs a, const ChunkStat* stats,
                                                                       int nchunk) {
  __shared__ int s_g[kAccWarps][16 * 16];
  [[maybe_unused]] const bool tr = blockIdx.x == 0 && threadIdx.x == 0;
  VERIFY_TRACE(tr, 8);
  pdl_wait();
  pdl_trigger();
  VERIFY_TRACE(tr, 9);
  const int wid = threadIdx.x >> 5;
  const int b = blockIdx.x * kAccWarps + wid;
  if (b >= a.B) return;                           // warp-uniform; no block-wide barrier below
  GreedyAcceptArgs f;
  f.stats = stats; f.nchunk = nchunk; f.drafts = a.drafts; f.block_guesses = a.block_guesses;
  f.accept_count = a.accept_count; f.out_tokens = a.out_tokens; f.next_drafts = a.next_drafts;
  f.selected_block = a.selected_block;
  greedy_accept_warp(f, a.n, a.k, b, s_g[wid], true);
  VERIFY_TRACE(tr, 10);
}

// Row normaliser from chunk stats: M = max of chunk maxima, Z = sum_c
// exp(max_c - M) * sum_c (fp64).
// The loops are unrolled by 8 so that the loads of 8 chunks' statistics go
// out together (one memory round trip per 8 chunks, not one per chunk).
__device__ void row_norm(const ChunkStat* st, int nchunk, double& M, double& Z) {
  float mf = -INFINITY;
#pragma unroll 8
  for (int c = 0; c < nchunk; ++c) mf = fmaxf(mf, st[c].max);
  M = (double)mf;
  Z = 0.0;
#pragma unroll 8
  for (int c = 0; c < nchunk; ++c) Z += exp((double)st[c].max - M) * st[c].sum;
}

// The accept scan for sequence b under the rejection rule; returns j.  Run by
// a whole warp: the n-1 tests are independent once the chunk statistics exist
// (only "stop at the first rejection" orders them), so lane i-1 evaluates
// test i -- the same fp64 arithmetic as a sequential scan -- and a ballot
// finds the first failure: j = that i, or n when every test passes.
template <typename T>
__device__ int rejection_scan_warp(const VerifyArgs& a, int b, const ChunkStat* stats, int nchunk) {
  const int prow = a.B * a.n;
  const int i = (threadIdx.x & 31) + 1;          // this lane's test decides d_{i+1}
  bool fail = false;
  if (i <= a.n - 1) {
    const int d = a.drafts[(size_t)b * a.k + i];
    // the normalisers do not depend on the draft: their loads go out with its
    const size_t lrow = (size_t)b * a.n + (i - 1);
    const size_t qrow = (size_t)b * (a.k - 1) + (i - 1);
    double Mp, Zp, Mq, Zq;
    row_norm(stats + lrow * nchunk, nchunk, Mp, Zp);
    row_norm(stats + (prow + qrow) * nchunk, nchunk, Mq, Zq);
    if (d < 0 || d >= a.V) {
      fail = true;
    } else {
      const double p = exp((double)ld(static_cast<const T*>(a.logits) + lrow * a.V, d) - Mp) / Zp;
      const double q = exp((double)ld(q_row<T>(a, b, i), d) - Mq) / Zq;
      const double u = (double)a.uniforms[(size_t)b * a.n + (i - 1)];
      fail = !(u * q < p);
    }
  }
  const unsigned bal = __ballot_sync(0xffffffffu, fail);
  return bal ? __ffs(bal) : a.n;                 // lowest failing lane L is test L+1
}

// Accept scan and the two normalisers of row j, for sequence b, into shared
// variables of the calling CTA (warp 0: the scan; lanes 0 and 1: the p_j and
// q_j normalisers).  Ends with __syncthreads.
template <typename T>
__device__ void scan_and_norms(const VerifyArgs& a, int b, bool first, const ChunkStat* stats,
                               int nchunk, int* jbuf, int& sj, double& sMp, double& sZp,
                               double& sMq, double& sZq) {
  if (threadIdx.x < 32) {
    const int j = rejection_scan_warp<T>(a, b, stats, nchunk);
    if (threadIdx.x == 0) {
      sj = j;
      if (first) {
        if (jbuf) jbuf[b] = j;
        if (a.draft_block && a.k > 1 && (a.draft_block[b] < 1 || a.draft_block[b] > a.k))
          raise_error(a.err, TIDAR_DEVERR_BAD_COUNT);
      }
      row_norm(stats + ((size_t)b * a.n + (j - 1)) * nchunk, nchunk, sMp, sZp);
    } else if (threadIdx.x == 1 && j < a.n) {      // the q_j normaliser on a second lane
      const size_t qrow = (size_t)a.B * a.n + (size_t)b * (a.k - 1) + (j - 1);
      row_norm(stats + qrow * nchunk, nchunk, sMq, sZq);
    }
  }
  __syncthreads();
}

// The same scan and normalisers with the whole CTA (nchunk <= kNormChunks):
// the chunk statistics of every row the scan can touch -- the n p rows and the
// n-1 q rows of sequence b -- are loaded by all threads at once into shared
// memory, one thread per row then forms (M, Z) with row_norm's arithmetic and
// order, and warp 0 runs the tests from that table.  The lanes' drafts and
// logits at the drafts are loaded before, alongside the statistics.  Ends with
// __syncthreads.
constexpr int kNormChunks = 16, kNormRows = 31;   // n <= 16: 2n - 1 rows
static_assert(kMaxCluster <= kNormChunks, "a cluster's chunks fit the table");
template <typename T>
__device__ void scan_and_norms_block(const VerifyArgs& a, int b, bool first, const ChunkStat* stats,
                                     int nchunk, int& sj, double& sMp, double& sZp, double& sMq,
                                     double& sZq) {
  __shared__ float s_cm[kNormRows * kNormChunks];
  __shared__ double s_cs[kNormRows * kNormChunks];
  __shared__ double s_M[kNormRows], s_Z[kNormRows];
  const int R = 2 * a.n - 1;                          // p rows 0..n-1, then q rows 0..n-2
  // the lanes' test operands: lane i-1 decides d_{i+1}
  const int i = (int)(threadIdx.x & 31) + 1;
  int d = -1;
  float lp = 0.f, lq = 0.f;
  if (threadIdx.x < 32 && i <= a.n - 1) {
    d = a.drafts[(size_t)b * a.k + i];
    if (d >= 0 && d < a.V) {
      lp = ld(static_cast<const T*>(a.logits) + ((size_t)b * a.n + (i - 1)) * a.V, d);
      lq = ld(q_row<T>(a, b, i), d);
    }
  }
  for (int idx = threadIdx.x; idx < R * nchunk; idx += blockDim.x) {
    const int r = idx / nchunk, c = idx - r * nchunk;
    const size_t srow = r < a.n ? (size_t)b * a.n + r : (size_t)a.B * a.n + (size_t)b * (a.k - 1) + (r - a.n);
    const ChunkStat st = stats[srow * nchunk + c];
    s_cm[idx] = st.max;
    s_cs[idx] = st.sum;
  }
  __syncthreads();
  // row_norm's terms exp(max_c - M) sum_c, one thread per (row, chunk), then
  // one thread per row adds them in chunk order (the same arithmetic)
  for (int idx = threadIdx.x; idx < R * nchunk; idx += blockDim.x) {
    const int r = idx / nchunk;
    const float* cm = s_cm + r * nchunk;
    float mf = -INFINITY;
    for (int c = 0; c < nchunk; ++c) mf = fmaxf(mf, cm[c]);
    s_cs[idx] = exp((double)s_cm[idx] - (double)mf) * s_cs[idx];
    if (idx == r * nchunk) s_M[r] = (double)mf;
  }
  __syncthreads();
  if ((int)threadIdx.x < R) {
    const double* terms = s_cs + threadIdx.x * nchunk;
    double Z = 0.0;
    for (int c = 0; c < nchunk; ++c) Z += terms[c];
    s_Z[threadIdx.x] = Z;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    bool fail = false;
    if (i <= a.n - 1) {
      if (d < 0 || d >= a.V) {
        fail = true;
      } else {
        const double p = exp((double)lp - s_M[i - 1]) / s_Z[i - 1];
        const double q = exp((double)lq - s_M[a.n + i - 1]) / s_Z[a.n + i - 1];
        const double u = (double)a.uniforms[(size_t)b * a.n + (i - 1)];
        fail = !(u * q < p);
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, fail);
    const int j = bal ? __ffs(bal) : a.n;             // lowest failing lane L is test L+1
    if (threadIdx.x == 0) {
      sj = j;
      if (first && a.draft_block && a.k > 1 && (a.draft_block[b] < 1 || a.draft_block[b] > a.k))
        raise_error(a.err, TIDAR_DEVERR_BAD_COUNT);
      sMp = s_M[j - 1];
      sZp = s_Z[j - 1];
      if (j < a.n) {
        sMq = s_M[a.n + j - 1];
        sZq = s_Z[a.n + j - 1];
      }
    }
  }
  __syncthreads();
}

// Chunk c's weights of both candidate laws for row j, in load_chunk's layout:
// wp = p_j, wr = max(0, p_j - q_j) (0 when j = n); slots past V hold 0.  The
// probabilities are exp(x - M) times the normaliser's reciprocal (fp64).
template <typename T, int TH = kThreads>
__device__ void chunk_weights(const VerifyArgs& a, int b, int c, int j, double Mp, double iZp,
                              double Mq, double iZq, bool vec_ok, double (&wr)[kChunk / TH],
                              double (&wp)[kChunk / TH]) {
  constexpr int kPer = kChunk / TH;
  const T* prow = static_cast<const T*>(a.logits) + ((size_t)b * a.n + (j - 1)) * a.V;
  float xp[kPer];
  int ix[kPer];
  load_chunk<T, TH>(prow, a.V, c * kChunk, xp, ix, vec_ok);
  if (j < a.n) {
    const T* qrow = q_row<T>(a, b, j);
    float xq[kPer];
    int iq[kPer];
    load_chunk<T, TH>(qrow, a.V, c * kChunk, xq, iq, vec_ok);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const bool ok = ix[e] != INT_MAX;
      const double p = ok ? exp((double)xp[e] - Mp) * iZp : 0.0;
      const double q = ok ? exp((double)xq[e] - Mq) * iZq : 0.0;
      wp[e] = p;
      wr[e] = p - q > 0.0 ? p - q : 0.0;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      wp[e] = ix[e] != INT_MAX ? exp((double)xp[e] - Mp) * iZp : 0.0;
      wr[e] = 0.0;
    }
  }
}

// Block sums of both weight arrays, valid in thread 0 (warp butterflies, then
// the warps in order).
template <int TH = kThreads>
__device__ void block_sums(const double (&wr)[kChunk / TH], const double (&wp)[kChunk / TH], double& out_r,
                           double& out_p) {
  constexpr int kPer = kChunk / TH, kThreads = TH;
  double sr = 0.0, sp = 0.0;
#pragma unroll
  for (int e = 0; e < kPer; ++e) { sr += wr[e]; sp += wp[e]; }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sr += __shfl_xor_sync(0xffffffffu, sr, o);
    sp += __shfl_xor_sync(0xffffffffu, sp, o);
  }
  __shared__ double s1[kThreads / 32], s2[kThreads / 32];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { s1[w] = sr; s2[w] = sp; }
  __syncthreads();
  if constexpr (kThreads / 32 <= 8) {
    if (threadIdx.x == 0) {
      sr = 0.0; sp = 0.0;
      for (int i = 0; i < kThreads / 32; ++i) { sr += s1[i]; sp += s2[i]; }
      out_r = sr;
      out_p = sp;
    }
  } else if (threadIdx.x < 32) {              // many warps: their sums by one more butterfly
    sr = threadIdx.x < kThreads / 32 ? s1[threadIdx.x] : 0.0;
    sp = threadIdx.x < kThreads / 32 ? s2[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sr += __shfl_xor_sync(0xffffffffu, sr, o);
      sp += __shfl_xor_sync(0xffffffffu, sp, o);
    }
    if (threadIdx.x == 0) { out_r = sr; out_p = sp; }
  }
}

// Inverse CDF over this CTA's chunk from weights held in load_chunk's layout:
// runs of L contiguous elements, run r of thread t starting at
// c0 + (r * TH + t) * L (L = the vector width, or 1 for scalar loads).
// Index-ordered running sums come from one block scan per run; the smallest
// id with target < running sum is the sample.  Writes the outputs of b.
template <int L, int TH = kThreads>
__device__ void select_from_regs(const VerifyArgs& a, int b, int j, int chunk, double target,
                                 const double (&w)[kChunk / TH]) {
  constexpr int kPer = kChunk / TH, kThreads = TH;
  __shared__ double s_wsum[kThreads / 32];
  __shared__ int s_found, s_last;
  if (threadIdx.x == 0) { s_found = INT_MAX; s_last = -1; }
  const int c0 = chunk * kChunk;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  double base = 0.0;
  int hit = INT_MAX, last_nz = -1;
#pragma unroll
  for (int r = 0; r < kPer / L; ++r) {
    double ts = 0.0;
#pragma unroll
    for (int e = 0; e < L; ++e) ts += w[r * L + e];
    double x = ts;                                   // inclusive scan over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    const double up = __shfl_up_sync(0xffffffffu, x, 1);
    const double excl = lane ? up : 0.0;             // lanes before this one
    if (lane == 31) s_wsum[wid] = x;
    __syncthreads();
    double wpre = 0.0, tot = 0.0;
    for (int k2 = 0; k2 < kThreads / 32; ++k2) {
      const double v = s_wsum[k2];
      if (k2 < wid) wpre += v;
      tot += v;
    }
    __syncthreads();                                 // s_wsum is rewritten next run
    double cum = base + wpre + excl;
#pragma unroll
    for (int e = 0; e < L; ++e) {
      const int id = c0 + (r * kThreads + (int)threadIdx.x) * L + e;
      cum += w[r * L + e];
      if (id < a.V) {
        if (hit == INT_MAX && target < cum) hit = id;
        if (w[r * L + e] > 0.0) last_nz = id;
      }
    }
    base += tot;
  }
  if (hit != INT_MAX) atomicMin(&s_found, hit);
  if (last_nz >= 0) atomicMax(&s_last, last_nz);
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = s_found;
    if (t == INT_MAX) t = s_last >= 0 ? s_last : min(c0 + kChunk, a.V) - 1;
    write_outputs_warp(a, b, j, t);
  }
}

// Inverse CDF inside the located chunk: smallest t with target < the running
// sum of w (fp64 block scan in index order, kPer contiguous elements per
// thread); writes the outputs of sequence b.  Called by the whole CTA.
template <typename T>
__device__ void select_in_chunk(const VerifyArgs& a, int b, int j, int chunk, bool resid,
                                double target, double Mp, double iZp, double Mq, double iZq) {
  __shared__ int s_found, s_last;
  __shared__ double s_scan[kThreads];
  if (threadIdx.x == 0) { s_found = INT_MAX; s_last = -1; }
  const int c0 = chunk * kChunk;
  const T* prow = static_cast<const T*>(a.logits) + ((size_t)b * a.n + (j - 1)) * a.V;
  const T* qrow = resid ? q_row<T>(a, b, j) : nullptr;
  double w[kPer];
  double tsum = 0.0;
  int last_nz = -1;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int id = c0 + threadIdx.x * kPer + e;
    double v = 0.0;
    if (id < a.V) {
      const double p = exp((double)ld(prow, id) - Mp) * iZp;
      if (resid) {
        const double q = exp((double)ld(qrow, id) - Mq) * iZq;
        v = p - q > 0.0 ? p - q : 0.0;
      } else {
        v = p;
      }
      if (v > 0.0) last_nz = id;
    }
    w[e] = v;
    tsum += v;
  }
  s_scan[threadIdx.x] = tsum;
  __syncthreads();
  // Hillis-Steele inclusive scan over the per-thread sums
  for (int off = 1; off < kThreads; off <<= 1) {
    const double v = threadIdx.x >= (unsigned)off ? s_scan[threadIdx.x - off] : 0.0;
    __syncthreads();
    s_scan[threadIdx.x] += v;
    __syncthreads();
  }
  double cum = threadIdx.x ? s_scan[threadIdx.x - 1] : 0.0;
  int hit = INT_MAX;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int id = c0 + threadIdx.x * kPer + e;
    cum += w[e];
    if (hit == INT_MAX && id < a.V && target < cum) hit = id;
  }
  if (hit != INT_MAX) atomicMin(&s_found, hit);
  if (last_nz >= 0) atomicMax(&s_last, last_nz);
  __syncthreads();
  if (threadIdx.x < 32) {
    int t = s_found;
    if (t == INT_MAX) t = s_last >= 0 ? s_last : min(c0 + kChunk, a.V) - 1;
    write_outputs_warp(a, b, j, t);
  }
}

// Per (chunk, b): the sampling weights' chunk sums (vocabularies of more
// chunks than a cluster holds).
template <typename T>
__global__ void __launch_bounds__(kThreads) residual_kernel(VerifyArgs a, const ChunkStat* stats,
                                                            int nchunk, double* wsum, int* jbuf,
                                                            bool vec_ok) {
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x, b = blockIdx.y;
  __shared__ int sj;
  __shared__ double sMp, sZp, sMq, sZq;
  scan_and_norms<T>(a, b, c == 0, stats, nchunk, jbuf, sj, sMp, sZp, sMq, sZq);
  double wr[kPer], wp[kPer];
  chunk_weights<T>(a, b, c, sj, sMp, 1.0 / sZp, sMq, sj < a.n ? 1.0 / sZq : 0.0, vec_ok, wr, wp);
  double sr = 0.0, sp = 0.0;
  block_sums(wr, wp, sr, sp);
  if (threadIdx.x == 0) {
    wsum[((size_t)b * nchunk + c) * 2 + 0] = sr;
    wsum[((size_t)b * nchunk + c) * 2 + 1] = sp;
  }
}

// Inverse CDF from the chunk sums of residual_kernel (one CTA per sequence).
template <typename T>
__global__ void __launch_bounds__(kThreads) select_kernel(VerifyArgs a, const ChunkStat* stats,
                                                          int nchunk, const double* wsum,
                                                          const int* jbuf) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const int j = jbuf[b];
  __shared__ int s_chunk, s_resid;
  __shared__ double s_target, sMp, sZp, sMq, sZq;
  if (threadIdx.x == 0) {
    double tr = 0.0, tp = 0.0;
    for (int c = 0; c < nchunk; ++c) { tr += wsum[((size_t)b * nchunk + c) * 2]; tp += wsum[((size_t)b * nchunk + c) * 2 + 1]; }
    const int resid = (j < a.n) && (tr > 0.0);
    const double total = resid ? tr : tp;
    const double target = (double)a.uniforms[(size_t)b * a.n + (a.n - 1)] * total;
    double cum = 0.0;
    int ch = nchunk - 1;
    for (int c = 0; c < nchunk; ++c) {     // first chunk whose running sum exceeds target
      const double wc = wsum[((size_t)b * nchunk + c) * 2 + (resid ? 0 : 1)];
      if (target < cum + wc) { ch = c; break; }
      cum += wc;
      if (c == nchunk - 1) cum -= wc;
    }
    const double rem = target - cum;
    s_chunk = ch;
    s_resid = resid;
    s_target = rem;
    row_norm(stats + ((size_t)b * a.n + (j - 1)) * nchunk, nchunk, sMp, sZp);
  } else if (threadIdx.x == 32 && j < a.n) {       // q_j normaliser, in parallel (used if resid)
    row_norm(stats + ((size_t)a.B * a.n + (size_t)b * (a.k - 1) + (j - 1)) * nchunk, nchunk, sMq, sZq);
  }
  __syncthreads();
  select_in_chunk<T>(a, b, j, s_chunk, s_resid != 0, s_target, sMp, 1.0 / sZp, sMq,
                     s_resid ? 1.0 / sZq : 0.0);
}

// Residual sums and inverse CDF in one launch: one thread-block cluster per
// sequence, CTA c = chunk c.  Each CTA runs the accept scan, sums its chunk's
// weights and leaves them in shared memory; after a cluster barrier every CTA
// reads all chunk sums over distributed shared memory (added in chunk order,
// as select_kernel does), locates the target chunk, and the CTA that owns it
// runs the inverse CDF.  A second cluster barrier keeps every CTA's shared
// memory alive until the remote reads are done.
template <typename T>
__global__ void __launch_bounds__(rej_threads<T>()) resid_select_cluster_kernel(VerifyArgs a,
                                                                        const ChunkStat* stats,
                                                                        int nchunk, bool vec_ok) {
  constexpr int TH = rej_threads<T>(), kPer = kChunk / TH;
  [[maybe_unused]] const bool tr = blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0;
  VERIFY_TRACE(tr, 16);
  pdl_wait();
  pdl_trigger();
  VERIFY_TRACE(tr, 17);
  cg::cluster_group cl = cg::this_cluster();
  const int c = (int)cl.block_rank(), b = blockIdx.y;
  __shared__ int sj, s_chunk, s_resid;
  __shared__ double sMp, sZp, sMq, sZq, s_target;
  __shared__ double s_sum[2];                         // this chunk's (residual, p) sums
  scan_and_norms_block<T>(a, b, c == 0, stats, nchunk, sj, sMp, sZp, sMq, sZq);
  VERIFY_TRACE(tr, 18);
  const int j = sj;
  double wr[kPer], wp[kPer];
  chunk_weights<T, TH>(a, b, c, j, sMp, 1.0 / sZp, sMq, j < a.n ? 1.0 / sZq : 0.0, vec_ok, wr, wp);
  VERIFY_TRACE(tr, 19);
  double sr = 0.0, sp = 0.0;
  block_sums<TH>(wr, wp, sr, sp);
  if (threadIdx.x == 0) { s_sum[0] = sr; s_sum[1] = sp; }
  VERIFY_TRACE(tr, 20);
  cl.sync();
  VERIFY_TRACE(tr, 21);
  if (threadIdx.x < 32) {
    // every CTA's chunk sums, one peer per lane (all distributed shared memory
    // reads in flight at once), into local shared memory; then thread 0 adds
    // them in chunk order (the arithmetic of select_kernel)
    __shared__ double s_all[kMaxCluster][2];
    if ((int)threadIdx.x < nchunk) {
      const double* peer = cl.map_shared_rank(s_sum, (int)threadIdx.x);
      s_all[threadIdx.x][0] = peer[0];
      s_all[threadIdx.x][1] = peer[1];
    }
    __syncwarp();
    if (threadIdx.x == 0) {
      double tr = 0.0, tp = 0.0;
      for (int r = 0; r < nchunk; ++r) {
        tr += s_all[r][0];
        tp += s_all[r][1];
      }
      const int resid = (j < a.n) && (tr > 0.0);
      const double total = resid ? tr : tp;
      const double target = (double)a.uniforms[(size_t)b * a.n + (a.n - 1)] * total;
      double cum = 0.0;
      int ch = nchunk - 1;
      for (int r = 0; r < nchunk; ++r) {
        const double wc = s_all[r][resid ? 0 : 1];
        if (target < cum + wc) { ch = r; break; }
        cum += wc;
        if (r == nchunk - 1) cum -= wc;   // not found: scan the last chunk
      }
      s_chunk = ch;
      s_resid = resid;
      s_target = target - cum;
    }
  }
  VERIFY_TRACE(tr, 22);
  cl.sync();                                          // remote reads done; s_* visible
  VERIFY_TRACE(tr, 23);
  if (s_chunk != c) return;
  // the owner scans the weights it already holds (no reload, no recompute)
  constexpr int kVec = 16 / sizeof(T);
  const double target = s_target;
  if (s_resid) {
    if (vec_ok) select_from_regs<kVec, TH>(a, b, j, c, target, wr);
    else select_from_regs<1, TH>(a, b, j, c, target, wr);
  } else {
    if (vec_ok) select_from_regs<kVec, TH>(a, b, j, c, target, wp);
    else select_from_regs<1, TH>(a, b, j, c, target, wp);
  }
  VERIFY_TRACE(blockIdx.y == 0 && threadIdx.x == 0, 24);
}

template <typename T>
cudaError_t launch_greedy_stats_t(const VerifyArgs& a, cudaStream_t s) {
  const int nchunk = (a.V + kChunk - 1) / kChunk;
  const bool vec_ok = ((size_t)a.V * sizeof(T)) % 16 == 0;
  ChunkStat* stats = static_cast<ChunkStat*>(a.workspace);
  return launch_pdl(stats_kernel<T>, dim3(nchunk, a.B * a.n), kThreads, 0, s, a, stats, nchunk, vec_ok);
}

template <typename T>
cudaError_t launch_greedy(const VerifyArgs& a, cudaStream_t s) {
  cudaError_t e = launch_greedy_stats_t<T>(a, s);
  if (e != cudaSuccess) return e;
  const int nchunk = (a.V + kChunk - 1) / kChunk;
  return launch_pdl(greedy_accept_kernel, dim3((a.B + kAccWarps - 1) / kAccWarps), kAccWarps * 32, 0, s, a,
                    (const ChunkStat*)a.workspace, nchunk);
}

template <typename T>
cudaError_t launch_t(const VerifyArgs& a, cudaStream_t s) {
  if (a.mode == TIDAR_GREEDY) return launch_greedy<T>(a, s);
  const int nchunk = (a.V + kChunk - 1) / kChunk;
  const bool vec_ok = ((size_t)a.V * sizeof(T)) % 16 == 0;
  ChunkStat* stats = static_cast<ChunkStat*>(a.workspace);
  const int rows = a.B * a.n + (a.mode == TIDAR_REJECTION ? a.B * (a.k > 1 ? a.k - 1 : 0) : 0);
  cudaError_t e = a.mode == TIDAR_REJECTION
                      ? launch_pdl(stats_kernel<T, rej_threads<T>()>, dim3(nchunk, rows), rej_threads<T>(), 0, s, a,
                                   stats, nchunk, vec_ok)
                      : launch_pdl(stats_kernel<T>, dim3(nchunk, rows), kThreads, 0, s, a, stats, nchunk, vec_ok);
  if (e != cudaSuccess) return e;
  char* base = static_cast<char*>(a.workspace) + (((size_t)rows * nchunk * sizeof(ChunkStat) + 255) & ~(size_t)255);
  double* wsum = reinterpret_cast<double*>(base);
  int* jbuf = reinterpret_cast<int*>(base + (((size_t)a.B * nchunk * 2 * sizeof(double) + 255) & ~(size_t)255));
  // residual sums + inverse CDF: one cluster per sequence when the chunks fit
  // one cluster, else two launches through the workspace
  static int rs_limit[64];
  if (nchunk <= cluster_limit(resid_select_cluster_kernel<T>, rej_threads<T>(), rs_limit))
    return launch_cluster(resid_select_cluster_kernel<T>, nchunk, a.B, rej_threads<T>(), 0, s, a,
                          (const ChunkStat*)stats, nchunk, vec_ok);
  e = launch_pdl(residual_kernel<T>, dim3(nchunk, a.B), kThreads, 0, s, a, (const ChunkStat*)stats, nchunk, wsum, jbuf,
                 vec_ok);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel<T>, dim3(a.B), kThreads, 0, s, a, (const ChunkStat*)stats, nchunk,
                    (const double*)wsum, (const int*)jbuf);
}

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_verify_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_verify_trace, bytes);
}
#endif

size_t verify_workspace_bytes(int B, int k, int V, int mode) {
  const size_t nchunk = (V + kChunk - 1) / kChunk;
  const int n = k > 0 ? k : 1;
  if (mode != TIDAR_REJECTION)                      // greedy: the chunk statistics of the B n rows
    return (((size_t)B * n * nchunk * sizeof(ChunkStat) + 255) & ~(size_t)255);
  const size_t rows = (size_t)B * n + (size_t)B * (k > 1 ? k - 1 : 0);
  size_t bytes = ((rows * nchunk * sizeof(ChunkStat) + 255) & ~(size_t)255);
  bytes += (((size_t)B * nchunk * 2 * sizeof(double) + 255) & ~(size_t)255);
  bytes += (((size_t)B * sizeof(int) + 255) & ~(size_t)255);
  return bytes;
}

bool verify_grid_ok(int B, int k, int mode) {
  const long long n = k > 0 ? k : 1;
  // grid.y is one vocab row of the chunk statistics (rejection: also the q rows)
  const long long y = mode == TIDAR_REJECTION ? (long long)B * (2 * n - 1) : (long long)B * n;
  return y <= 65535;
}

cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t s) {
  return a.bf16 ? launch_t<__nv_bfloat16>(a, s) : launch_t<float>(a, s);
}

cudaError_t launch_greedy_stats(const VerifyArgs& a, cudaStream_t s) {
  return a.bf16 ? launch_greedy_stats_t<__nv_bfloat16>(a, s) : launch_greedy_stats_t<float>(a, s);
}

int verify_chunks(int V) { return (V + kChunk - 1) / kChunk; }


}  // namespace tidar

// ---------------------------------------------------------------------------
// tidar_verify_noalloc: the same verification without a caller workspace.
//
// For callers that cannot allocate device memory when they call verify: for
// example a decode loop being recorded into a CUDA graph, where an allocation
// would break the capture, or a host runtime that only hands the library
// tensors it already owns and has no way to create scratch buffers.  The
// scratch lives in this file's fixed device array instead; every GPU that
// loads the library keeps it until the process exits.
//
// The device address of the array is looked up (cudaGetSymbolAddress) on the
// first call made with each device current, under a mutex, so host threads
// that make their first calls at once are safe; that first call should still
// happen before any stream capture.  All calls share the one array and it
// keeps whatever the last call left there.  Verification needs no part of it
// zeroed: every statistic is written before it is read.  Calls that overlap on
// the GPU (different streams, no ordering between them) race on the array.
// CUDA failures return TIDAR_ERR_CUDA with the message recorded for
// tidar_last_cuda_error, as every other entry point does.
namespace tidar {
namespace {

constexpr size_t kNoAllocScratchBytes = TIDAR_VERIFY_NOALLOC_MAX_SCRATCH_BYTES;   // per device
static __device__ __align__(256) unsigned char g_verify_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void* g_verify_scratch_ptr[kNoAllocMaxDevices] = {nullptr};
std::mutex g_verify_scratch_mutex;

// Device address of this device's scratch array (looked up once per device).
tidar_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return TIDAR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_verify_scratch_mutex);
  if (!g_verify_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_verify_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    if (!ptr) return TIDAR_ERR_CUDA;
    g_verify_scratch_ptr[dev] = ptr;
  }
  *out = g_verify_scratch_ptr[dev];
  return TIDAR_OK;
}

}  // namespace
}  // namespace tidar

extern "C" tidar_status tidar_verify_noalloc(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                             tidar_accept_mode mode, const void* logits,
                                             const int32_t* drafts, const void* draft_logits,
                                             const float* uniforms, const int32_t* block_guesses,
                                             int32_t* accept_count, int32_t* out_tokens,
                                             int32_t* next_drafts, int32_t* selected_block,
                                             tidar_stream_t stream) {
  if (batch < 0 || k < 0 || vocab <= 0) return TIDAR_ERR_INVALID_ARG;
  if (k > 16) return TIDAR_ERR_UNSUPPORTED;
  if (dtype != TIDAR_F32 && dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (mode != TIDAR_GREEDY && mode != TIDAR_REJECTION) return TIDAR_ERR_INVALID_ARG;
  if (batch == 0) return TIDAR_OK;
  if (!logits || !accept_count || !out_tokens) return TIDAR_ERR_INVALID_ARG;
  if (k > 1 && !drafts) return TIDAR_ERR_INVALID_ARG;
  if (mode == TIDAR_REJECTION && (!uniforms || (k > 1 && !draft_logits))) return TIDAR_ERR_INVALID_ARG;
  if (!tidar::verify_grid_ok(batch, k, mode)) return TIDAR_ERR_UNSUPPORTED;
  // too large for the fixed scratch: refuse before touching the device
  if (tidar::verify_workspace_bytes(batch, k, vocab, mode) > tidar::kNoAllocScratchBytes)
    return TIDAR_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  tidar_status st = tidar::scratch_address(&scratch);
  if (st != TIDAR_OK) return st;
  tidar::VerifyArgs a{};
  a.B = batch; a.k = k; a.n = k > 0 ? k : 1; a.V = vocab; a.bf16 = dtype == TIDAR_BF16; a.mode = mode;
  a.logits = logits; a.drafts = drafts; a.draft_logits = draft_logits; a.uniforms = uniforms;
  a.block_guesses = block_guesses; a.accept_count = accept_count; a.out_tokens = out_tokens;
  a.next_drafts = next_drafts; a.selected_block = selected_block;
  a.workspace = scratch;
  if ((st = tidar::error_word_status(&a.err)) != TIDAR_OK) return st;
  const cudaError_t e = tidar::launch_verify(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return tidar::cuda_status(e);
  return TIDAR_OK;
}
