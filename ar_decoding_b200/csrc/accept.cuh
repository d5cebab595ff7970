// accept.cuh -- greedy acceptance of one sequence by one warp, from the
// per-chunk (max, argmax) statistics of its logits rows.  Shared by the
// acceptance kernel of tidar_verify and the commit kernel of
// tidar_verify_commit.
//
// "Talk in Autoregression": the carried drafts are scored strictly left to
// right (nodesdaily.com (fr), paragraph on betting on every outcome): d_{i+1}
// is kept while it equals argmax l_i, so j = the first mismatching i, else n,
// and t* = argmax l_{j-1}; block j of the pre-drafted guesses is selected
// (mauroscia.it section 2).
#pragma once

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace tidar {

__device__ __forceinline__ void amax_merge_acc(float& v, int& i, float v2, int i2) {
  if (v2 > v || (v2 == v && i2 < i)) { v = v2; i = i2; }
}

// The whole warp runs it for sequence b (n <= 32 rows, k <= 16): lane i merges
// the chunk statistics of row i in chunk order.  The drafts and all block
// guesses are fetched first (they do not depend on the statistics); s_g is
// this warp's 256-int scratch.  With `write` the verification outputs are
// stored.  Returns j (warp-uniform).
__device__ __forceinline__ int greedy_accept_warp(const GreedyAcceptArgs& f, int n, int k, int b, int* s_g,
                                                  bool write) {
  const int lane = threadIdx.x & 31;
  constexpr unsigned kAll = 0xffffffffu;
  const bool want_g = write && f.next_drafts && f.block_guesses && k > 0;
  const int d = (lane >= 1 && lane < n && k > 1) ? f.drafts[(size_t)b * k + lane] : -1;
  if (want_g)
    for (int t = lane; t < k * k; t += 32) s_g[t] = f.block_guesses[(size_t)b * k * k + t];
  float mv = -INFINITY;
  int am = INT_MAX;
  if (lane < n) {
    // eight chunks' statistics in flight at a time, merged in chunk order
    const ChunkStat* st = f.stats + ((size_t)b * n + lane) * f.nchunk;
    for (int c0 = 0; c0 < f.nchunk; c0 += 8) {
      float v8[8];
      int i8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        v8[u] = -INFINITY;
        i8[u] = INT_MAX;
        if (c0 + u < f.nchunk) { v8[u] = st[c0 + u].max; i8[u] = st[c0 + u].arg; }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) amax_merge_acc(mv, am, v8[u], i8[u]);
    }
  }
  __syncwarp();
  const int am_prev = __shfl_up_sync(kAll, am, 1);            // argmax l_{lane-1}
  const bool mism = lane >= 1 && lane < n && d != am_prev;
  const unsigned bal = __ballot_sync(kAll, mism);
  const int j = bal ? __ffs(bal) - 1 : n;
  const int t_star = __shfl_sync(kAll, am, j - 1);
  const int d_next = __shfl_down_sync(kAll, d, 1);            // d_{lane+1}
  if (write) {
    if (lane < n) f.out_tokens[(size_t)b * n + lane] = lane < j - 1 ? d_next : (lane == j - 1 ? t_star : -1);
    if (f.next_drafts && k > 0 && lane < k)
      f.next_drafts[(size_t)b * k + lane] = lane == 0 ? t_star : (want_g ? s_g[(j - 1) * k + lane] : -1);
    if (lane == 0) {
      f.accept_count[b] = j;
      if (f.selected_block) f.selected_block[b] = k > 0 ? j : 0;
    }
  }
  return j;
}

// Writes accept_count, out_tokens, selected_block, next_drafts for sequence b.
// Called by a whole warp (n, k <= 16): every lane loads its draft and its
// block guess first, all in flight at once, then the lanes store (one thread
// storing as it loads would wait a memory round trip per element, the loads
// not being movable past stores that might alias).
__device__ __forceinline__ void write_outputs_warp(const VerifyArgs& a, int b, int j, int t_star) {
  const int e = (int)threadIdx.x & 31;
  int v = -1, gv = -1;
  if (e < a.n) {
    if (e < j - 1) v = a.drafts[(size_t)b * a.k + e + 1];
    else if (e == j - 1) v = t_star;
  }
  const bool nd = a.next_drafts && a.k > 0;
  if (nd && e >= 1 && e < a.k && a.block_guesses) gv = a.block_guesses[((size_t)b * a.k + (j - 1)) * a.k + e];
  __syncwarp();
  if (e < a.n) a.out_tokens[(size_t)b * a.n + e] = v;
  if (nd && e < a.k) a.next_drafts[(size_t)b * a.k + e] = e == 0 ? t_star : gv;
  if (e == 0) {
    a.accept_count[b] = j;
    if (a.selected_block) a.selected_block[b] = a.k > 0 ? j : 0;
  }
}

}  // namespace tidar
