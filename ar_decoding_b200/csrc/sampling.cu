// sampling.cu -- verification and draft sampling under a sampling transform
// (temperature, nucleus truncation), sm_100a.
//
// The speculative-sampling rule keeps the AR law exact for any pair of
// distributions p (AR) and q (drafts) ("TiDAR: Think in Diffusion, Talk in
// Autoregression", mauroscia.it: the speculative-decoding lineage, Leviathan et
// al. and Chen et al.; engineer-news.pages.dev, section "TiDAR 在做什麼": the
// output equals AR sampling), so sampling controls apply to both alike.  The
// pages fix none; this library takes the usual ones:
//   temperature T > 0:  p(x) proportional to exp(l(x) / T);
//   nucleus top_p:      tokens ordered larger logit first, lower index first on
//                       equal logits; token x is kept iff the probability of the
//                       tokens before it is below top_p; the kept tokens are
//                       renormalised.  top_p >= 1 keeps every token.
// The next drafts come from the selected mask block's slot distributions under
// the same transform (mauroscia.it section 2: the mask slots' predictions are
// the drafts; nodesdaily.com (fr), paragraph on betting on every outcome).
//
// Kernels:
//   dist_kernel      one CTA per distribution row: the row maximum of l / T,
//                    the fp64 normaliser, and -- with truncation -- the exact
//                    nucleus cut: an MSB-first radix select (four 8-bit digits)
//                    of the order key of the logits, each digit's histogram
//                    weighted by the fp64 mass exp(l/T - max), then an
//                    index-order scan of the tie group at the cut key.  Writes
//                    a RowDist (max, 1 / kept mass, cut key, cut index).
//   accept_kernel    one CTA per sequence: the accept scan in fp64 from the row
//                    descriptors, then t* by the inverse CDF of the residual
//                    max(0, p_j - q_j) (or p_j) in index order: per-thread
//                    contiguous chunks, a block scan of the chunk sums, the
//                    crossing chunk scanned in order.
//   draft_kernel     one CTA per (sequence, slot 2..k) of the selected block:
//                    the slot row's RowDist and its inverse CDF (or argmax).
// Rows are vocab-sized and read a few times from L2; this is latency-bound
// work, not a contraction.
#include <climits>
#include <math.h>

#include "accept.cuh"
#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

constexpr int kSThreads = 512;
constexpr int kSWarps = kSThreads / 32;

struct RowDist {
  double M;          // max over the row of l / T
  double inv_S;      // 1 / (sum of exp(l/T - M) over the kept tokens)
  uint32_t key_cut;  // kept iff key > key_cut, or key == key_cut and index <= idx_cut
  int idx_cut;
};

template <typename T>
__device__ __forceinline__ float ld_logit(const T* p, int i) { return to_f32(p[i]); }

// Order-preserving key of a finite logit (larger logit, larger key); -0 and +0
// are the same logit.
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x == 0.0f) x = 0.0f;
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ bool is_kept(const RowDist& d, uint32_t key, int x) {
  return key > d.key_cut || (key == d.key_cut && x <= d.idx_cut);
}
// Probability of token x under the transformed distribution of its row.
__device__ __forceinline__ double prob(const RowDist& d, float l, int x, double T) {
  return is_kept(d, order_key(l), x) ? exp((double)l / T - d.M) * d.inv_S : 0.0;
}

struct SScratch {
  double red[kSWarps];
  float redf[kSWarps];
  int redi[kSWarps];
  double hist[256];
  double chunk[kSThreads];   // per-thread chunk sums, then their exclusive prefix
  double bcast[4];
  int ibcast[4];
};

__device__ __forceinline__ double block_sum(double v, SScratch& s) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) s.red[w] = v;
  __syncthreads();
  double t = 0.0;
  for (int i = 0; i < kSWarps; ++i) t += s.red[i];     // the same order in every thread
  return t;
}
__device__ __forceinline__ float block_max(float v, SScratch& s) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) s.redf[w] = v;
  __syncthreads();
  float t = -INFINITY;
  for (int i = 0; i < kSWarps; ++i) t = fmaxf(t, s.redf[i]);
  return t;
}
// Exclusive prefix of one double per thread, in thread order (s.chunk).
__device__ __forceinline__ double block_exclusive_scan(double v, SScratch& s) {
  __syncthreads();
  s.chunk[threadIdx.x] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    // warp 0: lane l sums threads [16 l, 16 l + 16), scans the lanes, writes back
    const int per = kSThreads / 32;
    double loc = 0.0;
    for (int i = 0; i < per; ++i) loc += s.chunk[threadIdx.x * per + i];
    double inc = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, inc, o);
      if ((int)threadIdx.x >= o) inc += y;
    }
    double run = inc - loc;
    for (int i = 0; i < per; ++i) {
      const double c = s.chunk[threadIdx.x * per + i];
      s.chunk[threadIdx.x * per + i] = run;
      run += c;
    }
  }
  __syncthreads();
  return s.chunk[threadIdx.x];
}

// The transformed distribution's descriptor of one row (every thread of the CTA
// calls it and gets the result).
template <typename T>
__device__ RowDist row_dist(const T* row, int V, double temp, double top_p, SScratch& s) {
  float mx = -INFINITY;
  for (int x = threadIdx.x; x < V; x += kSThreads) mx = fmaxf(mx, ld_logit(row, x));
  mx = block_max(mx, s);
  RowDist d;
  d.M = (double)mx / temp;
  double z = 0.0;
  for (int x = threadIdx.x; x < V; x += kSThreads) z += exp((double)ld_logit(row, x) / temp - d.M);
  const double Z = block_sum(z, s);
  if (!(top_p < 1.0)) {
    d.inv_S = 1.0 / Z;
    d.key_cut = 0u;
    d.idx_cut = INT_MAX;
    return d;
  }
  const double tau = top_p * Z;
  // the cut key: the largest key whose tokens of key >= it reach tau
  uint32_t prefix = 0u;
  double above = 0.0;                                   // mass of keys above the prefix range
  for (int level = 0; level < 4; ++level) {
    const int shift = 24 - 8 * level;
    __syncthreads();
    if (threadIdx.x < 256) s.hist[threadIdx.x] = 0.0;
    __syncthreads();
    for (int x = threadIdx.x; x < V; x += kSThreads) {
      const float l = ld_logit(row, x);
      const uint32_t key = order_key(l);
      if (level == 0 || (key >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&s.hist[(key >> shift) & 255u], exp((double)l / temp - d.M));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l holds bins [8 l, 8 l + 8); suffix sums from bin 255 down
      const int lane = threadIdx.x;
      double loc = 0.0;
      for (int i = 0; i < 8; ++i) loc += s.hist[8 * lane + i];
      double suf = loc;                                 // inclusive suffix over lanes >= lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += y;
      }
      const double beyond = suf - loc;                  // bins above this lane's range
      // the digit: the largest bin b with above + sum_{bins >= b} >= tau
      int digit = -1;
      double run = above + beyond;
      double above_digit = 0.0;
      for (int i = 7; i >= 0; --i) {
        const double h = s.hist[8 * lane + i];
        if (run + h >= tau) { digit = 8 * lane + i; above_digit = run; break; }
        run += h;
      }
      const unsigned has = __ballot_sync(0xffffffffu, digit >= 0);
      const int src = has ? 31 - __clz(has) : 0;        // the highest lane that found one
      const int dsel = __shfl_sync(0xffffffffu, digit, src);
      const double asel = __shfl_sync(0xffffffffu, above_digit, src);
      if (lane == 0) {
        s.ibcast[0] = has ? dsel : 0;
        s.bcast[0] = has ? asel : above;
      }
    }
    __syncthreads();
    prefix |= (uint32_t)s.ibcast[0] << shift;
    above = s.bcast[0];
  }
  d.key_cut = prefix;
  // the tie group at the cut key, in index order: thread t owns the contiguous
  // chunk [t c, t c + c); kept while above + mass before the token < tau
  const int ch = (V + kSThreads - 1) / kSThreads;
  const int x0 = threadIdx.x * ch, x1 = min(V, x0 + ch);
  double own = 0.0;
  for (int x = x0; x < x1; ++x) {
    const float l = ld_logit(row, x);
    if (order_key(l) == prefix) own += exp((double)l / temp - d.M);
  }
  const double before = block_exclusive_scan(own, s);
  int last = -1;
  double kept_group = 0.0;
  {
    double c = above + before;
    for (int x = x0; x < x1; ++x) {
      const float l = ld_logit(row, x);
      if (order_key(l) != prefix) continue;
      if (c < tau) {
        last = x;
        const double e = exp((double)l / temp - d.M);
        c += e;
        kept_group += e;
      } else {
        break;
      }
    }
  }
  // idx_cut = the largest kept index of the group; kept mass = above + group's
  __syncthreads();
  if (threadIdx.x < kSWarps) s.redi[threadIdx.x] = -1;
  __syncthreads();
  int lm = last;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) lm = max(lm, __shfl_xor_sync(0xffffffffu, lm, o));
  if ((threadIdx.x & 31) == 0) s.redi[threadIdx.x >> 5] = lm;
  const double kg = block_sum(kept_group, s);           // (synchronises: redi is complete)
  int cut = -1;
  for (int i = 0; i < kSWarps; ++i) cut = max(cut, s.redi[i]);
  d.idx_cut = cut;
  d.inv_S = 1.0 / (above + kg);
  return d;
}

// Inverse CDF over the weights w(x), x in index order: the smallest t with
// u * sum(w) < sum_{y <= t} w(y) (V - 1 if rounding leaves none).  Every thread
// of the CTA calls it; wfn(x) gives w(x).
template <typename W>
__device__ int inverse_cdf(int V, double u, W wfn, SScratch& s, double* total_out) {
  const int ch = (V + kSThreads - 1) / kSThreads;
  const int x0 = threadIdx.x * ch, x1 = min(V, x0 + ch);
  double own = 0.0;
  for (int x = x0; x < x1; ++x) own += wfn(x);
  const double before = block_exclusive_scan(own, s);
  const double total = block_sum(own, s);
  if (total_out) *total_out = total;
  const double target = u * total;
  __syncthreads();
  if (threadIdx.x == 0) s.ibcast[1] = INT_MAX;
  __syncthreads();
  if (target >= before) {
    double c = before;
    for (int x = x0; x < x1; ++x) {
      c += wfn(x);
      if (target < c) { atomicMin(&s.ibcast[1], x); break; }
    }
  }
  __syncthreads();
  const int t = s.ibcast[1];
  return t == INT_MAX ? V - 1 : t;
}

// Lowest index of the row maximum (exact on the stored values).
template <typename T>
__device__ int row_argmax(const T* row, int V, SScratch& s) {
  float bv = -INFINITY;
  int bi = INT_MAX;
  for (int x = threadIdx.x; x < V; x += kSThreads) {
    const float v = ld_logit(row, x);
    if (v > bv || bi == INT_MAX) { bv = v; bi = x; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(0xffffffffu, bv, o);
    const int i2 = __shfl_xor_sync(0xffffffffu, bi, o);
    if (v2 > bv || (v2 == bv && i2 < bi)) { bv = v2; bi = i2; }
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) { s.redf[threadIdx.x >> 5] = bv; s.redi[threadIdx.x >> 5] = bi; }
  __syncthreads();
  float fv = s.redf[0];
  int fi = s.redi[0];
  for (int i = 1; i < kSWarps; ++i)
    if (s.redf[i] > fv || (s.redf[i] == fv && s.redi[i] < fi)) { fv = s.redf[i]; fi = s.redi[i]; }
  return fi;
}

struct SampledArgs {
  VerifyArgs v;
  double temp, top_p;
  RowDist* dist;      // [B][n + k - 1]: p rows, then q rows
};

// Row r of sequence b's distributions: r < n -> logits row r (p_{r+1});
// else draft row r - n (q_{r-n+1}).
template <typename T>
__device__ __forceinline__ const T* dist_row_ptr(const VerifyArgs& a, int b, int r) {
  if (r < a.n) return static_cast<const T*>(a.logits) + ((size_t)b * a.n + r) * a.V;
  const int i = r - a.n + 1;                           // q_i
  const T* base = static_cast<const T*>(a.draft_logits);
  if (!a.draft_block) return base + ((size_t)b * (a.k - 1) + (i - 1)) * a.V;
  int j = a.draft_block[b];
  if (j < 1 || j > a.k) j = 1;
  return base + (((size_t)b * a.k + (j - 1)) * a.k + i) * a.V;
}

template <typename T>
__global__ void __launch_bounds__(kSThreads) dist_kernel(SampledArgs sa) {
  __shared__ SScratch s;
  pdl_wait();
  pdl_trigger();
  const VerifyArgs& a = sa.v;
  const int rows = a.n + a.k - 1 > a.n ? a.n + a.k - 1 : a.n;
  const int b = blockIdx.y, r = blockIdx.x;
  if (r >= rows) return;
  if (threadIdx.x == 0 && r >= a.n && a.draft_block) {
    const int j = a.draft_block[b];
    if (j < 1 || j > a.k) raise_error(a.err, TIDAR_DEVERR_BAD_COUNT);
  }
  const RowDist d = row_dist(dist_row_ptr<T>(a, b, r), a.V, sa.temp, sa.top_p, s);
  if (threadIdx.x == 0) sa.dist[(size_t)b * rows + r] = d;
}

template <typename T>
__global__ void __launch_bounds__(kSThreads) accept_kernel(SampledArgs sa) {
  __shared__ SScratch s;
  __shared__ int s_j;
  pdl_wait();
  pdl_trigger();
  const VerifyArgs& a = sa.v;
  const int b = blockIdx.x;
  const int rows = a.n + a.k - 1 > a.n ? a.n + a.k - 1 : a.n;
  const RowDist* dd = sa.dist + (size_t)b * rows;
  if (threadIdx.x < 32) {
    // accept scan: the n-1 tests are independent (only "stop at the first
    // rejection" orders them), so lane i-1 evaluates test i in fp64 and a
    // ballot finds the first failure: j = that i, else n
    const int i = (int)threadIdx.x + 1;
    bool fail = false;
    if (i <= a.n - 1) {
      const int d = a.drafts[(size_t)b * a.k + i];
      fail = true;
      if (d >= 0 && d < a.V) {
        const double u = (double)a.uniforms[(size_t)b * a.n + (i - 1)];
        const float lp = ld_logit(dist_row_ptr<T>(a, b, i - 1), d);
        const float lq = ld_logit(dist_row_ptr<T>(a, b, a.n + i - 1), d);
        const double p = prob(dd[i - 1], lp, d, sa.temp), q = prob(dd[a.n + i - 1], lq, d, sa.temp);
        fail = !(u * q < p);
      }
    }
    const unsigned bal = __ballot_sync(0xffffffffu, fail);
    if (threadIdx.x == 0) s_j = bal ? __ffs(bal) : a.n;
  }
  __syncthreads();
  const int j = s_j;
  const T* prow = dist_row_ptr<T>(a, b, j - 1);
  const RowDist dp = dd[j - 1];
  const double u = (double)a.uniforms[(size_t)b * a.n + (a.n - 1)];
  int t_star;
  if (j < a.n) {
    const T* qrow = dist_row_ptr<T>(a, b, a.n + j - 1);
    const RowDist dq = dd[a.n + j - 1];
    double total = 0.0;
    auto resid = [&](int x) -> double {
      const double r = prob(dp, ld_logit(prow, x), x, sa.temp) - prob(dq, ld_logit(qrow, x), x, sa.temp);
      return r > 0.0 ? r : 0.0;
    };
    t_star = inverse_cdf(a.V, u, resid, s, &total);
    if (!(total > 0.0))                                 // residual all zero (rounding): p_j
      t_star = inverse_cdf(a.V, u, [&](int x) { return prob(dp, ld_logit(prow, x), x, sa.temp); }, s, nullptr);
  } else {
    t_star = inverse_cdf(a.V, u, [&](int x) { return prob(dp, ld_logit(prow, x), x, sa.temp); }, s, nullptr);
  }
  if (threadIdx.x < 32) write_outputs_warp(a, b, j, t_star);
}

struct DraftArgs {
  int B, k, V, mode;
  double temp, top_p;
  const void* block_logits;      // [B][k][k][V]
  const int32_t* selected_block;
  const float* uniforms;         // [B][k]
  int32_t* next_drafts;          // [B][k]
  unsigned int* err;
};

template <typename T>
__global__ void __launch_bounds__(kSThreads) draft_kernel(DraftArgs da) {
  __shared__ SScratch s;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y, slot = blockIdx.x + 2;     // slots 2..k
  int j = da.selected_block[b];
  if (j < 1 || j > da.k) {
    if (threadIdx.x == 0 && slot == 2) raise_error(da.err, TIDAR_DEVERR_BAD_COUNT);
    j = 1;
  }
  const T* row = static_cast<const T*>(da.block_logits) + (((size_t)b * da.k + (j - 1)) * da.k + (slot - 1)) * da.V;
  int tok;
  if (da.mode == TIDAR_GREEDY) {
    tok = row_argmax(row, da.V, s);
  } else {
    const RowDist d = row_dist(row, da.V, da.temp, da.top_p, s);
    const double u = (double)da.uniforms[(size_t)b * da.k + (slot - 1)];
    tok = inverse_cdf(da.V, u, [&](int x) { return prob(d, ld_logit(row, x), x, da.temp); }, s, nullptr);
  }
  if (threadIdx.x == 0) da.next_drafts[(size_t)b * da.k + (slot - 1)] = tok;
}

}  // namespace

size_t sampled_verify_workspace_bytes(int B, int k) {
  const int n = k > 0 ? k : 1;
  const int rows = n + (k > 1 ? k - 1 : 0);
  return (size_t)B * rows * sizeof(RowDist);
}

cudaError_t launch_sampled_verify(const VerifyArgs& a, double temp, double top_p, cudaStream_t st) {
  SampledArgs sa;
  sa.v = a;
  sa.temp = temp;
  sa.top_p = top_p;
  sa.dist = static_cast<RowDist*>(a.workspace);
  const int rows = a.n + (a.k > 1 ? a.k - 1 : 0);
  const dim3 g1(rows, a.B);
  cudaError_t e = a.bf16 ? launch_pdl(dist_kernel<__nv_bfloat16>, g1, kSThreads, 0, st, sa)
                         : launch_pdl(dist_kernel<float>, g1, kSThreads, 0, st, sa);
  if (e != cudaSuccess) return e;
  return a.bf16 ? launch_pdl(accept_kernel<__nv_bfloat16>, dim3(a.B), kSThreads, 0, st, sa)
                : launch_pdl(accept_kernel<float>, dim3(a.B), kSThreads, 0, st, sa);
}

cudaError_t launch_sample_drafts(int B, int k, int V, int bf16, int mode, double temp, double top_p,
                                 const void* block_logits, const int32_t* selected_block,
                                 const float* uniforms, int32_t* next_drafts, unsigned int* err,
                                 cudaStream_t st) {
  if (k < 2 || B == 0) return cudaSuccess;
  DraftArgs da;
  da.B = B; da.k = k; da.V = V; da.mode = mode; da.temp = temp; da.top_p = top_p;
  da.block_logits = block_logits; da.selected_block = selected_block; da.uniforms = uniforms;
  da.next_drafts = next_drafts; da.err = err;
  const dim3 g(k - 1, B);
  return bf16 ? launch_pdl(draft_kernel<__nv_bfloat16>, g, kSThreads, 0, st, da)
              : launch_pdl(draft_kernel<float>, g, kSThreads, 0, st, da);
}

}  // namespace tidar
