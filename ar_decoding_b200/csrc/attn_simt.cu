// attn_simt.cu -- CUDA-core step attention, split-KV merge and draft-row append.
//
// The step attention of one TiDAR decode step ("TiDAR: Think in Diffusion,
// Talk in Autoregression", mauroscia.it, section 2 "Single Forward Pass &
// Structured Attention Mask"; nodesdaily.com (fr), paragraphs on the three
// zones and on the masking puzzle): every query row attends the whole cached
// prefix plus the step keys its zone may see.
//
// This is the fp32 path (the tiny workload needs 1e-5 agreement, so no tf32
// tensor cores) and the general fallback for shapes the tensor-core kernel
// does not take.  One warp owns one packed query row (b, rho, h); lanes split
// the head dimension; keys are visited in order with an online softmax in
// fp32 (accurate expf).  Split-KV: blockIdx.y selects a contiguous key range;
// the last split also takes the step keys.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

constexpr int kWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int VPL = D / 32;  // elements per lane
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int bg = blockIdx.z;
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int M = a.R * a.G;
  const int m = blockIdx.x * kWarps + warp;
  if (m >= M) return;
  const int rho = m / a.G, h = g * a.G + m % a.G;
  const int split = blockIdx.y;

  int P = a.seq_lens[b];
  if (P < 0 || P > a.max_prefix) {
    if (lane == 0 && split == 0 && m == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    P = 0;
  }

  const T* qp = static_cast<const T*>(a.q) + ((size_t)(b * a.R + rho) * a.Hq + h) * D + lane * VPL;
  float qv[VPL];
  load_vec<T, VPL>(qp, qv);
#pragma unroll
  for (int i = 0; i < VPL; ++i) qv[i] *= a.scale;

  float mx = -INFINITY, l = 0.f, acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;

  // Online-softmax update with a batch of up to kKB keys whose K and V slices
  // are in registers (ok[u]: key u exists): all the batch's dot products and
  // warp sums first, then one rescale of (l, acc) by the batch's new maximum.
  constexpr int kKB = 8;
  auto update = [&](const float (&kv)[kKB][VPL], const float (&vv)[kKB][VPL], const bool (&ok)[kKB]) {
    float sc[kKB];
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) dot = fmaf(qv[i], kv[u][i], dot);
      sc[u] = dot;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < kKB; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
    float mn = mx;
#pragma unroll
    for (int u = 0; u < kKB; ++u)
      if (ok[u]) mn = fmaxf(mn, sc[u]);
    if (mn == -INFINITY) return;                    // no key in the batch (and none before)
    const float corr = expf(mx - mn);               // 0 while mx = -inf
    float ps = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] *= corr;
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      if (!ok[u]) continue;                          // its K/V registers were never loaded
      const float pe = expf(sc[u] - mn);
      ps += pe;
#pragma unroll
      for (int i = 0; i < VPL; ++i) acc[i] = fmaf(pe, vv[u][i], acc[i]);
    }
    l = fmaf(l, corr, ps);
    mx = mn;
  };
  // Keys go in batches of kKB: the K and V slices of a batch are all loaded
  // before the first is used (one memory round trip per batch, not two per
  // key).

  // prefix keys of this split
  const int k0 = split * a.keys_per_split;
  const int k1 = min(P, k0 + a.keys_per_split);
  const T* kpages = static_cast<const T*>(a.k_pages);
  const T* vpages = static_cast<const T*>(a.v_pages);
  const int32_t* table = a.page_table + (size_t)b * a.max_pages;
  bool bad_page = false;
  for (int key0 = k0; key0 < k1; key0 += kKB) {
    float kv[kKB][VPL], vv[kKB][VPL];
    bool ok[kKB];
#pragma unroll
    for (int u = 0; u < kKB; ++u) {
      const int key = key0 + u;
      ok[u] = false;
      if (key < k1) {
        const int page = table[key / a.page_size];
        if (page < 0 || page >= a.num_pages) {
          bad_page = true;
        } else {
          const size_t off = ((size_t)(page * a.Hkv + g) * a.page_size + key % a.page_size) * D + lane * VPL;
          load_vec<T, VPL>(kpages + off, kv[u]);
          load_vec<T, VPL>(vpages + off, vv[u]);
          ok[u] = true;
        }
      }
    }
    update(kv, vv, ok);
  }
  if (bad_page && lane == 0) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);

  // step keys (drafts and mask slots), last split only
  if (split == a.nsplit - 1 && a.step_keys) {
    const StepVis vis = step_visibility(a.k, rho);
    const T* kb = static_cast<const T*>(a.k_blk);
    const T* vb = static_cast<const T*>(a.v_blk);
    for (int key0 = 0; key0 < a.R; key0 += kKB) {
      float kv[kKB][VPL], vv[kKB][VPL];
      bool ok[kKB];
#pragma unroll
      for (int u = 0; u < kKB; ++u) {
        const int key = key0 + u;
        ok[u] = key < a.R && step_visible(vis, key);
        if (ok[u]) {
          const size_t off = ((size_t)(b * a.R + key) * a.Hkv + g) * D + lane * VPL;
          load_vec<T, VPL>(kb + off, kv[u]);
          load_vec<T, VPL>(vb + off, vv[u]);
        }
      }
      update(kv, vv, ok);
    }
  }

  const float inv = l > 0.f ? 1.f / l : 0.f;
  float o[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) o[i] = acc[i] * inv;
  const size_t row = (size_t)(b * a.R + rho) * a.Hq + h;
  const float lse = l > 0.f ? mx + logf(l) : -INFINITY;
  if (a.nsplit == 1) {
    store_vec<T, VPL>(static_cast<T*>(a.out) + row * D + lane * VPL, o);
    if (a.lse_out && lane == 0) a.lse_out[row] = lse;
  } else {
    const size_t prow = (size_t)split * a.B * a.R * a.Hq + row;
    store_vec<float, VPL>(a.part_o + prow * D + lane * VPL, o);
    if (lane == 0) a.part_lse[prow] = lse;
  }
}

// Merge the split partials (weights exp(lse_s - max)) and, in the blocks past
// the merge, copy the draft rows' K/V into the cache at P_b .. P_b+n-1.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) finalize_kernel(AttnArgs a, int merge_blocks) {
  pdl_wait();
  pdl_trigger();
  constexpr int VPL = D / 32;
  if ((int)blockIdx.x < merge_blocks) {
    // one warp per output row.  The split weights are computed lane-parallel
    // (lane s holds splits s and s + 32; at most 64 splits).  The partial rows
    // of up to kFinChunk splits are loaded in the same round trip as the lse
    // values -- unconditionally, since an empty split's row may be unwritten,
    // and then selected away rather than multiplied by its zero weight.
    constexpr int kFinChunk = 16;
    const int lane = threadIdx.x & 31;
    const size_t rows = (size_t)a.B * a.R * a.Hq;
    const size_t row = (size_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int ns = a.nsplit;
    const float la = lane < ns ? a.part_lse[lane * rows + row] : -INFINITY;
    const float lb = lane + 32 < ns ? a.part_lse[(lane + 32) * rows + row] : -INFINITY;
    float acc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
    float wa = 0.f, wb = 0.f, mx = -INFINITY, wsum = 0.f;
    for (int s0 = 0; s0 < ns; s0 += kFinChunk) {
      float v[kFinChunk][VPL];
#pragma unroll
      for (int u = 0; u < kFinChunk; ++u) {
        if (s0 + u < ns) load_vec<float, VPL>(a.part_o + ((s0 + u) * rows + row) * D + lane * VPL, v[u]);
      }
      if (s0 == 0) {
        mx = fmaxf(la, lb);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        wa = la == -INFINITY ? 0.f : expf(la - mx);
        wb = lb == -INFINITY ? 0.f : expf(lb - mx);
        wsum = wa + wb;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
      }
#pragma unroll
      for (int u = 0; u < kFinChunk; ++u) {
        const int sp = s0 + u;
        const float w = __shfl_sync(0xffffffffu, sp < 32 ? wa : wb, sp & 31);
        if (sp < ns && w > 0.f) {
#pragma unroll
          for (int i = 0; i < VPL; ++i) acc[i] = fmaf(w, v[u][i], acc[i]);
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] *= inv;
    store_vec<T, VPL>(static_cast<T*>(a.out) + row * D + lane * VPL, acc);
    if (a.lse_out && lane == 0) a.lse_out[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
    return;
  }
  // draft-row append: one block per (b, r)
  const int idx = blockIdx.x - merge_blocks;
  const int b = idx / a.n, r = idx % a.n;
  const int P = a.seq_lens[b];
  if (P < 0 || P > a.max_prefix) return;   // reported by the attention kernel
  const int pos = P + r;
  const int page = a.page_table[(size_t)b * a.max_pages + pos / a.page_size];
  if (page < 0 || page >= a.num_pages) {
    if (threadIdx.x == 0) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
    return;
  }
  constexpr int kVec = 16 / sizeof(T);     // elements per 16-byte chunk
  const int chunks = a.Hkv * D / kVec;     // per K (and per V) row
  for (int c = threadIdx.x; c < 2 * chunks; c += blockDim.x) {
    const int which = c / chunks, cc = c % chunks;
    const int g = cc / (D / kVec), e = (cc % (D / kVec)) * kVec;
    const T* src = static_cast<const T*>(which ? a.v_blk : a.k_blk) +
                   ((size_t)(b * a.R + r) * a.Hkv + g) * D + e;
    T* dst = static_cast<T*>(const_cast<void*>(which ? a.v_pages : a.k_pages)) +
             ((size_t)(page * a.Hkv + g) * a.page_size + pos % a.page_size) * D + e;
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  }
}

// Log-sum-exp merge of nparts attention results over disjoint key sets (one
// warp per row): O = sum_r w_r O_r / sum_r w_r with w_r = exp(lse_r - max);
// lse = max + log(sum_r w_r).  A part with lse = -inf (no key) gets no weight
// and its row is not read.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) merge_parts_kernel(int nparts, long long rows, const T* part_o,
                                                                  const float* part_lse, T* out, float* lse_out) {
  pdl_wait();
  pdl_trigger();
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float la = lane < nparts ? part_lse[(size_t)lane * rows + row] : -INFINITY;
  const float lb = lane + 32 < nparts ? part_lse[(size_t)(lane + 32) * rows + row] : -INFINITY;
  float mx = fmaxf(la, lb);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float wa = la == -INFINITY ? 0.f : expf(la - mx);
  const float wb = lb == -INFINITY ? 0.f : expf(lb - mx);
  float wsum = wa + wb;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  for (int r = 0; r < nparts; ++r) {
    const float w = __shfl_sync(0xffffffffu, r < 32 ? wa : wb, r & 31);
    if (w == 0.f) continue;
    float v[VPL];
    load_vec<T, VPL>(part_o + ((size_t)r * rows + row) * D + lane * VPL, v);
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = fmaf(w, v[i], acc[i]);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] *= inv;
  store_vec<T, VPL>(out + (size_t)row * D + lane * VPL, acc);
  if (lse_out && lane == 0) lse_out[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_merge_t(int nparts, long long rows, const void* part_o, const float* part_lse, void* out,
                           float* lse_out, cudaStream_t s) {
  const long long blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  return launch_pdl(merge_parts_kernel<T, D>, dim3((unsigned)blocks), kWarps * 32, 0, s, nparts, rows,
                    static_cast<const T*>(part_o), part_lse, static_cast<T*>(out), lse_out);
}

template <typename T, int D>
cudaError_t launch_simt_t(const AttnArgs& a, cudaStream_t s) {
  const int M = a.R * a.G;
  dim3 grid((M + kWarps - 1) / kWarps, a.nsplit, a.B * a.Hkv);
  return launch_pdl(attn_simt_kernel<T, D>, grid, kWarps * 32, 0, s, a);
}

template <typename T, int D>
cudaError_t launch_finalize_t(const AttnArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.B * a.R * a.Hq;
  const int merge_blocks = a.nsplit > 1 ? (int)((rows + kWarps - 1) / kWarps) : 0;
  const int blocks = merge_blocks + (a.append ? a.B * a.n : 0);
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(finalize_kernel<T, D>, dim3(blocks), kWarps * 32, 0, s, a, merge_blocks);
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s) {
  if (a.bf16) return a.D == 64 ? launch_simt_t<__nv_bfloat16, 64>(a, s) : launch_simt_t<__nv_bfloat16, 128>(a, s);
  return a.D == 64 ? launch_simt_t<float, 64>(a, s) : launch_simt_t<float, 128>(a, s);
}

cudaError_t launch_merge_parts(int nparts, long long rows, int D, int bf16, const void* part_o,
                               const float* part_lse, void* out, float* lse_out, cudaStream_t s) {
  if (bf16) return D == 64 ? launch_merge_t<__nv_bfloat16, 64>(nparts, rows, part_o, part_lse, out, lse_out, s)
                           : launch_merge_t<__nv_bfloat16, 128>(nparts, rows, part_o, part_lse, out, lse_out, s);
  return D == 64 ? launch_merge_t<float, 64>(nparts, rows, part_o, part_lse, out, lse_out, s)
                 : launch_merge_t<float, 128>(nparts, rows, part_o, part_lse, out, lse_out, s);
}

cudaError_t launch_finalize(const AttnArgs& a, cudaStream_t s) {
  if (a.bf16) return a.D == 64 ? launch_finalize_t<__nv_bfloat16, 64>(a, s) : launch_finalize_t<__nv_bfloat16, 128>(a, s);
  return a.D == 64 ? launch_finalize_t<float, 64>(a, s) : launch_finalize_t<float, 128>(a, s);
}

}  // namespace tidar
