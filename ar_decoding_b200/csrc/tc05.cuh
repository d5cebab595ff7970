// tc05.cuh -- tcgen05 (5th-generation tensor core) helpers shared by the
// sm_100a attention kernels: TMEM fences, shared-memory matrix descriptors,
// MMA issue and commit, TMEM loads and stores, packed fp32x2 arithmetic, and
// the per-CTA key-block plan of a step attention (prefix blocks of 128 keys,
// then the step-key windows the tile's rows can see).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace tidar {
namespace tc05 {

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptors (SWIZZLE_128B, sm_100 version bits).
// K-major: 8-row groups 1024 B apart; the K offset inside the 128-byte swizzle
// row is added to the start address.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major: 64-element MN atoms `lbo` bytes apart, 8-row K groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d), "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

#define TIDAR_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define TIDAR_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : TIDAR_R8(0), TIDAR_R8(8), TIDAR_R8(16), TIDAR_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), TIDAR_W8(0), TIDAR_W8(8), TIDAR_W8(16), TIDAR_W8(24)
      : "memory");
}
#define TIDAR_R16(i) TIDAR_R8(i), TIDAR_R8(i + 8)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : TIDAR_R16(0)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16};"
      ::"r"(taddr), TIDAR_W8(0), TIDAR_W8(8)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// ---- packed fp32x2 helpers (sm_100) and the exponential split --------------
__device__ __forceinline__ uint64_t f2_make(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (lo, hi) -> bf16x2, round to nearest even
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// ------------------------------------------------------------------ key masks
// Bits [a, b) of the 32-column word w (columns 32 w .. 32 w + 31).
__device__ __forceinline__ uint32_t col_bits(int lo, int hi, int w) {
  const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 32);
  if (b <= a) return 0u;
  const uint32_t run = b - a == 32 ? 0xffffffffu : ((1u << (b - a)) - 1u);
  return run << a;
}
// Visibility of the 128 columns of a key block as four 32-bit words.  A
// step-key window starting at step key kb: the row's visible step keys are
// the intervals [0, e1) and [b0, b1) (zone mask), below R.  A prefix block:
// columns [0, lo_valid) of its first page and [64, 64 + hi_valid) of its second.
__device__ __forceinline__ void block_mask(bool window, int kb, const StepVis& vis, int R, int lo_valid,
                                           int hi_valid, uint32_t (&mw)[4]) {
  int l1, h1, l2, h2;
  if (window) {
    const int top = R - kb;                              // keys past R are not step keys
    l1 = 0;
    h1 = min(vis.e1 - kb, top);
    l2 = vis.b0 - kb;
    h2 = min(vis.b1 - kb, top);
  } else {
    l1 = 0;
    h1 = lo_valid;
    l2 = 64;
    h2 = 64 + hi_valid;
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) mw[w] = col_bits(l1, h1, w) | col_bits(l2, h2, w);
}
// ------------------------------------------------------------------ block plan
// Blocks 0..npb-1: 128 prefix keys from k0; then nw step-key windows.
struct BlockPlan {
  int k0, kend, npb, nw, nb;
  int wins[4];
};

__device__ __forceinline__ BlockPlan make_block_plan(const AttnArgs& a, int P, int split, int rho0,
                                                     int rho1) {
  BlockPlan bp;
  bp.k0 = split * a.keys_per_split;
  bp.kend = min(P, bp.k0 + a.keys_per_split);
  bp.npb = bp.kend > bp.k0 ? (bp.kend - bp.k0 + 127) / 128 : 0;
  bp.nw = 0;
  if (split == a.nsplit - 1 && a.step_keys) {
    bp.wins[bp.nw++] = 0;                       // drafts D_1..D_k (k <= 16) live in window 0
    if (a.k > 0 && rho1 - 1 >= a.k) {           // the tile holds mask-slot rows
      const int jlo = (max(rho0, a.k) - a.k) / a.k + 1;
      const int jhi = (rho1 - 1 - a.k) / a.k + 1;
      const int lo = a.k + (jlo - 1) * a.k, hi = a.k + jhi * a.k;
      for (int w = lo / 128; w <= (hi - 1) / 128 && bp.nw < 4; ++w)
        if (w != 0) bp.wins[bp.nw++] = w;
    }
  }
  bp.nb = bp.npb + bp.nw;
  return bp;
}

__device__ __forceinline__ bool page_ok(int page, int num_pages) { return page >= 0 && page < num_pages; }

// ------------------------------------------------------------------ split merge
// Key splits of one query tile run as the CTAs of a thread-block cluster and
// merge through L2.  Every split has written its normalised partial rows (fp32
// O of 128 columns, and the row's lse) to part_o / part_lse, laid out
// [split][stride rows]; a cluster barrier (release / acquire at cluster scope)
// orders those writes before these reads.  This CTA merges `owned` rows,
// row_of(i) giving the i-th one's row index (negative: skip).  A group of
// 32 / CPT threads merges one row, CPT float4 columns each, so that with
// enough threads every owned row is in flight at once: one round trip for the
// lse of all splits, one for the rows.  Loads bypass L1 (other SMs wrote the
// partials).  The weights are exp(lse_s - max); a split with lse = -inf saw no
// key and may have written no values: it is selected away, not multiplied.
template <int CPT, class RowOf>
__device__ __forceinline__ void merge_l2_rows_t(const float* __restrict__ part_o,
                                                const float* __restrict__ part_lse, long long stride, int ns,
                                                int owned, RowOf row_of, __nv_bfloat16* out, float* lse_out) {
  constexpr int kG = 32 / CPT;
  const int sub = (int)threadIdx.x % kG;
  const int groups = (int)blockDim.x / kG;
  for (int i = (int)threadIdx.x / kG; i < owned; i += groups) {
    const long long row = row_of(i);
    if (row < 0) continue;
    float l2[kMaxCluster];
    float mx = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxCluster; ++s) {
      l2[s] = s < ns ? __ldcg(part_lse + s * stride + row) * 1.4426950408889634f : -INFINITY;
      mx = fmaxf(mx, l2[s]);
    }
    float4 acc[CPT];
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxCluster; ++s) {
      if (s < ns) {
        const float4* src = reinterpret_cast<const float4*>(part_o + (s * stride + row) * 128) + sub * CPT;
        float4 x[CPT];
#pragma unroll
        for (int c = 0; c < CPT; ++c) x[c] = __ldcg(src + c);
        if (l2[s] != -INFINITY) {
          const float w = ex2(l2[s] - mx);
          wsum += w;
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            acc[c].x = fmaf(w, x[c].x, acc[c].x); acc[c].y = fmaf(w, x[c].y, acc[c].y);
            acc[c].z = fmaf(w, x[c].z, acc[c].z); acc[c].w = fmaf(w, x[c].w, acc[c].w);
          }
        }
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      uint2 u;
      u.x = cvt_bf16x2(acc[c].x * inv, acc[c].y * inv);
      u.y = cvt_bf16x2(acc[c].z * inv, acc[c].w * inv);
      *reinterpret_cast<uint2*>(out + row * 128 + 4 * (sub * CPT + c)) = u;
    }
    if (sub == 0 && lse_out) lse_out[row] = wsum > 0.f ? (mx + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
  }
}

// This CTA's share of the merge, the group size picked so that all `owned`
// rows go in one pass when the block has the threads (at most 8 columns of 4
// per thread).
template <class RowOf>
__device__ __forceinline__ void merge_l2_rows(const float* part_o, const float* part_lse, long long stride,
                                              int ns, int owned, RowOf row_of, __nv_bfloat16* out,
                                              float* lse_out) {
  const int per = (32 * owned + (int)blockDim.x - 1) / (int)blockDim.x;
  if (per <= 1) merge_l2_rows_t<1>(part_o, part_lse, stride, ns, owned, row_of, out, lse_out);
  else if (per <= 2) merge_l2_rows_t<2>(part_o, part_lse, stride, ns, owned, row_of, out, lse_out);
  else if (per <= 4) merge_l2_rows_t<4>(part_o, part_lse, stride, ns, owned, row_of, out, lse_out);
  else merge_l2_rows_t<8>(part_o, part_lse, stride, ns, owned, row_of, out, lse_out);
}

}  // namespace tc05
}  // namespace tidar
