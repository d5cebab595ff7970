// tc05.cuh -- tcgen05 (5th-generation tensor core) helpers shared by the
// sm_100a attention kernels: TMEM fences, shared-memory matrix descriptors,
// MMA issue and commit, TMEM loads and stores, packed fp32x2 arithmetic, and
// the per-CTA key-block plan of a step attention (prefix blocks of 128 keys,
// then the step-key windows the tile's rows can see).
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

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
// Eight MMAs accumulating into one D (a 128-deep K sweep in steps of 16) as
// one asm block: the 16 operands are formed before it, so the issuing thread
// spends its instructions on the MMAs themselves.  The first MMA accumulates
// when acc0 != 0, the other seven always.
__device__ __forceinline__ void mma_ss_x8(uint32_t d, const uint64_t (&a)[8], const uint64_t (&b)[8], uint32_t idesc,
                                          uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %18, 0;\n\tsetp.eq.b32 q, %18, %18;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %9, %17, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %10, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %3, %11, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %4, %12, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %5, %13, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %6, %14, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %7, %15, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %8, %16, %17, q;\n\t}"
      ::"r"(d), "l"(a[0]), "l"(a[1]), "l"(a[2]), "l"(a[3]), "l"(a[4]), "l"(a[5]), "l"(a[6]), "l"(a[7]),
        "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
        "r"(acc0)
      : "memory");
}
__device__ __forceinline__ void mma_ts_x8(uint32_t d, const uint32_t (&a)[8], const uint64_t (&b)[8], uint32_t idesc,
                                          uint32_t acc0) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %18, 0;\n\tsetp.eq.b32 q, %18, %18;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %9, %17, p;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%2], %10, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%3], %11, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%4], %12, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%5], %13, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%6], %14, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%7], %15, %17, q;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%8], %16, %17, q;\n\t}"
      ::"r"(d), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
        "l"(b[0]), "l"(b[1]), "l"(b[2]), "l"(b[3]), "l"(b[4]), "l"(b[5]), "l"(b[6]), "l"(b[7]), "r"(idesc),
        "r"(acc0)
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
// 64 consecutive 32-bit TMEM columns of this thread's lane (one round trip).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, "
      "%51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : TIDAR_R8(0), TIDAR_R8(8), TIDAR_R8(16), TIDAR_R8(24), TIDAR_R8(32), TIDAR_R8(40), TIDAR_R8(48),
        TIDAR_R8(56)
      : "r"(taddr));
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

// ------------------------------------------------------------------ row write-out
// After the main loop a CTA's normalised O rows pass through shared memory,
// `kStageStride` floats per row (the padding keeps the softmax threads' row
// writes -- one row per lane -- free of bank conflicts), so that every global
// store and load below moves whole rows: one warp instruction per row of 128
// columns, lane l holding columns 4l .. 4l+3.  lst / wst hold each row's lse
// (-inf where the row could not be computed) and whether it is valid (a CTA
// whose bounded wait ran out writes no output rows, and its partial rows get
// lse = -inf).
constexpr int kStageStride = 132;

// Final bf16 rows and their lse; row_of(i) = output row of staged row i
// (negative: no such row).
template <class RowOf>
__device__ __forceinline__ void store_rows_bf16(const float* ost, const float* lst, const int* wst, int nrows,
                                                RowOf row_of, __nv_bfloat16* out, float* lse_out) {
  const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31, nw = (int)blockDim.x >> 5;
  for (int i = warp; i < nrows; i += nw) {
    if (!wst[i]) continue;
    const long long row = row_of(i);
    if (row < 0) continue;
    const float4 v = *reinterpret_cast<const float4*>(ost + i * kStageStride + 4 * lane);
    uint2 u;
    u.x = cvt_bf16x2(v.x, v.y);
    u.y = cvt_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(out + row * 128 + 4 * lane) = u;
    if (lane == 0 && lse_out) lse_out[row] = lst[i];
  }
}

// fp32 partial rows of one key split; prow_of(i) = row of staged row i in the
// partials, laid out [split][rows][128] and [split][rows] (negative: no such
// row).
template <class RowOf>
__device__ __forceinline__ void store_rows_partial(const float* ost, const float* lst, const int* wst, int nrows,
                                                   RowOf prow_of, float* part_o, float* part_lse) {
  const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31, nw = (int)blockDim.x >> 5;
  for (int i = warp; i < nrows; i += nw) {
    const long long prow = prow_of(i);
    if (prow < 0) continue;
    const bool w = wst[i] != 0;
    if (w) reinterpret_cast<float4*>(part_o + prow * 128)[lane] = *reinterpret_cast<const float4*>(ost + i * kStageStride + 4 * lane);
    if (lane == 0) part_lse[prow] = w ? lst[i] : -INFINITY;
  }
}

// Split merge over distributed shared memory.  The splits of a query tile are
// the CTAs of one thread-block cluster (cluster rank = split); every CTA has
// staged its normalised rows (ost, kStageStride floats per row) and their lse
// (lst; -inf for a row it could not compute) in its own shared memory, and a
// cluster barrier orders that before these reads.  This CTA merges staged
// rows r = i * ns + rank for i < owned: lane s < ns reads split s's lse, the
// weights exp(lse_s - max) and their sum come from warp shuffles, then every
// lane reads its 4 columns of each split's row -- 512 contiguous bytes per
// warp and split, so the owner's banks see no conflicts -- U rows per warp in
// flight.  A split with lse = -inf saw no key: its weight is 0 and its row is
// selected away, not multiplied.  out_row(r) = output row of staged row r
// (negative: no such row).  The caller keeps its shared memory alive (a second
// cluster barrier) until every peer is done reading.
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
template <int U, int NC, class RowOf>
__device__ __forceinline__ void merge_rows_t(const float* ost, const float* lst, int ns, int rank, int owned,
                                             RowOf out_row, __nv_bfloat16* out, float* lse_out) {
  const int warp = (int)threadIdx.x >> 5, lane = (int)threadIdx.x & 31, nw = (int)blockDim.x >> 5;
  constexpr unsigned kAll = 0xffffffffu;
  const uint32_t ost_a = smem_u32(ost), lst_a = smem_u32(lst);
  for (int i0 = warp * U; i0 < owned; i0 += nw * U) {
    int r[U];
    long long orow[U];
    float w[U], wsum[U], mx[U];
    float4 x[U][NC];
    // the lse of every split and the rows of the first NC splits are all in
    // flight before the first of them is used
    auto load_chunk = [&](int s0) {
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const int sp = s0 + j;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          x[u][j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (orow[u] >= 0 && sp < ns) {
            const int e = r[u] * kStageStride + 4 * lane;
            x[u][j] = sp == rank ? *reinterpret_cast<const float4*>(ost + e)
                                 : ld_cluster_f32x4(mapa(ost_a + 4u * (uint32_t)e, (uint32_t)sp));
          }
        }
      }
    };
#pragma unroll
    for (int u = 0; u < U; ++u) {
      r[u] = (i0 + u) * ns + rank;
      orow[u] = i0 + u < owned ? out_row(r[u]) : -1;
      w[u] = (orow[u] >= 0 && lane < ns)
                 ? ld_cluster_f32(mapa(lst_a + 4u * (uint32_t)r[u], (uint32_t)lane)) * 1.4426950408889634f
                 : -INFINITY;
    }
    load_chunk(0);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float m = w[u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kAll, m, o));
      mx[u] = m;
      w[u] = w[u] == -INFINITY ? 0.f : ex2(w[u] - m);
      float sm = w[u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(kAll, sm, o);
      wsum[u] = sm;
    }
    float4 acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += NC) {
      if (s0 > 0) load_chunk(s0);
#pragma unroll
      for (int j = 0; j < NC; ++j) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const float ws = __shfl_sync(kAll, w[u], (s0 + j) & 31);
          if (s0 + j < ns && ws > 0.f) {
            acc[u].x = fmaf(ws, x[u][j].x, acc[u].x); acc[u].y = fmaf(ws, x[u][j].y, acc[u].y);
            acc[u].z = fmaf(ws, x[u][j].z, acc[u].z); acc[u].w = fmaf(ws, x[u][j].w, acc[u].w);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (orow[u] < 0) continue;
      const float inv = wsum[u] > 0.f ? 1.f / wsum[u] : 0.f;
      uint2 o;
      o.x = cvt_bf16x2(acc[u].x * inv, acc[u].y * inv);
      o.y = cvt_bf16x2(acc[u].z * inv, acc[u].w * inv);
      *reinterpret_cast<uint2*>(out + orow[u] * 128 + 4 * lane) = o;
      if (lane == 0 && lse_out)
        lse_out[orow[u]] = wsum[u] > 0.f ? (mx[u] + log2f(wsum[u])) * 0.69314718055994531f : -INFINITY;
    }
  }
}

// This CTA's share of the merge: U rows per warp (at most kMaxU), NC splits'
// rows in flight per chunk, U picked so that the block's warps take all
// `owned` rows in one pass where they can (ns <= 32).
template <int kMaxU, int NC, class RowOf>
__device__ __forceinline__ void merge_rows(const float* ost, const float* lst, int ns, int rank, int owned,
                                           RowOf out_row, __nv_bfloat16* out, float* lse_out) {
  const int nw = (int)blockDim.x >> 5;
  const int per = (owned + nw - 1) / nw;
  if (per <= 1 || kMaxU == 1) merge_rows_t<1, NC>(ost, lst, ns, rank, owned, out_row, out, lse_out);
  else if (per <= 2 || kMaxU == 2) merge_rows_t<2, NC>(ost, lst, ns, rank, owned, out_row, out, lse_out);
  else merge_rows_t<4, NC>(ost, lst, ns, rank, owned, out_row, out, lse_out);
}

}  // namespace tc05
}  // namespace tidar
