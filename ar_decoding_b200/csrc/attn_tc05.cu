// attn_tc05.cu -- tensor-core step attention for sm_100a (tcgen05 + TMEM + TMA).
//
// Same operation as the CUDA-core kernel (the three-zone structured-mask
// attention of one TiDAR step: "TiDAR: Think in Diffusion, Talk in
// Autoregression", mauroscia.it section 2; nodesdaily.com (fr), paragraphs on
// the three zones and the masking puzzle), for bf16, head_dim 128, page 64.
//
// Work unit (one CTA): sequence b, KV head g, a tile of 128/G consecutive query
// rows packed with their G query heads into the 128 lanes of the MMA M
// dimension (row m = (rho - rho0) * G + head-in-group), and one split of the
// cached prefix.  The last split also runs the step-key windows (128 step keys
// each) that hold keys visible to the tile, with the mask applied in softmax.
//
// Roles (6 warps):
//   warp 0      TMA producer: Q tile once; per 128-key block two 64-row pages
//               of K and V (paged cache, SWIZZLE_128B) or one step-key window.
//               3-stage ring.  No multicast.
//   warp 1      TMEM owner and MMA issuer (one thread):
//               S_i = Q K_i^T  (kind::f16, A and B from shared memory, fp32 in
//               TMEM, 3 S buffers), then O += P_{i-1} V_{i-1} with P read from
//               TMEM (bf16, written over S) and V as an MN-major operand.
//   warps 2..5  softmax: one thread per TMEM lane (= packed query row).
//               tcgen05.ld of S, mask, online softmax in the log2 domain, P
//               back to TMEM as bf16; O in TMEM is rescaled only when the row
//               maximum grows by more than 2^8; epilogue normalises O.
// Every mbarrier wait is bounded: on expiry the CTA records TIDAR_DEVERR_TIMEOUT,
// stops issuing, drains what it issued (bounded), frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 3;       // K/V ring depth; also the number of S buffers
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // every mbarrier wait gives up after ~1 s

constexpr uint32_t kChunkBytes = 16384;                 // 128 rows x 128 B (64 bf16)
constexpr uint32_t kTileBytes = 2 * kChunkBytes;        // 128 x 128 bf16
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
// barrier indices
constexpr int BAR_Q = 0;
constexpr int BAR_KFULL = 1;     // + stage
constexpr int BAR_VFULL = 4;     // + stage
constexpr int BAR_EMPTY = 7;     // + stage
constexpr int BAR_SFULL = 10;    // + S buffer
constexpr int BAR_PFULL = 13;    // + S buffer
constexpr int BAR_PVDONE = 16;   // + S buffer
constexpr int BAR_FINAL = 19;
constexpr int kNumBars = 20;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;   // [0] TMEM base, [1] abort flag
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;       // slack for 1024-byte alignment

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;                         // S buffers at 0, 128, 256

// kind::f16 instruction descriptors: fp32 accumulate, bf16 A and B, M = 128, N = 128.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);     // B (= V) is MN-major

struct Tc05Params {
  AttnArgs a;
  int rho_per_tile;   // query rows per tile (128 / G)
  int tiles;          // tiles per (b, g)
  float scale_log2;   // softmax scale * log2(e)
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for a phase with a time limit, no error reporting (drain paths).
__device__ __forceinline__ bool wait_quiet(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
  }
}
// Bounded wait.  Gives up after kWaitLimitNs (or early once another thread of
// the CTA has given up), records the timeout and returns false.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitLimitNs) break;
    }
  }
  *abort_flag = 1;
  raise_error(err, TIDAR_DEVERR_TIMEOUT);
  return false;
}

// Bounded wait by a whole warp with a warp-uniform result (the tcgen05.ld/st
// that follow are .sync.aligned and need every lane).
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                              unsigned int* err) {
  const bool ok = wait_bar(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

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
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  if (split == a.nsplit - 1) {
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

// ------------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kThreads, 1)
attn_tc05_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                 const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                 const __grid_constant__ CUtensorMap tm_vs, const Tc05Params prm) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const AttnArgs& a = prm.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int tile = blockIdx.x, split = blockIdx.y;
  const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
  const int rho0 = tile * prm.rho_per_tile;
  const int rho1 = min(a.R, rho0 + prm.rho_per_tile);
  const int rows_valid = (rho1 - rho0) * a.G;

  int P = a.seq_lens[b];
  if (P < 0 || P > a.max_prefix) {
    if (threadIdx.x == 0 && tile == 0 && split == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    P = 0;
  }
  const BlockPlan bp = make_block_plan(a, P, split, rho0, rho1);
  const int32_t* table = a.page_table + (size_t)b * a.max_pages;

  auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool pfull = i >= BAR_PFULL && i < BAR_PFULL + kStages;
      mbar_init(bar(i), pfull ? 4u : 1u);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1 && bp.nb > 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kOffMisc),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = misc[0];

  if (bp.nb == 0) {
    // This split holds no prefix keys of sequence b: an empty partial.
    if (warp >= 2) {
      const int r = 32 * (warp & 3) + lane;
      if (r < rows_valid) {
        const int rho = rho0 + r / a.G, h = g * a.G + r % a.G;
        const size_t row = (size_t)(b * a.R + rho) * a.Hq + h;
        const size_t prow = (size_t)split * a.B * a.R * a.Hq + row;
        float4* po = reinterpret_cast<float4*>(a.part_o + prow * 128);
        for (int i = 0; i < 32; ++i) po[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.part_lse[prow] = -INFINITY;
      }
    }
    return;
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int issued_phase[kStages] = {-1, -1, -1};
      mbar_expect_tx(bar(BAR_Q), 2u * 128u * (uint32_t)(prm.rho_per_tile * a.G));
      tma_load_4d(sb + kOffQ, &tm_q, 0, g * a.G, rho0, b, bar(BAR_Q));
      tma_load_4d(sb + kOffQ + kChunkBytes, &tm_q, 64, g * a.G, rho0, b, bar(BAR_Q));
      bool bad = false;
      for (int i = 0; i < bp.nb; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !wait_bar(bar(BAR_EMPTY + s), (uint32_t)((i / kStages - 1) & 1), abort_flag, a.err)) break;
        const uint32_t kdst = sb + kOffK + s * kTileBytes, vdst = sb + kOffV + s * kTileBytes;
        if (i < bp.npb) {
          const int start = bp.k0 + i * 128;
          const int pa = table[start / 64];
          const bool need_b = start + 64 < bp.kend;
          const int pb = need_b ? table[start / 64 + 1] : -1;
          const bool oka = page_ok(pa, a.num_pages), okb = need_b && page_ok(pb, a.num_pages);
          if (!oka || (need_b && !okb)) bad = true;
          const uint32_t bytes = (uint32_t)(oka + okb) * 2u * 8192u;
          mbar_expect_tx(bar(BAR_KFULL + s), bytes);
          if (oka) {
            tma_load_2d(kdst, &tm_kp, 0, (pa * a.Hkv + g) * 64, bar(BAR_KFULL + s));
            tma_load_2d(kdst + kChunkBytes, &tm_kp, 64, (pa * a.Hkv + g) * 64, bar(BAR_KFULL + s));
          }
          if (okb) {
            tma_load_2d(kdst + 8192, &tm_kp, 0, (pb * a.Hkv + g) * 64, bar(BAR_KFULL + s));
            tma_load_2d(kdst + kChunkBytes + 8192, &tm_kp, 64, (pb * a.Hkv + g) * 64, bar(BAR_KFULL + s));
          }
          mbar_expect_tx(bar(BAR_VFULL + s), bytes);
          if (oka) {
            tma_load_2d(vdst, &tm_vp, 0, (pa * a.Hkv + g) * 64, bar(BAR_VFULL + s));
            tma_load_2d(vdst + kChunkBytes, &tm_vp, 64, (pa * a.Hkv + g) * 64, bar(BAR_VFULL + s));
          }
          if (okb) {
            tma_load_2d(vdst + 8192, &tm_vp, 0, (pb * a.Hkv + g) * 64, bar(BAR_VFULL + s));
            tma_load_2d(vdst + kChunkBytes + 8192, &tm_vp, 64, (pb * a.Hkv + g) * 64, bar(BAR_VFULL + s));
          }
        } else {
          const int w = bp.wins[i - bp.npb];
          mbar_expect_tx(bar(BAR_KFULL + s), kTileBytes);
          tma_load_4d(kdst, &tm_ks, 0, g, w * 128, b, bar(BAR_KFULL + s));
          tma_load_4d(kdst + kChunkBytes, &tm_ks, 64, g, w * 128, b, bar(BAR_KFULL + s));
          mbar_expect_tx(bar(BAR_VFULL + s), kTileBytes);
          tma_load_4d(vdst, &tm_vs, 0, g, w * 128, b, bar(BAR_VFULL + s));
          tma_load_4d(vdst + kChunkBytes, &tm_vs, 64, g, w * 128, b, bar(BAR_VFULL + s));
        }
        issued_phase[s] = i / kStages;
      }
      if (bad) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
      // Drain: on the normal path every load was consumed; after a timeout make
      // sure no copy is still writing shared memory when the CTA exits.
      if (*abort_flag) {
        for (int s = 0; s < kStages; ++s) {
          if (issued_phase[s] < 0) continue;
          wait_quiet(bar(BAR_KFULL + s), issued_phase[s] & 1);
          wait_quiet(bar(BAR_VFULL + s), issued_phase[s] & 1);
        }
        wait_quiet(bar(BAR_Q), 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(bar(BAR_Q), 0, abort_flag, a.err);
      fence_after();
      const uint32_t qa = sb + kOffQ;
      for (int it = 0; ok && it <= bp.nb; ++it) {
        if (it < bp.nb) {
          const int i = it, s = i % kStages;
          if (!wait_bar(bar(BAR_KFULL + s), (uint32_t)((i / kStages) & 1), abort_flag, a.err)) break;
          if (i >= kStages && !wait_bar(bar(BAR_PVDONE + s), (uint32_t)(((i - kStages) / kStages) & 1), abort_flag, a.err)) break;
          fence_after();
          const uint32_t ka = sb + kOffK + s * kTileBytes;
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            const uint32_t off = (kc >> 2) * kChunkBytes + (kc & 3) * 32;
            mma_ss(tmem + s * 128, desc_k_sw128(qa + off), desc_k_sw128(ka + off), kIdescS, kc > 0);
          }
          mma_commit(bar(BAR_SFULL + s));
        }
        if (it >= 1) {
          const int j = it - 1, s = j % kStages;
          if (!wait_bar(bar(BAR_VFULL + s), (uint32_t)((j / kStages) & 1), abort_flag, a.err)) break;
          if (!wait_bar(bar(BAR_PFULL + s), (uint32_t)((j / kStages) & 1), abort_flag, a.err)) break;
          fence_after();
          const uint32_t va = sb + kOffV + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kColO, tmem + s * 128 + kk * 8, desc_mn_sw128(va + kk * 2048, kChunkBytes), kIdescPV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(BAR_PVDONE + s));
          mma_commit(bar(BAR_EMPTY + s));
        }
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar(BAR_FINAL));
      wait_quiet(bar(BAR_FINAL), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int rho_c = min(rho0 + r / a.G, a.R - 1);
    const StepVis vis = step_visibility(a.k, rho_c);
    const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
    const int gt = threadIdx.x - 64;              // 0..127 within the softmax group
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < bp.nb && ok; ++i) {
      const int s = i % kStages;
      if (!warp_wait_bar(bar(BAR_SFULL + s), (uint32_t)((i / kStages) & 1), abort_flag, a.err)) { ok = false; break; }
      fence_after();
      uint32_t x[128];
      tmem_ld32(trow + s * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(x + 0));
      tmem_ld32(trow + s * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
      tmem_ld32(trow + s * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
      tmem_ld32(trow + s * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
      tmem_wait_ld();
      // mask and scale into the log2 domain
      int lo_valid = 64, hi_valid = 64;
      float mb = -INFINITY;
      if (i < bp.npb) {
        const int start = bp.k0 + i * 128;
        lo_valid = min(64, bp.kend - start);
        hi_valid = max(0, min(64, bp.kend - start - 64));
        if (!page_ok(table[start / 64], a.num_pages)) lo_valid = 0;
        if (hi_valid > 0 && !page_ok(table[start / 64 + 1], a.num_pages)) hi_valid = 0;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const bool v = c < 64 ? c < lo_valid : c - 64 < hi_valid;
          const float xs = v ? __uint_as_float(x[c]) * prm.scale_log2 : -INFINITY;
          x[c] = __float_as_uint(xs);
          mb = fmaxf(mb, xs);
        }
      } else {
        const int kb = bp.wins[i - bp.npb] * 128;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int key = kb + c;
          const bool v = key < a.R && step_visible(vis, key);
          const float xs = v ? __uint_as_float(x[c]) * prm.scale_log2 : -INFINITY;
          x[c] = __float_as_uint(xs);
          mb = fmaxf(mb, xs);
        }
      }
      const float m_new = fmaxf(m, mb);
      const bool need = m_new > m + 8.0f;
      if (__any_sync(0xffffffffu, need) && i > 0) {
        // O holds PV of blocks < i: wait for the last one, then rescale in TMEM
        if (!warp_wait_bar(bar(BAR_PVDONE + (i - 1) % kStages), (uint32_t)(((i - 1) / kStages) & 1), abort_flag, a.err)) { ok = false; }
        fence_after();
        const float f = need ? ex2(m - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(trow + kColO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(trow + kColO + 32 * c, o);
        }
        tmem_wait_st();
        l *= f;
      }
      if (need) m = m_new;
      const float base = m == -INFINITY ? 0.f : m;
      uint32_t pk[64];
      float ls = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2(__uint_as_float(x[2 * c]) - base);
        const float p1 = ex2(__uint_as_float(x[2 * c + 1]) - base);
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        const float2 back = __bfloat1622float2(h2);
        ls += back.x + back.y;
        pk[c] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      l += ls;
      tmem_st32(trow + s * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(pk + 0));
      tmem_st32(trow + s * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
      if (i < bp.npb && (lo_valid < 64 || hi_valid < 64)) {
        // keys past the prefix end or on an unmapped page: zero their V rows so
        // that 0 * (whatever the page holds) cannot turn into NaN
        if (!warp_wait_bar(bar(BAR_VFULL + s), (uint32_t)((i / kStages) & 1), abort_flag, a.err)) ok = false;
        uint8_t* vs = smem + kOffV + s * kTileBytes;
        for (int idx = gt; idx < 128 * 16; idx += 128) {
          const int row = idx >> 4, piece = idx & 15;
          const bool inval = row < 64 ? row >= lo_valid : row - 64 >= hi_valid;
          if (inval)
            *reinterpret_cast<uint4*>(vs + (piece >> 3) * kChunkBytes + row * 128 + (piece & 7) * 16) =
                make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_wait_st();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_PFULL + s));
    }
    // epilogue: O / l for this lane's row
    const int last = bp.nb - 1;
    if (ok && !warp_wait_bar(bar(BAR_PVDONE + last % kStages), (uint32_t)((last / kStages) & 1), abort_flag, a.err)) ok = false;
    fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const float lse = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    const bool write = r < rows_valid;
    const int rho = rho0 + r / a.G, h = g * a.G + r % a.G;
    const size_t row = (size_t)(b * a.R + (write ? rho : 0)) * a.Hq + h;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t o[32];
      tmem_ld32(trow + kColO + 32 * c, o);
      tmem_wait_ld();
      if (!write || !ok) continue;
      if (a.nsplit == 1) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + row * 128 + 32 * c;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 v;
          __nv_bfloat162 t0 = __floats2bfloat162_rn(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
          __nv_bfloat162 t1 = __floats2bfloat162_rn(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
          __nv_bfloat162 t3 = __floats2bfloat162_rn(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
          v.x = *reinterpret_cast<uint32_t*>(&t0); v.y = *reinterpret_cast<uint32_t*>(&t1);
          v.z = *reinterpret_cast<uint32_t*>(&t2); v.w = *reinterpret_cast<uint32_t*>(&t3);
          *reinterpret_cast<uint4*>(dst + e) = v;
        }
      } else {
        const size_t prow = (size_t)split * a.B * a.R * a.Hq + row;
        float4* dst = reinterpret_cast<float4*>(a.part_o + prow * 128 + 32 * c);
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          dst[e / 4] = make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                                   __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
      }
    }
    if (write && ok) {
      if (a.nsplit == 1) {
        if (a.lse_out) a.lse_out[row] = lse;
      } else {
        a.part_lse[(size_t)split * a.B * a.R * a.Hq + row] = lse;
      }
    }
  }

  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_tc05(const AttnArgs& a, cudaStream_t s) {
  if (!a.bf16 || a.D != 128 || a.page_size != 64 || a.G > 128) return cudaErrorNotSupported;
  Tc05Params prm;
  prm.a = a;
  prm.rho_per_tile = 128 / a.G;
  prm.tiles = (a.R + prm.rho_per_tile - 1) / prm.rho_per_tile;
  prm.scale_log2 = a.scale * 1.4426950408889634f;

  CUtensorMap tq, tkp, tvp, tks, tvs;
  {
    const cuuint64_t dims[4] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.R, (cuuint64_t)a.B};
    const cuuint64_t str[3] = {256, (cuuint64_t)a.Hq * 256, (cuuint64_t)a.R * a.Hq * 256};
    const cuuint32_t box[4] = {64, (cuuint32_t)a.G, (cuuint32_t)prm.rho_per_tile, 1};
    if (!encode(&tq, a.q, 4, dims, str, box)) return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[2] = {128, (cuuint64_t)a.num_pages * a.Hkv * 64};
    const cuuint64_t str[1] = {256};
    const cuuint32_t box[2] = {64, 64};
    if (!encode(&tkp, a.k_pages, 2, dims, str, box)) return cudaErrorNotSupported;
    if (!encode(&tvp, a.v_pages, 2, dims, str, box)) return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[4] = {128, (cuuint64_t)a.Hkv, (cuuint64_t)a.R, (cuuint64_t)a.B};
    const cuuint64_t str[3] = {256, (cuuint64_t)a.Hkv * 256, (cuuint64_t)a.R * a.Hkv * 256};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    if (!encode(&tks, a.k_blk, 4, dims, str, box)) return cudaErrorNotSupported;
    if (!encode(&tvs, a.v_blk, 4, dims, str, box)) return cudaErrorNotSupported;
  }
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(attn_tc05_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  dim3 grid(prm.tiles, a.nsplit, a.B * a.Hkv);
  attn_tc05_kernel<<<grid, kThreads, kSmemAlloc, s>>>(tq, tkp, tvp, tks, tvs, prm);
  return cudaGetLastError();
}

}  // namespace tidar
