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
// Roles (10 warps):
//   warp 0      TMA producer: Q tile once; per 128-key block two 64-row pages
//               of K and V (paged cache, SWIZZLE_128B) or one step-key window.
//               3-stage ring.  No multicast.
//   warp 1      TMEM owner and MMA issuer (one thread):
//               S = Q K_b^T  (kind::f16, A and B from shared memory, fp32 in
//               TMEM), O_t += P V_b with P read from TMEM (bf16, written over
//               S_t) and V as an MN-major operand.  Blocks alternate between
//               two softmax sets (t = b & 1), each with its own S_t and O_t, so
//               one set's exponentials overlap the other set's loads, maxima
//               and hand-offs.
//   warps 2..9  softmax: set 0 = warps 2..5, set 1 = warps 6..9; one thread
//               per TMEM lane (= packed query row), all 128 block columns.
//               tcgen05.ld of S, mask, online softmax in the log2 domain, P
//               back to TMEM as bf16; O_t is rescaled only when the set's row
//               maximum grows by more than 2^8.  The epilogue merges the two
//               sets (max, sums, O) and writes O / l.
// Every mbarrier wait is bounded: on expiry the CTA records TIDAR_DEVERR_TIMEOUT,
// stops issuing, drains what it issued (bounded), frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"

namespace tidar {

namespace {

constexpr int kThreads = 320;       // producer, MMA, 8 softmax warps
constexpr int kStages = 3;       // K/V ring depth; also the number of S buffers
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // every mbarrier wait gives up after ~1 s
constexpr uint32_t kSuspendHintNs = 10000000u;      // one try_wait sleeps at most 10 ms

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
constexpr uint32_t kOffRed = kOffMisc + 16;              // softmax halves: maxima [2][2][128] f32
constexpr uint32_t kOffOk = kOffRed + 2048;              // and warp status [2][2][4] i32
constexpr uint32_t kSmemUsed = kOffOk + 64;
constexpr uint32_t kSmemAlloc = kSmemUsed;               // the dynamic window is 1024-byte aligned
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
// Softmax set t (block parity) owns S_t (P_t is written over its first 64
// columns) and the accumulator O_t.
__device__ __forceinline__ uint32_t col_s(int t) { return 128u * (uint32_t)t; }
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + 128u * (uint32_t)t; }

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
// Test the phase; if it is incomplete the thread may sleep in hardware until
// the phase completes or the hint (ns) expires, whichever is first.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Optional timeline of one CTA and the start/end of every CTA (build with
// -DTIDAR_TRACE; absent from normal builds).  Slots: [0..15] setup, [16+i]
// producer issue of block i, [256+i] MMA sees K(i), [512+i] S(i) issued,
// [768+i] PV(i) issued, [1024+i] softmax sees S(i), [1280+i] P(i) handed over,
// [1536..] epilogue, [2048 + 2*cta] CTA start / end.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_tidar_trace[2048 + 2 * 8192];
__device__ __forceinline__ bool trace_cta() { return blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0; }
#define TIDAR_TRACE_AT(slot) do { if (trace_cta()) g_tidar_trace[(slot)] = global_ns(); } while (0)
#define TIDAR_TRACE_PH(i, ph) do { if ((i) == 2 && warp == 4 && lane == 0) TIDAR_TRACE_AT(1600 + (ph)); } while (0)
#define TIDAR_TRACE_CTA(which) do { const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (cta_ < 8192) g_tidar_trace[2048 + 2 * cta_ + (which)] = global_ns(); } while (0)
#else
#define TIDAR_TRACE_AT(slot) do {} while (0)
#define TIDAR_TRACE_PH(i, ph) do {} while (0)
#define TIDAR_TRACE_CTA(which) do {} while (0)
#endif

// Wait for a phase with a time limit, no error reporting (drain paths).
__device__ __forceinline__ bool wait_quiet(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}
// Bounded wait.  Gives up after kWaitLimitNs (or early once another thread of
// the CTA has given up), records the timeout and returns false.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitLimitNs) break;
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

// Two non-negative floats -> packed bf16x2 (low half = a), rounded to nearest
// with ties away from zero, using integer ops only (keeps the conversion off
// the transcendental pipe that ex2 saturates).
__device__ __forceinline__ uint32_t pack_bf16x2_pos(float a, float b) {
  return __byte_perm(__float_as_uint(a) + 0x8000u, __float_as_uint(b) + 0x8000u, 0x7632);
}

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
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  if (sb & 1023u) {        // SWIZZLE_128B tiles need 1024-byte alignment: refuse, never misread
    if (threadIdx.x == 0) raise_error(prm.a.err, TIDAR_DEVERR_LAYOUT);
    return;
  }
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
    TIDAR_TRACE_CTA(0);
    TIDAR_TRACE_AT(0);
#ifdef TIDAR_TRACE
    if (trace_cta()) g_tidar_trace[2] = clock64();
#endif
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
  if (threadIdx.x == 0) TIDAR_TRACE_AT(1);

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
        TIDAR_TRACE_AT(16 + min(i, 239));
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
    // Block b belongs to softmax set t = b & 1, which owns S_t and O_t in TMEM.
    // Order: S(0), S(1); then per block b: PV_t(b) and, behind it in the same
    // in-order MMA pipe, S(b+2) into S_t (the columns PV_t(b) reads P from).
    if (lane == 0) {
      bool ok = wait_bar(bar(BAR_Q), 0, abort_flag, a.err);
      fence_after();
      const uint32_t qa = sb + kOffQ;
      auto issue_s = [&](int blk) -> bool {
        const int st = blk % kStages, t = blk & 1;
        if (!wait_bar(bar(BAR_KFULL + st), (uint32_t)((blk / kStages) & 1), abort_flag, a.err)) return false;
        TIDAR_TRACE_AT(256 + min(blk, 255));
        fence_after();
        const uint32_t ka = sb + kOffK + st * kTileBytes;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const uint32_t off = (kc >> 2) * kChunkBytes + (kc & 3) * 32;
          mma_ss(tmem + col_s(t), desc_k_sw128(qa + off), desc_k_sw128(ka + off), kIdescS, kc > 0);
        }
        mma_commit(bar(BAR_SFULL + t));
        TIDAR_TRACE_AT(512 + min(blk, 255));
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && bp.nb > 1) ok = issue_s(1);
      for (int b2 = 0; ok && b2 < bp.nb; ++b2) {
        const int st = b2 % kStages, t = b2 & 1, j = b2 >> 1;
        if (!wait_bar(bar(BAR_VFULL + st), (uint32_t)((b2 / kStages) & 1), abort_flag, a.err)) break;
        if (!wait_bar(bar(BAR_PFULL + t), (uint32_t)(j & 1), abort_flag, a.err)) break;
        fence_after();
        const uint32_t va = sb + kOffV + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8, desc_mn_sw128(va + kk * 2048, kChunkBytes), kIdescPV,
                 (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(BAR_PVDONE + t));
        mma_commit(bar(BAR_EMPTY + st));
        TIDAR_TRACE_AT(768 + min(b2, 255));
        if (b2 + 2 < bp.nb && !issue_s(b2 + 2)) break;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar(BAR_FINAL));
      wait_quiet(bar(BAR_FINAL), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    // Set t (warps 2..5: t = 0, warps 6..9: t = 1) takes blocks b with b & 1 == t
    // and keeps its own running max, row sum and O_t; the two sets' results are
    // merged in the epilogue like two split-KV partials.  One thread per TMEM
    // lane (= packed query row), all 128 columns of the block.
    const int q4 = warp & 3;
    const int t = (warp - 2) >> 2;
    const int r = 32 * q4 + lane;
    const int rho_c = min(rho0 + r / a.G, a.R - 1);
    const StepVis vis = step_visibility(a.k, rho_c);
    const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
    const int gt = threadIdx.x - 64 - 128 * t;          // 0..127 within the set
    const bool live = 32 * q4 < rows_valid;             // the warp holds at least one real row
    const float sl2 = prm.scale_log2;
    const int nbt = (bp.nb - t + 1) >> 1;               // blocks of this set
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nbt; ++j) {
      const int b2 = 2 * j + t;
      if (t == 0 && warp == 4 && lane == 0) TIDAR_TRACE_AT(1700 + min(b2, 255));
      if (!warp_wait_bar(bar(BAR_SFULL + t), (uint32_t)(j & 1), abort_flag, a.err)) { ok = false; break; }
      fence_after();
      if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1024 + min(b2, 255));
      TIDAR_TRACE_PH(b2, 0);
      int lo_valid = 64, hi_valid = 64, kb = 0;
      const bool window = b2 >= bp.npb;
      if (!window) {
        const int start = bp.k0 + b2 * 128;
        lo_valid = min(64, bp.kend - start);
        hi_valid = max(0, min(64, bp.kend - start - 64));
        if (lo_valid < 64 || hi_valid < 64) {            // page checks only where a page may be absent
          if (!page_ok(table[start / 64], a.num_pages)) lo_valid = 0;
          if (hi_valid > 0 && !page_ok(table[start / 64 + 1], a.num_pages)) hi_valid = 0;
        }
      } else {
        kb = bp.wins[b2 - bp.npb] * 128;
      }
      const bool full = !window && lo_valid == 64 && hi_valid == 64;
      const uint32_t scol = col_s(t);
      // visibility of column c of this block for this thread's row (masked blocks)
      auto visible = [&](int c) -> bool {
        if (window) {
          const int key = kb + c;
          return key < a.R && step_visible(vis, key);
        }
        return c < 64 ? c < lo_valid : c - 64 < hi_valid;
      };
      // pass 1: block maximum of the raw scores (the positive scale commutes)
      float mb = -INFINITY;
      if (live) {
        uint32_t x[128];
        tmem_ld32(trow + scol + 0, *reinterpret_cast<uint32_t(*)[32]>(x + 0));
        tmem_ld32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
        tmem_ld32(trow + scol + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
        tmem_ld32(trow + scol + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
        tmem_wait_ld();
        TIDAR_TRACE_PH(b2, 2);
        if (!full) {
          // masked block (rare): invisible keys become -inf in TMEM as well, so
          // pass 2 needs no mask (2^-inf = 0)
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!visible(c)) x[c] = 0xff800000u;
          tmem_st32(trow + scol + 0, *reinterpret_cast<uint32_t(*)[32]>(x + 0));
          tmem_st32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
          tmem_st32(trow + scol + 64, *reinterpret_cast<uint32_t(*)[32]>(x + 64));
          tmem_st32(trow + scol + 96, *reinterpret_cast<uint32_t(*)[32]>(x + 96));
          tmem_wait_st();
        }
        float mx[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mx[e] = __uint_as_float(x[e]);
#pragma unroll
        for (int c = 4; c < 128; ++c) mx[c & 3] = fmaxf(mx[c & 3], __uint_as_float(x[c]));
        mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
      }
      TIDAR_TRACE_PH(b2, 3);
      const float m_new = fmaxf(m, mb);
      const bool need = m_new > m + 8.0f;
      const float f_resc = need ? ex2(m - m_new) : 1.0f;   // factor for O_t and l (m = -inf -> 0)
      if (need) m = m_new;
      const float nbase = m == -INFINITY ? 0.f : -m;
      TIDAR_TRACE_PH(b2, 4);
      // pass 2: P = 2^(score * scale - m) in bf16, packed in registers from two
      // 64-column reloads of S and stored to TMEM (over S) only after both
      // reloads; the row sum keeps the fp32 values
      float lblk = 0.f;
      if (live) {
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[64];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t x[64];
          tmem_ld32(trow + scol + 64 * h2, *reinterpret_cast<uint32_t(*)[32]>(x + 0));
          tmem_ld32(trow + scol + 64 * h2 + 32, *reinterpret_cast<uint32_t(*)[32]>(x + 32));
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2(fmaf(__uint_as_float(x[2 * c]), sl2, nbase));
            const float p1 = ex2(fmaf(__uint_as_float(x[2 * c + 1]), sl2, nbase));
            ls[c & 3] += p0 + p1;
            pk[32 * h2 + c] = pack_bf16x2_pos(p0, p1);
          }
        }
        tmem_st32(trow + scol + 0, *reinterpret_cast<uint32_t(*)[32]>(pk + 0));
        tmem_st32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
        lblk = (ls[0] + ls[1]) + (ls[2] + ls[3]);
      }
      TIDAR_TRACE_PH(b2, 5);
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O_t holds PV of this set's earlier blocks: wait for the last one and
        // rescale it before this block's PV is released to the MMA warp
        if (!warp_wait_bar(bar(BAR_PVDONE + t), (uint32_t)((j - 1) & 1), abort_flag, a.err)) { ok = false; break; }
        fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[16];
          tmem_ld16(trow + col_o(t) + 16 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_resc);
          tmem_st16(trow + col_o(t) + 16 * c, o);
        }
      }
      l = l * f_resc + lblk;
      if (!window && (lo_valid < 64 || hi_valid < 64)) {
        // keys past the prefix end or on an unmapped page: zero their V rows so
        // that 0 * (whatever the page holds) cannot turn into NaN
        const int st = b2 % kStages;
        if (!warp_wait_bar(bar(BAR_VFULL + st), (uint32_t)((b2 / kStages) & 1), abort_flag, a.err)) { ok = false; break; }
        uint8_t* vs = smem + kOffV + st * kTileBytes;
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
      TIDAR_TRACE_PH(b2, 6);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_PFULL + t));
      if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1280 + min(b2, 255));
      if (b2 == 2 && lane == 0) TIDAR_TRACE_AT(1632 + warp);
    }
    // ---- epilogue: merge the two sets' partials; set t writes columns [64t, 64t+64)
    float* xm = reinterpret_cast<float*>(smem + kOffRed);            // [2 set][128] running max
    float* xl = xm + 256;                                            // [2 set][128] row sums
    xm[t * 128 + r] = m;
    xl[t * 128 + r] = l;
    int* xok = reinterpret_cast<int*>(smem + kOffOk);
    if (lane == 0) xok[t * 4 + q4] = ok ? 1 : 0;
    asm volatile("bar.sync %0, 64;" ::"r"(1 + q4) : "memory");
    const float mo = xm[(t ^ 1) * 128 + r], lo = xl[(t ^ 1) * 128 + r];
    ok = ok && xok[(t ^ 1) * 4 + q4] != 0;
    // both sets' last PV must be complete before O_0 and O_1 are read
    const int nb0 = (bp.nb + 1) >> 1, nb1 = bp.nb >> 1;
    if (ok && nb0 > 0 && !warp_wait_bar(bar(BAR_PVDONE + 0), (uint32_t)((nb0 - 1) & 1), abort_flag, a.err)) ok = false;
    if (ok && nb1 > 0 && !warp_wait_bar(bar(BAR_PVDONE + 1), (uint32_t)((nb1 - 1) & 1), abort_flag, a.err)) ok = false;
    fence_after();
    if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1536);
    const float m0 = t == 0 ? m : mo, m1 = t == 0 ? mo : m;
    const float l0 = t == 0 ? l : lo, l1 = t == 0 ? lo : l;
    const float mt = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - mt);
    const float f1 = (m1 == -INFINITY || nb1 == 0) ? 0.f : ex2(m1 - mt);
    const float lt = l0 * f0 + l1 * f1;
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    const float g0 = f0 * inv, g1 = f1 * inv;
    const float lse = lt > 0.f ? (mt + log2f(lt)) * 0.69314718055994531f : -INFINITY;
    const bool write = r < rows_valid && ok;
    const int rho = rho0 + r / a.G, h = g * a.G + r % a.G;
    const size_t row = (size_t)(b * a.R + (r < rows_valid ? rho : 0)) * a.Hq + h;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t o0[32], o1[32];
      const int col0 = 64 * t + 32 * c;
      tmem_ld32(trow + col_o(0) + col0, o0);
      if (nb1 > 0) tmem_ld32(trow + col_o(1) + col0, o1);
      tmem_wait_ld();
      if (!write) continue;
      float* v = reinterpret_cast<float*>(o0);
#pragma unroll
      for (int e = 0; e < 32; ++e)
        v[e] = __uint_as_float(o0[e]) * g0 + (nb1 > 0 ? __uint_as_float(o1[e]) * g1 : 0.f);
      if (a.nsplit == 1) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + row * 128 + col0;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 u;
          __nv_bfloat162 t0 = __floats2bfloat162_rn(v[e], v[e + 1]);
          __nv_bfloat162 t1 = __floats2bfloat162_rn(v[e + 2], v[e + 3]);
          __nv_bfloat162 t2 = __floats2bfloat162_rn(v[e + 4], v[e + 5]);
          __nv_bfloat162 t3 = __floats2bfloat162_rn(v[e + 6], v[e + 7]);
          u.x = *reinterpret_cast<uint32_t*>(&t0); u.y = *reinterpret_cast<uint32_t*>(&t1);
          u.z = *reinterpret_cast<uint32_t*>(&t2); u.w = *reinterpret_cast<uint32_t*>(&t3);
          *reinterpret_cast<uint4*>(dst + e) = u;
        }
      } else {
        const size_t prow = (size_t)split * a.B * a.R * a.Hq + row;
        float4* dst = reinterpret_cast<float4*>(a.part_o + prow * 128 + col0);
#pragma unroll
        for (int e = 0; e < 32; e += 4) dst[e / 4] = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
      }
    }
    if (write && t == 0) {
      if (a.nsplit == 1) {
        if (a.lse_out) a.lse_out[row] = lse;
      } else {
        a.part_lse[(size_t)split * a.B * a.R * a.Hq + row] = lse;
      }
    }
  }

  fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    TIDAR_TRACE_AT(1537);
    TIDAR_TRACE_CTA(1);
#ifdef TIDAR_TRACE
    if (trace_cta()) g_tidar_trace[3] = clock64();
#endif
  }
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

#ifdef TIDAR_TRACE
extern "C" int tidar_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_tidar_trace, bytes);
}
extern "C" int tidar_trace_clear(void) {
  static unsigned long long zeros[2048 + 2 * 8192];
  return (int)cudaMemcpyToSymbol(g_tidar_trace, zeros, sizeof zeros);
}
#endif

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
