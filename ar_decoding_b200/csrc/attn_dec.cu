// attn_dec.cu -- warp-MMA step attention for small query blocks (sm_100a).
//
// The same three-zone step attention as the other kernels ("TiDAR: Think in
// Diffusion, Talk in Autoregression", mauroscia.it section 2; nodesdaily.com
// (fr), paragraphs on the three zones and the masking puzzle), for steps whose
// query block packs into at most 16 rows per KV head (R * G <= 16: plain
// decode with k = 0, and k = 1 with G <= 8).  Such a block is far too thin for
// the 128-row tcgen05 tiles and the step is a stream of the paged KV cache,
// so this kernel is built to keep HBM busy: one TMA producer warp keeps a
// 6-stage ring of 64-key K/V pages (192 KB) in flight, and eight compute warps
// work on two pages at a time (pages alternate between two groups of four
// warps, so every SM sub-partition has two independent warps); each warp takes
// 16 keys of its page with mma.sync m16n8k16 (bf16, fp32 accumulate): S = Q K^T,
// an online softmax in registers, and the score fragments reused directly as
// the A operand of O += P V.  The eight warps' (max, sum, O) merge in shared
// memory at the end; key splits go to the workspace and the finalize launch
// merges them and appends the draft rows.
//
// Grid (split, b * Hkv); 288 threads (warp 0 producer, warps 1..8 compute).
// Every mbarrier wait is bounded (~1 s): on expiry the CTA records
// TIDAR_DEVERR_TIMEOUT, the producer drains the copies it issued, and the CTA
// exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tidar {

namespace {

constexpr int kDecThreads = 288;
constexpr int kDecCompute = 8;                          // compute warps: 2 page groups x 4 key quarters
constexpr int kDecStages = 6;
constexpr uint32_t kHalfPage = 8192;                    // 64 keys x 64 dims bf16 (one 128-byte swizzled box)
constexpr uint32_t kPageBytes = 2 * kHalfPage;          // 64 keys x 128 dims
constexpr uint32_t kStageBytes = 2 * kPageBytes;        // K page then V page
constexpr uint32_t kQHalf = 2048;                       // 16 rows x 64 dims bf16
constexpr uint32_t kOffQd = 0;
constexpr uint32_t kOffStage = 4096;
constexpr uint32_t kOffBarD = kOffStage + kDecStages * kStageBytes;
constexpr int DBAR_Q = 0;
constexpr int DBAR_FULL = 1;                            // + stage
constexpr int DBAR_EMPTY = 1 + kDecStages;              // + stage (count: the page group's 4 warps)
constexpr int kDecBars = 1 + 2 * kDecStages;
constexpr uint32_t kOffMiscD = kOffBarD + kDecBars * 8;  // [0] abort flag, [1 + s] stage s holds no page
constexpr uint32_t kDecSmem = kOffMiscD + 4 * (1 + kDecStages);
static_assert(kDecSmem <= 232448, "shared memory budget");

// Optional timeline (build with -DTIDAR_TRACE; absent from normal builds):
// CTA (0, 0): [0] setup done, [1] prefix length read, [2] first copy issued,
// [3] Q seen by compute warp 1, [16+i] page i seen by warp 1, [80+i] page i
// done by warp 1, [150] merge start, [151] end; [256 + 2*cta] start / end of
// every CTA.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_dec_trace[256 + 2 * 4096];
#define DEC_TRACE(slot) do { if (blockIdx.x == 0 && blockIdx.y == 0) g_dec_trace[(slot)] = global_ns(); } while (0)
#define DEC_TRACE_CTA(w) do { const unsigned c_ = blockIdx.x + gridDim.x * blockIdx.y; \
    if (c_ < 4096) g_dec_trace[256 + 2 * c_ + (w)] = global_ns(); } while (0)
#else
#define DEC_TRACE(slot) do {} while (0)
#define DEC_TRACE_CTA(w) do {} while (0)
#endif

struct DecParams {
  AttnArgs a;
  float scale_log2;
  int M;              // packed query rows per KV head (R * G <= 16)
  int cluster;        // the nsplit CTAs of one (b, g) form a cluster and merge on chip
};

// CTA result area for the cluster merge (past the warp-merge scratch):
// normalised O [16 rows][128] fp32 and lse [16].
constexpr uint32_t kOffCpo = kOffStage + 96 * 1024;
constexpr uint32_t kOffCpl = kOffCpo + 16 * 128 * 4;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Byte address of (row, 16-byte unit u) in a 128-byte-swizzled tile whose rows
// are 128 bytes (64 bf16): the unit index is XORed with row % 8.
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int u) {
  return base + (uint32_t)row * 128u + ((uint32_t)(u ^ (row & 7)) << 4);
}

__global__ void __launch_bounds__(kDecThreads, 1)
attn_dec_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                const __grid_constant__ CUtensorMap tm_vs, const DecParams prm) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const AttnArgs& a = prm.a;
  if (sb & 1023u) {        // 128-byte swizzled tiles need 1024-byte alignment: refuse, never misread
    if (threadIdx.x == 0) raise_error(a.err, TIDAR_DEVERR_LAYOUT);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int b = blockIdx.y / a.Hkv, g = blockIdx.y % a.Hkv;
  auto bar = [&](int i) -> uint32_t { return sb + kOffBarD + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMiscD);
  volatile int* stage_bad = abort_flag + 1;

  // Q rows M..15 of the tile stay zero (the copy writes rows 0..M-1)
  for (int i = threadIdx.x; i < 4096 / 16; i += kDecThreads)
    reinterpret_cast<uint4*>(smem + kOffQd)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecBars; ++i) mbar_init(bar(i), i >= DBAR_EMPTY ? 4u : 1u);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) { DEC_TRACE_CTA(0); DEC_TRACE(0); }

  pdl_wait();       // the previous kernel on the stream is complete from here on
  pdl_trigger();

  // The producer's first two 32-page windows of the page table do not depend on
  // the prefix length, so they load alongside it.
  const int32_t* table = a.page_table + (size_t)b * a.max_pages;
  const int pg0 = split * a.keys_per_split / 64;
  auto load_win = [&](int base) -> int {
    const int pi = pg0 + base + lane;
    return pi < a.max_pages ? table[pi] : -1;
  };
  int win_cur = -1, win_nxt = -1;
  if (warp == 0) {
    win_cur = load_win(0);
    win_nxt = load_win(32);
  }
  int P = a.seq_lens[b];
  const bool len_ok = P >= 0 && P <= a.max_prefix;
  if (!len_ok) {
    if (threadIdx.x == 0 && split == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    P = 0;
  }
  if (threadIdx.x == 0 && P >= 0) DEC_TRACE(1);
  const int k0 = split * a.keys_per_split;               // a multiple of 64
  const int kend = min(P, k0 + a.keys_per_split);
  const int npg = kend > k0 ? (kend - k0 + 63) / 64 : 0;
  const bool last = split == a.nsplit - 1;
  const int nb = npg + (last ? 1 : 0);                   // + the step-key window (R <= 16 keys)

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    constexpr unsigned kAll = 0xffffffffu;
    if (lane == 0) {
      mbar_expect_tx(bar(DBAR_Q), 2u * 128u * (uint32_t)prm.M);
      tma_load_4d(sb + kOffQd, &tm_q, 0, g * a.G, 0, b, bar(DBAR_Q));
      tma_load_4d(sb + kOffQd + kQHalf, &tm_q, 64, g * a.G, 0, b, bar(DBAR_Q));
    }
    // page-table entries of this split, 32 at a time, one per lane, the next
    // window already loading
    int wb = 0, cur = win_cur, nxt = win_nxt;
    int issued = 0;
    bool bad = false;
    for (int i = 0; i < nb; ++i) {
      const int s = i % kDecStages;
      if (i >= kDecStages) {
        // wait for the four compute warps to release the stage (bounded)
        bool ok = true;
        if (lane == 0) ok = wait_bar(bar(DBAR_EMPTY + s), (uint32_t)((i / kDecStages - 1) & 1), abort_flag, a.err);
        if (!__shfl_sync(kAll, ok ? 1 : 0, 0)) break;
      }
      const uint32_t dst = sb + kOffStage + s * kStageBytes;
      const uint32_t full = bar(DBAR_FULL + s);
      if (i < npg) {
        while (i >= wb + 32) { wb += 32; cur = nxt; nxt = load_win(wb + 32); }
        const int page = __shfl_sync(kAll, cur, i - wb);
        const bool ok = page >= 0 && page < a.num_pages;
        if (!ok) bad = true;
        if (lane == 0) {
          stage_bad[s] = ok ? 0 : 1;     // published by the arrive below
          if (ok) {
            mbar_expect_tx(full, kStageBytes);
            const int row = (page * a.Hkv + g) * 64;
            tma_load_2d(dst, &tm_kp, 0, row, full);
            tma_load_2d(dst + kHalfPage, &tm_kp, 64, row, full);
            tma_load_2d(dst + kPageBytes, &tm_vp, 0, row, full);
            tma_load_2d(dst + kPageBytes + kHalfPage, &tm_vp, 64, row, full);
          } else {
            mbar_arrive(full);           // nothing to copy: the consumers mask the page
          }
        }
      } else if (lane == 0) {
        mbar_expect_tx(full, kStageBytes);
        tma_load_4d(dst, &tm_ks, 0, g, 0, b, full);
        tma_load_4d(dst + kHalfPage, &tm_ks, 64, g, 0, b, full);
        tma_load_4d(dst + kPageBytes, &tm_vs, 0, g, 0, b, full);
        tma_load_4d(dst + kPageBytes + kHalfPage, &tm_vs, 64, g, 0, b, full);
      }
      issued = i + 1;
      if (i == 0 && lane == 0) DEC_TRACE(2);
    }
    if (lane == 0) {
      if (bad) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
      if (*abort_flag) {
        // drain: no copy may still write shared memory when the CTA exits
        for (int i = max(0, issued - kDecStages); i < issued; ++i)
          wait_quiet(bar(DBAR_FULL + i % kDecStages), (uint32_t)((i / kDecStages) & 1));
        wait_quiet(bar(DBAR_Q), 0);
      }
    }
  } else {
    // ---------------------------------------------------------------- compute
    const int cw = (warp - 1) & 3;                // keys [16cw, 16cw+16) of every page of its group
    const int grp = (warp - 1) >> 2;              // pages i with i % 2 == grp
    const int wid = warp - 1;                     // 0..7
    const int gq = lane >> 2, cq = lane & 3;      // fragment row group and column pair
    const float sl2 = prm.scale_log2;
    // the two query rows this lane's fragments hold, and their zone masks
    const int r0 = gq, r1 = gq + 8;
    const StepVis vis0 = step_visibility(a.k, min(r0 / a.G, a.R - 1));
    const StepVis vis1 = step_visibility(a.k, min(r1 / a.G, a.R - 1));
    bool ok = warp_wait_bar(bar(DBAR_Q), 0, abort_flag, a.err);
    if (wid == 0 && lane == 0) DEC_TRACE(3);
    uint32_t qa[8][4];
    {
      const int j = lane >> 3, rr = lane & 7;
      const int row = rr + (j & 1) * 8;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int d = 16 * kk + (j >> 1) * 8;
        ldsm_x4(sw128(sb + kOffQd + (d >> 6) * kQHalf, row, (d & 63) >> 3), qa[kk][0], qa[kk][1], qa[kk][2],
                qa[kk][3]);
      }
    }
    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    for (int i = grp; ok && i < nb; i += 2) {
      const int s = i % kDecStages;
      if (!warp_wait_bar(bar(DBAR_FULL + s), (uint32_t)((i / kDecStages) & 1), abort_flag, a.err)) {
        ok = false;
        break;
      }
      if (cw == 0 && lane == 0 && i < 64) DEC_TRACE(16 + i);
      const uint32_t kb = sb + kOffStage + s * kStageBytes, vb = kb + kPageBytes;
      const bool window = i >= npg;
      // valid keys of this page among the warp's 16: prefix keys below kend on
      // a mapped page; window keys below R (the zone mask is per row, below)
      int nvalid = 16;
      if (!window) {
        const int key0 = k0 + 64 * i;
        nvalid = stage_bad[s] ? 0 : max(0, min(16, kend - key0 - 16 * cw));
      } else {
        nvalid = max(0, min(16, a.R - 16 * cw));
      }
      if (nvalid < 16) {
        // keys past the end (or on an unmapped page): zero their V rows so that
        // 0 * (whatever the stage holds) cannot turn into NaN
        for (int idx = lane; idx < 16 * 16; idx += 32) {
          const int kr = idx >> 4, piece = idx & 15;
          if (kr >= nvalid) {
            const int row = 16 * cw + kr;
            *reinterpret_cast<uint4*>(smem + (vb - sb) + (piece >> 3) * kHalfPage + row * 128 + (piece & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        __syncwarp();
      }
      // S = Q K^T for the warp's 16 keys (two n-tiles of 8); even and odd
      // dimension chunks accumulate separately to halve the dependent chain
      float sc[2][4], sd[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[t][e] = sd[t][e] = 0.f;
      {
        const int j = lane >> 3, rr = lane & 7;
        const int key = 16 * cw + (j >> 1) * 8 + rr;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int d = 16 * kk + (j & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sw128(kb + (d >> 6) * kHalfPage, key, (d & 63) >> 3), b0, b1, b2, b3);
          if (kk & 1) {
            mma16816(sd[0], qa[kk], b0, b1);
            mma16816(sd[1], qa[kk], b2, b3);
          } else {
            mma16816(sc[0], qa[kk], b0, b1);
            mma16816(sc[1], qa[kk], b2, b3);
          }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[t][e] += sd[t][e];
      }
      // mask, scale to the log2 domain, online softmax (stale base up to 2^8)
      float x[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kl = 8 * t + 2 * cq + (e & 1);          // key within the warp's 16
          bool v = kl < nvalid;
          if (window) v = v && step_visible(e < 2 ? vis0 : vis1, 16 * cw + kl);
          x[t][e] = v ? sc[t][e] * sl2 : -INFINITY;
        }
      float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
      float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const bool up0 = n0 > m0 + 8.0f, up1 = n1 > m1 + 8.0f;
      if (__any_sync(0xffffffffu, up0 || up1)) {
        const float f0 = up0 ? ex2(m0 - n0) : 1.0f, f1 = up1 ? ex2(m1 - n1) : 1.0f;   // m = -inf -> 0
        if (up0) m0 = n0;
        if (up1) m1 = n1;
        l0 *= f0;
        l1 *= f1;
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          o[n][0] *= f0; o[n][1] *= f0;
          o[n][2] *= f1; o[n][3] *= f1;
        }
      }
      const float b0s = m0 == -INFINITY ? 0.f : m0, b1s = m1 == -INFINITY ? 0.f : m1;
      float p[2][4];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        p[t][0] = ex2(x[t][0] - b0s);
        p[t][1] = ex2(x[t][1] - b0s);
        p[t][2] = ex2(x[t][2] - b1s);
        p[t][3] = ex2(x[t][3] - b1s);
        l0 += p[t][0] + p[t][1];
        l1 += p[t][2] + p[t][3];
      }
      // the score fragments, as bf16, are the A fragment of P (16 x 16 keys)
      const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), pack_bf16(p[0][2], p[0][3]),
                              pack_bf16(p[1][0], p[1][1]), pack_bf16(p[1][2], p[1][3])};
      // O += P V: sixteen n-tiles of 8 dims, V fragments by transposed ldmatrix
      {
        const int j = lane >> 3, rr = lane & 7;
        const int key = 16 * cw + (j & 1) * 8 + rr;
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          const int d = 16 * np + (j >> 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sw128(vb + (d >> 6) * kHalfPage, key, (d & 63) >> 3), b0, b1, b2, b3);
          mma16816(o[2 * np], pa, b0, b1);
          mma16816(o[2 * np + 1], pa, b2, b3);
        }
      }
      // the stage's shared memory has been read into registers: release it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(DBAR_EMPTY + s));
      if (cw == 0 && lane == 0 && i < 64) DEC_TRACE(80 + i);
    }
    if (wid == 0 && lane == 0) DEC_TRACE(150);
    // ---- merge the eight warps: (max, sum, O) per row through shared memory
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    asm volatile("bar.sync 1, 256;" ::: "memory");       // every compute warp is past its last stage
    // [8 warps][16 rows][kXo] fp32: rows padded to 136 floats so the eight row
    // groups of a fragment store land on distinct banks
    constexpr int kXo = 136;
    float* xo = reinterpret_cast<float*>(smem + kOffStage);
    float* xm = xo + kDecCompute * 16 * kXo;                             // [8][16] max
    float* xl = xm + kDecCompute * 16;                                   // [8][16] sum
    int* xk = reinterpret_cast<int*>(xl + kDecCompute * 16);             // [8] status
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      const int col = 8 * n + 2 * cq;
      *reinterpret_cast<float2*>(xo + (wid * 16 + r0) * kXo + col) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2*>(xo + (wid * 16 + r1) * kXo + col) = make_float2(o[n][2], o[n][3]);
    }
    if (cq == 0) {
      xm[wid * 16 + r0] = m0; xm[wid * 16 + r1] = m1;
      xl[wid * 16 + r0] = l0; xl[wid * 16 + r1] = l1;
    }
    if (lane == 0) xk[wid] = ok ? 1 : 0;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    // thread -> (row, 8 columns)
    const int t = threadIdx.x - 32;
    const int row = t >> 4, c0 = (t & 15) * 8;
    bool all_ok = true;
#pragma unroll
    for (int w = 0; w < kDecCompute; ++w) all_ok = all_ok && xk[w];
    float* cpo = reinterpret_cast<float*>(smem + kOffCpo);
    float* cpl = reinterpret_cast<float*>(smem + kOffCpl);
    if (prm.cluster && row < 16 && c0 == 0) cpl[row] = -INFINITY;   // overwritten below when valid
    if (row < prm.M && all_ok) {
      float mt = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) mt = fmaxf(mt, xm[w * 16 + row]);
      float f[kDecCompute], lt = 0.f;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) {
        const float mw = xm[w * 16 + row];
        f[w] = mw == -INFINITY ? 0.f : ex2(mw - mt);
        lt += f[w] * xl[w * 16 + row];
      }
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) {
        const float4 x0 = *reinterpret_cast<const float4*>(xo + (w * 16 + row) * kXo + c0);
        const float4 x1 = *reinterpret_cast<const float4*>(xo + (w * 16 + row) * kXo + c0 + 4);
        v[0] += f[w] * x0.x; v[1] += f[w] * x0.y; v[2] += f[w] * x0.z; v[3] += f[w] * x0.w;
        v[4] += f[w] * x1.x; v[5] += f[w] * x1.y; v[6] += f[w] * x1.z; v[7] += f[w] * x1.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= inv;
      const float lse = lt > 0.f ? (mt + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      const int rho = row / a.G, h = g * a.G + row % a.G;
      const size_t orow = (size_t)(b * a.R + rho) * a.Hq + h;
      if (prm.cluster) {
        *reinterpret_cast<float4*>(cpo + row * 128 + c0) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(cpo + row * 128 + c0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
        if (c0 == 0) cpl[row] = lse;
      } else if (a.nsplit == 1) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + orow * 128 + c0;
        uint4 u;
        u.x = pack_bf16(v[0], v[1]); u.y = pack_bf16(v[2], v[3]);
        u.z = pack_bf16(v[4], v[5]); u.w = pack_bf16(v[6], v[7]);
        *reinterpret_cast<uint4*>(dst) = u;
        if (c0 == 0 && a.lse_out) a.lse_out[orow] = lse;
      } else {
        const size_t prow = (size_t)split * a.B * a.R * a.Hq + orow;
        float4* dst = reinterpret_cast<float4*>(a.part_o + prow * 128 + c0);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        if (c0 == 0) a.part_lse[prow] = lse;
      }
    }
  }

  if (prm.cluster) {
    // ---------------------------------------------------------------- split merge
    // The CTAs of this cluster are the key splits of one (b, g).  CTA `rank`
    // merges rows rank, rank + nsplit, ... of the M packed rows from every
    // split's result over distributed shared memory; one warp per row, one
    // lane per four columns.
    cluster_sync_all();
    const int ns = a.nsplit;
    const uint32_t rank = cluster_rank();
    const uint32_t cpo_s = sb + kOffCpo, cpl_s = sb + kOffCpl;
    const int R = (int)rank + ns * warp;
    if (R < prm.M) {
      float l2 = -INFINITY;
      if (lane < ns) l2 = ld_cluster_f32(mapa(cpl_s + 4u * R, (uint32_t)lane)) * 1.4426950408889634f;
      float mx = l2;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float w = (lane < ns && l2 != -INFINITY) ? ex2(l2 - mx) : 0.f;
      float wsum = w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s2 = 0; s2 < ns; ++s2) {
        const float ws = __shfl_sync(0xffffffffu, w, s2);
        if (ws != 0.f) {
          const float4 x = ld_cluster_f32x4(mapa(cpo_s + 4u * (R * 128 + 4 * lane), (uint32_t)s2));
          acc.x = fmaf(ws, x.x, acc.x); acc.y = fmaf(ws, x.y, acc.y);
          acc.z = fmaf(ws, x.z, acc.z); acc.w = fmaf(ws, x.w, acc.w);
        }
      }
      const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
      const int rho = R / a.G, h = g * a.G + R % a.G;
      const size_t orow = (size_t)(b * a.R + rho) * a.Hq + h;
      uint2 u;
      u.x = pack_bf16(acc.x * inv, acc.y * inv);
      u.y = pack_bf16(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + orow * 128 + 4 * lane) = u;
      if (lane == 0 && a.lse_out)
        a.lse_out[orow] = wsum > 0.f ? (mx + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
    }
    cluster_sync_all();   // no CTA leaves while another may still read its shared memory
  }

  if (split == 0 && len_ok && !a.part_o) {
    // ---------------------------------------------------------------- append
    // Draft rows D_1..D_n of KV head g into cache rows P .. P+n-1 (the step
    // keys above were read from k_blk / v_blk, not from the cache).
    const int32_t* tb = a.page_table + (size_t)b * a.max_pages;
    for (int c = threadIdx.x; c < a.n * 2 * 16; c += kDecThreads) {
      const int r = c >> 5, which = (c >> 4) & 1, piece = c & 15;
      const int pos = P + r;
      const int page = tb[pos / 64];
      if (page < 0 || page >= a.num_pages) {
        if (piece == 0 && which == 0) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
        continue;
      }
      const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(which ? a.v_blk : a.k_blk) +
                                 ((size_t)(b * a.R + r) * a.Hkv + g) * 128 + piece * 8;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(const_cast<void*>(which ? a.v_pages : a.k_pages)) +
                           ((size_t)(page * a.Hkv + g) * 64 + pos % 64) * 128 + piece * 8;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
  if (threadIdx.x == 32) { DEC_TRACE(151); DEC_TRACE_CTA(1); }
}

// The kernel's dynamic shared memory opt-in, once per device.
cudaError_t dec_smem_attr() {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(attn_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_dec_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_dec_trace, bytes);
}
#endif

int dec_resident_clusters(int ns) {
  static int cache[64][kMaxCluster + 1];
  if (ns < 1 || ns > kMaxCluster) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev][ns]) return cache[dev][ns] - 1;
  int n = 0;
  if (dec_smem_attr() == cudaSuccess &&
      (ns <= 8 || cudaFuncSetAttribute(attn_dec_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ns, 1, 1);
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = kDecSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = ns;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_dec_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache[dev][ns] = n + 1;
  return n;
}

cudaError_t launch_attn_dec(const AttnArgs& a, cudaStream_t s) {
  const int M = a.R * a.G;
  if (!a.bf16 || a.D != 128 || a.page_size != 64 || M > 16 || a.keys_per_split % 64) return cudaErrorNotSupported;
  DecParams prm;
  prm.a = a;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.M = M;
  prm.cluster = a.nsplit > 1 && !a.part_o;
  if (prm.cluster && a.nsplit > kMaxCluster) return cudaErrorNotSupported;
  CUtensorMap tq, tkp, tvp, tks, tvs;
  {
    const cuuint64_t dims[4] = {128, (cuuint64_t)a.Hq, (cuuint64_t)a.R, (cuuint64_t)a.B};
    const cuuint64_t str[3] = {256, (cuuint64_t)a.Hq * 256, (cuuint64_t)a.R * a.Hq * 256};
    const cuuint32_t box[4] = {64, (cuuint32_t)a.G, (cuuint32_t)a.R, 1};
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
    const cuuint32_t box[4] = {64, 1, 64, 1};
    if (!encode(&tks, a.k_blk, 4, dims, str, box)) return cudaErrorNotSupported;
    if (!encode(&tvs, a.v_blk, 4, dims, str, box)) return cudaErrorNotSupported;
  }
  cudaError_t e = dec_smem_attr();
  if (e != cudaSuccess) return e;
  return launch_clustered(attn_dec_kernel, dim3(a.nsplit, a.B * a.Hkv), dim3(prm.cluster ? a.nsplit : 1, 1, 1),
                          kDecThreads, kDecSmem, s, tq, tkp, tvp, tks, tvs, prm);
}

}  // namespace tidar
