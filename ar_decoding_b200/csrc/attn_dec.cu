// attn_dec.cu -- warp-MMA step attention for small query blocks (sm_100a).
//
// The same three-zone step attention as the other kernels ("TiDAR: Think in
// Diffusion, Talk in Autoregression", mauroscia.it section 2; nodesdaily.com
// (fr), paragraphs on the three zones and the masking puzzle), for steps whose
// query block packs into at most 16 rows per KV head (R * G <= 16: plain
// decode with k = 0, and k = 1 with G <= 8).  Such a block is far too thin for
// the 128-row tcgen05 tiles and the step is a stream of the paged KV cache,
// so this kernel is built to keep HBM busy: one TMA producer warp keeps a
// 6-stage ring of 64-key K/V pages (192 KB) in flight, and groups of four
// compute warps take pages in turn (three groups when the rows fit one 8-row
// MMA tile, two when they need two), each warp 16 keys of its page, with
// mma.sync m16n8k16 (bf16, fp32 accumulate) in transposed form so the query
// rows fill the N dimension: S^T = K Q^T, an online softmax in registers, P^T
// moved into the B-operand layout with movmatrix, O^T += V^T P^T.  The warps'
// (max, sum, O) merge in shared memory at the end; key splits merge on chip
// through a cluster when the wave's clusters fit, else through workspace
// partials and the finalize launch.
//
// Grid (split, b * Hkv); 32 * (1 + 4 * groups) threads (warp 0 producer).
// Every mbarrier wait is bounded (~1 s): on expiry the CTA records
// TIDAR_DEVERR_TIMEOUT, the producer drains the copies it issued, and the CTA
// exits.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tidar {

namespace {

// NT = number of 8-row query tiles (1: M <= 8, 2: M <= 16).  Compute warps come
// in page groups of four (one per 16-key quarter of a page); NT = 1 leaves
// room in the register file for three groups, NT = 2 for two.
template <int NT> struct DecShape {
  static constexpr int kGroups = NT == 1 ? 3 : 2;
  static constexpr int kCompute = 4 * kGroups;
  static constexpr int kThreads = 32 * (1 + kCompute);
};
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
constexpr int DBAR_MERGE = 1 + 2 * kDecStages;          // split merge: one arrival per CTA of the cluster
constexpr int kDecBars = 2 + 2 * kDecStages;
constexpr uint32_t kOffMiscD = kOffBarD + kDecBars * 8;  // [0] abort flag, [1 + s] stage s holds no page
// Split-merge receive area of a row-owning CTA, apart from every buffer that
// is still in use while other CTAs push into it: normalised partial O rows
// [nsplit][ceil(M / nsplit) slots][128] fp32 (at most 30 rows for M, nsplit
// <= 16) and their lse.  Row R is merged by CTA R % nsplit in slot R / nsplit.
constexpr int kRecvRows = 30;
constexpr uint32_t kOffRecv = (kOffMiscD + 4 * (1 + kDecStages) + 15u) & ~15u;
constexpr uint32_t kOffRecvL = kOffRecv + kRecvRows * 128 * 4;
constexpr uint32_t kDecSmem = kOffRecvL + kRecvRows * 4;
static_assert(kDecSmem <= 232448, "shared memory budget");

// Optional timeline (build with -DTIDAR_TRACE; absent from normal builds):
// CTA (0, 0): [0] setup done, [1] prefix length read, [2] first copy issued,
// [3] Q seen by compute warp 1, [16+i] page i seen by warp 1, [80+i] page i
// done by warp 1, [150] merge start, [151] end; [256 + 2*cta] start / end of
// every CTA.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_dec_trace[256 + 2 * 4096 + 4096];   // + per-CTA pages-done time
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
// Transpose of an 8x8 matrix of 16-bit elements held as one fragment register
// per lane (row lane/4, columns 2*(lane%4) and +1).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
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

template <int NT>
__global__ void __launch_bounds__(DecShape<NT>::kThreads, 1)
attn_dec_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                const __grid_constant__ CUtensorMap tm_vs, const DecParams prm) {
  constexpr int kDecThreads = DecShape<NT>::kThreads;
  constexpr int kDecCompute = DecShape<NT>::kCompute;
  constexpr int kGroups = DecShape<NT>::kGroups;
  constexpr int kRows = 8 * NT;                 // query rows held by the MMA tiles
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const AttnArgs& a = prm.a;
  if (sb & 1023u) {        // 128-byte swizzled tiles need 1024-byte alignment: refuse, never misread
    if (threadIdx.x == 0) raise_error(a.err, TIDAR_DEVERR_LAYOUT);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int g = blockIdx.y % a.Hkv;
  auto bar = [&](int i) -> uint32_t { return sb + kOffBarD + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMiscD);
  volatile int* stage_bad = abort_flag + 1;

  // Q rows M..15 of the tile stay zero (the copy writes rows 0..M-1)
  for (int i = threadIdx.x; i < 4096 / 16; i += kDecThreads)
    reinterpret_cast<uint4*>(smem + kOffQd)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecBars; ++i)
      mbar_init(bar(i), i == DBAR_MERGE ? (uint32_t)a.nsplit : (i >= DBAR_EMPTY ? 4u : 1u));
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tm_q);      // kernel parameters: safe before the dependency wait
    prefetch_tmap(&tm_kp);
    prefetch_tmap(&tm_vp);
    prefetch_tmap(&tm_ks);
    prefetch_tmap(&tm_vs);
    const int bq = blockIdx.y / a.Hkv;
    prefetch_l2(a.seq_lens + bq, 4, 0, 1);
    const int pgq = blockIdx.x * a.keys_per_split / 64;
    if (pgq < a.max_pages)
      prefetch_l2(a.page_table + (size_t)bq * a.max_pages + pgq, min(256, 4 * (a.max_pages - pgq)), 0, 1);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  // Split cluster: every CTA is running and has initialised its merge barrier
  // before anyone pushes to it (the matching wait comes after the key sweep).
  if (prm.cluster) asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  if (threadIdx.x == 0) { DEC_TRACE_CTA(0); DEC_TRACE(0); }

  pdl_wait();       // the previous kernel on the stream is complete from here on
  pdl_trigger();
  // longest sequences first (ragged batches of up to 32 sequences)
  const int b = longest_first(a.seq_lens, a.B, (int)blockIdx.y / a.Hkv);

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
  const int nb = npg + ((last && a.step_keys) ? 1 : 0);   // + the step-key window (R <= 16 keys)

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
    // Transposed formulation, query rows in the MMA N dimension:
    //   S^T (16 keys x 8 rows) = K (16 keys x 16 dims) . Q^T, eight dim chunks;
    //   O^T (16 dims x 8 rows) += V^T (16 dims x 16 keys) . P^T, eight dim tiles.
    // A lane holds rows 8nt + 2cq and + 1 of each n-tile nt, keys gq and gq + 8
    // of its warp's 16 (S^T fragment), and dims 16mt + gq, + 8 of O^T.
    const int wid = warp - 1;                     // 0 .. kDecCompute - 1
    const int cw = wid & 3;                       // keys [16cw, 16cw+16) of every page of its group
    const int grp = wid >> 2;                     // pages i with i % kGroups == grp
    const int gq = lane >> 2, cq = lane & 3;
    const float sl2 = prm.scale_log2;
    StepVis vis[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) vis[nt][h] = step_visibility(a.k, min((8 * nt + 2 * cq + h) / a.G, a.R - 1));
    bool ok = warp_wait_bar(bar(DBAR_Q), 0, abort_flag, a.err);
    if (wid == 0 && lane == 0) DEC_TRACE(3);
    // Q^T as the B operand: qb[kk][nt] = {dims 16kk + 2cq.., dims 16kk + 8 + 2cq..} of row 8nt + gq
    uint32_t qb[8][NT][2];
    {
      const int j = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < 8; kk += 2) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          // matrices: (rows 8nt.., dims 16kk), (.., 16kk+8), (.., 16(kk+1)), (.., 16(kk+1)+8)
          const int d = 16 * kk + j * 8;
          ldsm_x4(sw128(sb + kOffQd + (d >> 6) * kQHalf, 8 * nt + rr, (d & 63) >> 3), qb[kk][nt][0],
                  qb[kk][nt][1], qb[kk + 1][nt][0], qb[kk + 1][nt][1]);
        }
      }
    }
    float o[8][NT][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = -INFINITY, l[nt][0] = l[nt][1] = 0.f;
    for (int i = grp; ok && i < nb; i += kGroups) {
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
      // S^T = K Q^T: even and odd dim chunks accumulate separately (shorter
      // dependent chains)
      float sc[NT][4], sd[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = sd[nt][e] = 0.f;
      {
        const int j = lane >> 3, rr = lane & 7;
        const int key = 16 * cw + (j & 1) * 8 + rr;   // matrices: keys 0-7 / 8-15 x dims +0 / +8
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int d = 16 * kk + (j >> 1) * 8;
          uint32_t ka[4];
          ldsm_x4(sw128(kb + (d >> 6) * kHalfPage, key, (d & 63) >> 3), ka[0], ka[1], ka[2], ka[3]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            if (kk & 1) mma16816(sd[nt], ka, qb[kk][nt][0], qb[kk][nt][1]);
            else mma16816(sc[nt], ka, qb[kk][nt][0], qb[kk][nt][1]);
          }
        }
      }
      // mask, log2-domain scale, online softmax per row (stale base up to 2^8)
      float x[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kl = gq + (e >> 1) * 8;             // key within the warp's 16
          bool v = kl < nvalid;
          if (window) v = v && step_visible(vis[nt][e & 1], 16 * cw + kl);
          x[nt][e] = v ? (sc[nt][e] + sd[nt][e]) * sl2 : -INFINITY;
        }
      float f[NT][2];
      bool any_up = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float mx = fmaxf(x[nt][h], x[nt][h + 2]);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float nm = fmaxf(m[nt][h], mx);
          const bool up = nm > m[nt][h] + 8.0f;
          f[nt][h] = up ? ex2(m[nt][h] - nm) : 1.0f;      // m = -inf -> 0
          if (up) m[nt][h] = nm;
          any_up = any_up || up;
        }
      if (__any_sync(0xffffffffu, any_up)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          l[nt][0] *= f[nt][0];
          l[nt][1] *= f[nt][1];
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            o[mt][nt][0] *= f[nt][0]; o[mt][nt][1] *= f[nt][1];
            o[mt][nt][2] *= f[nt][0]; o[mt][nt][3] *= f[nt][1];
          }
        }
      }
      // P^T, transposed in registers into the B operand of the PV MMA
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const float b0s = m[nt][0] == -INFINITY ? 0.f : m[nt][0];
        const float b1s = m[nt][1] == -INFINITY ? 0.f : m[nt][1];
        const float p0 = ex2(x[nt][0] - b0s), p1 = ex2(x[nt][1] - b1s);
        const float p2 = ex2(x[nt][2] - b0s), p3 = ex2(x[nt][3] - b1s);
        l[nt][0] += p0 + p2;
        l[nt][1] += p1 + p3;
        pb[nt][0] = movmatrix_t(pack_bf16(p0, p1));     // keys 0-7 of the warp's 16
        pb[nt][1] = movmatrix_t(pack_bf16(p2, p3));     // keys 8-15
      }
      // O^T += V^T P^T: eight 16-dim tiles, V^T fragments by transposed ldmatrix
      {
        const int j = lane >> 3, rr = lane & 7;
        const int key = 16 * cw + (j >> 1) * 8 + rr;   // matrices: (keys 0-7, dims +0 / +8), (keys 8-15, ..)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int d = 16 * mt + (j & 1) * 8;
          uint32_t va[4];
          ldsm_x4_t(sw128(vb + (d >> 6) * kHalfPage, key, (d & 63) >> 3), va[0], va[1], va[2], va[3]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma16816(o[mt][nt], va, pb[nt][0], pb[nt][1]);
        }
      }
      // the stage's shared memory has been read into registers: release it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(DBAR_EMPTY + s));
      if (cw == 0 && lane == 0 && i < 64) DEC_TRACE(80 + i);
    }
    if (wid == 0 && lane == 0) DEC_TRACE(150);
#ifdef TIDAR_TRACE
    if (wid == 0 && lane == 0) {
      const unsigned c_ = blockIdx.x + gridDim.x * blockIdx.y;
      if (c_ < 4096) g_dec_trace[256 + 2 * 4096 + c_] = global_ns();
    }
#endif
    // ---- merge the compute warps: (max, sum, O) per row through shared memory
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        l[nt][h] += __shfl_xor_sync(0xffffffffu, l[nt][h], 4);
        l[nt][h] += __shfl_xor_sync(0xffffffffu, l[nt][h], 8);
        l[nt][h] += __shfl_xor_sync(0xffffffffu, l[nt][h], 16);
      }
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecCompute) : "memory");   // every compute warp is past its last stage
    // [warps][kRows rows][kXo] fp32, rows padded to 136 floats against bank conflicts
    constexpr int kXo = 136;
    float* xo = reinterpret_cast<float*>(smem + kOffStage);
    float* xm = xo + kDecCompute * kRows * kXo;                        // [warps][kRows] max
    float* xl = xm + kDecCompute * kRows;                              // [warps][kRows] sum
    int* xk = reinterpret_cast<int*>(xl + kDecCompute * kRows);        // [warps] status
    // only the M real rows are merged (rows past M are tile padding)
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int r0 = 8 * nt + 2 * cq, d0 = 16 * mt + gq;
        if (r0 < prm.M) {
          xo[(wid * kRows + r0) * kXo + d0] = o[mt][nt][0];
          xo[(wid * kRows + r0) * kXo + d0 + 8] = o[mt][nt][2];
        }
        if (r0 + 1 < prm.M) {
          xo[(wid * kRows + r0 + 1) * kXo + d0] = o[mt][nt][1];
          xo[(wid * kRows + r0 + 1) * kXo + d0 + 8] = o[mt][nt][3];
        }
      }
    if (gq == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          xm[wid * kRows + 8 * nt + 2 * cq + h] = m[nt][h];
          xl[wid * kRows + 8 * nt + 2 * cq + h] = l[nt][h];
        }
    }
    if (lane == 0) xk[wid] = ok ? 1 : 0;
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kDecCompute) : "memory");
    // thread -> (row, 8 columns)
    const int t = threadIdx.x - 32;
    const int row = t >> 4, c0 = (t & 15) * 8;
    bool all_ok = true;
#pragma unroll
    for (int w = 0; w < kDecCompute; ++w) all_ok = all_ok && xk[w];
    if (prm.cluster) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    const int nsp = a.nsplit;
    const uint32_t rank = prm.cluster ? cluster_rank() : 0u;
    const int slots = (prm.M + nsp - 1) / nsp;        // rows owned per CTA
    auto recv_addr = [&](int r) -> uint32_t {          // row r's slot for this split in its owner CTA
      return mapa(sb + kOffRecv + 4u * (((uint32_t)rank * slots + (uint32_t)(r / nsp)) * 128u), (uint32_t)(r % nsp));
    };
    auto recvl_addr = [&](int r) -> uint32_t {
      return mapa(sb + kOffRecvL + 4u * ((uint32_t)rank * slots + (uint32_t)(r / nsp)), (uint32_t)(r % nsp));
    };
    if (prm.cluster && row < prm.M && c0 == 0 && !all_ok) {
      const float ninf = -INFINITY;                   // this split contributes nothing
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(recvl_addr(row)), "f"(ninf) : "memory");
    }
    if (row < prm.M && all_ok) {
      float mtop = -INFINITY;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) mtop = fmaxf(mtop, xm[w * kRows + row]);
      float fw[kDecCompute], lt = 0.f;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) {
        const float mw = xm[w * kRows + row];
        fw[w] = mw == -INFINITY ? 0.f : ex2(mw - mtop);
        lt += fw[w] * xl[w * kRows + row];
      }
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll
      for (int w = 0; w < kDecCompute; ++w) {
        const float4 x0 = *reinterpret_cast<const float4*>(xo + (w * kRows + row) * kXo + c0);
        const float4 x1 = *reinterpret_cast<const float4*>(xo + (w * kRows + row) * kXo + c0 + 4);
        v[0] += fw[w] * x0.x; v[1] += fw[w] * x0.y; v[2] += fw[w] * x0.z; v[3] += fw[w] * x0.w;
        v[4] += fw[w] * x1.x; v[5] += fw[w] * x1.y; v[6] += fw[w] * x1.z; v[7] += fw[w] * x1.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] *= inv;
      const float lse = lt > 0.f ? (mtop + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      const int rho = row / a.G, h = g * a.G + row % a.G;
      const size_t orow = (size_t)(b * a.R + rho) * a.Hq + h;
      if (prm.cluster) {
        // push this split's normalised row slice and lse to the row's owner
        const uint32_t dst = recv_addr(row) + 4u * c0;
        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "f"(v[0]), "f"(v[1]),
                     "f"(v[2]), "f"(v[3])
                     : "memory");
        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 16u), "f"(v[4]), "f"(v[5]),
                     "f"(v[6]), "f"(v[7])
                     : "memory");
        if (c0 == 0) asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(recvl_addr(row)), "f"(lse) : "memory");
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
    // Every CTA of the cluster (the key splits of one (b, g)) has pushed its
    // rows into their owners; once all of a CTA's pushes are issued, one thread
    // arrives (release, cluster scope) on each owner's merge barrier.  Owners
    // (CTAs 0 .. min(nsplit, M) - 1) wait for all nsplit arrivals, merge their
    // rows from local shared memory and write O and lse; the other CTAs are
    // done: nothing reads their shared memory.
    const int ns = a.nsplit;
    const uint32_t rank = cluster_rank();
    if (threadIdx.x == 32) DEC_TRACE(152);
    __syncthreads();                                   // all of this CTA's pushes are issued
    if (threadIdx.x == 0) {
      asm volatile("fence.acq_rel.cluster;" ::: "memory");
      for (int o = 0; o < min(ns, prm.M); ++o)
        asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(mapa(bar(DBAR_MERGE), o))
                     : "memory");
    }
    if ((int)rank < min(ns, prm.M)) {
      const int slots = (prm.M + ns - 1) / ns;
      const int slot = warp;                           // one warp per owned row, one lane per 4 columns
      const int R = (int)rank + ns * slot;
      if (slot < slots && R < prm.M) {
        bool ok = false;
        {
          const uint64_t t0 = global_ns();
          for (;;) {
            uint32_t done;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(done)
                : "r"(bar(DBAR_MERGE))
                : "memory");
            if (done) { ok = true; break; }
            if (global_ns() - t0 > kWaitLimitNs) break;
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          if (lane == 0) raise_error(a.err, TIDAR_DEVERR_TIMEOUT);
        } else {
          if (threadIdx.x == 32) DEC_TRACE(153);
          const float* rv = reinterpret_cast<const float*>(smem + kOffRecv);
          const float* rl = reinterpret_cast<const float*>(smem + kOffRecvL);
          float l2 = -INFINITY;
          if (lane < ns) l2 = rl[lane * slots + slot] * 1.4426950408889634f;
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
            // a split with weight 0 may have left its row unwritten: select, not multiply
            const float4 x = *reinterpret_cast<const float4*>(rv + (s2 * slots + slot) * 128 + 4 * lane);
            if (ws != 0.f) {
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
      }
    }
    if (threadIdx.x == 32) DEC_TRACE(154);
  }

  if (split == 0 && len_ok && (a.nsplit == 1 || a.cluster_merge) && a.append) {
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
template <int NT>
cudaError_t dec_smem_attr() {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(attn_dec_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return cudaSuccess;
}

template <int NT>
int resident_clusters_t(int ns) {
  static int cache[64][kMaxCluster + 1];
  if (ns < 1 || ns > kMaxCluster) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev][ns]) return cache[dev][ns] - 1;
  int n = 0;
  if (dec_smem_attr<NT>() == cudaSuccess &&
      (ns <= 8 || cudaFuncSetAttribute(attn_dec_kernel<NT>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ns, 1, 1);
    cfg.blockDim = dim3(DecShape<NT>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kDecSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = ns;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_dec_kernel<NT>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache[dev][ns] = n + 1;
  return n;
}

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_dec_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_dec_trace, bytes);
}
#endif

int dec_resident_clusters(int ns, int M) {
  return M <= 8 ? resident_clusters_t<1>(ns) : resident_clusters_t<2>(ns);
}

cudaError_t launch_attn_dec(const AttnArgs& a, cudaStream_t s) {
  const int M = a.R * a.G;
  if (!a.bf16 || a.D != 128 || a.page_size != 64 || M > 16 || a.keys_per_split % 64) return cudaErrorNotSupported;
  DecParams prm;
  prm.a = a;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.M = M;
  prm.cluster = a.nsplit > 1 && a.cluster_merge;
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
  const dim3 grid(a.nsplit, a.B * a.Hkv), cluster(prm.cluster ? a.nsplit : 1, 1, 1);
  if (M <= 8) {
    cudaError_t e = dec_smem_attr<1>();
    if (e != cudaSuccess) return e;
    return launch_clustered(attn_dec_kernel<1>, grid, cluster, DecShape<1>::kThreads, kDecSmem, s, tq, tkp, tvp,
                            tks, tvs, prm);
  }
  cudaError_t e = dec_smem_attr<2>();
  if (e != cudaSuccess) return e;
  return launch_clustered(attn_dec_kernel<2>, grid, cluster, DecShape<2>::kThreads, kDecSmem, s, tq, tkp, tvp, tks,
                          tvs, prm);
}

}  // namespace tidar
