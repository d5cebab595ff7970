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
// Roles (18 warps, 576 threads):
//   warp 0       TMA producer: Q tile once; per 128-key block two 64-row pages
//                of K and V (paged cache, SWIZZLE_128B) or one step-key window.
//                Separate 3-stage K and V rings.  No multicast.
//   warp 1       TMEM owner and MMA issuer (one thread):
//                S_t = Q K_b^T  (kind::f16, A and B from shared memory, fp32 in
//                TMEM), O_t += P V_b with P read from TMEM (bf16, written over
//                S_t) and V as an MN-major operand.  Blocks alternate between
//                two softmax sets (t = b & 1), each with its own S_t and O_t, so
//                one set's exponentials overlap the other set's loads, maxima
//                and hand-offs.
//   warps 2..17  softmax: set 0 = warps 2..9, set 1 = warps 10..17.  Within a
//                set, the four warps of each half hf take TMEM lane quarter
//                warp % 4 (32 packed query rows each) and columns
//                [64 hf, 64 hf + 64) of the block: one thread holds half a row.
//                The two halves of a row swap their block maxima at a named
//                barrier; then tcgen05.ld of S, mask, online softmax in the
//                log2 domain, P back to TMEM as bf16 (each half over the first
//                32 columns of its own 64).  O_t is rescaled only when the
//                row maximum grows by more than 2^8.  The epilogue merges the
//                two sets and the two halves (max, sums, O) and writes O / l.
// Key splits of one (b, g, tile) either form one thread-block cluster and
// merge in this kernel (cluster_merge: each CTA stages its normalised rows in
// shared memory and owners read their peers' rows over distributed shared
// memory), or write fp32 partials to the workspace for a finalize launch.
// Every mbarrier wait is bounded: on expiry the CTA records TIDAR_DEVERR_TIMEOUT,
// stops issuing, drains what it issued (bounded), frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc05.cuh"

namespace tidar {

namespace {

constexpr int kThreads = 576;       // producer, MMA, 16 softmax warps
constexpr int kStages = 3;       // K/V ring depth; also the number of S buffers

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
constexpr int BAR_KEMPTY = 7;    // + stage: K stage free again (its S MMA is done)
constexpr int BAR_SFULL = 10;    // + S buffer
constexpr int BAR_PFULL = 13;    // + S buffer
constexpr int BAR_PVDONE = 16;   // + S buffer
constexpr int BAR_FINAL = 19;
constexpr int BAR_VEMPTY = 20;   // + stage: V stage free again (its PV MMA is done)
constexpr int kNumBars = 23;
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
// P (bf16, two keys per column) of keys [16kk, 16kk+16) within S_t: each softmax
// half writes the P of its 64 keys into the first 32 columns of its own 64 S
// columns, so the halves never overwrite scores the other half still reads.
__device__ __forceinline__ uint32_t p_col(int kk) { return kk < 4 ? 8u * kk : 64u + 8u * (kk - 4); }
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + 128u * (uint32_t)t; }

// kind::f16 instruction descriptors: fp32 accumulate, bf16 A and B, M = 128, N = 128.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);     // B (= V) is MN-major

struct Tc05Params {
  AttnArgs a;
  int rho_per_tile;   // query rows per tile (128 / G)
  int tiles;          // tiles per (b, g)
  float scale_log2;   // softmax scale * log2(e)
  int starve;         // test hook: issue no K/V copies (the waits for them run out)
};

int g_starve_loads = 0;   // tidar_debug_starve_attention_loads

// Optional timeline of one CTA and the start/end of every CTA (build with
// -DTIDAR_TRACE; absent from normal builds).  Slots: [0..15] setup, [16+i]
// producer issue of block i, [256+i] MMA sees K(i), [512+i] S(i) issued,
// [768+i] PV(i) issued, [1024+i] softmax sees S(i), [1280+i] P(i) handed over,
// [1536..] epilogue (1536 sets merged, 1538 O formed, 1539 partials stored,
// 1540 past the cluster barrier, 1541 merged, 1537 end), [2048 + 4*cta] CTA
// start / end / epilogue / past the cluster barrier.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_tidar_trace[2048 + 4 * 8192];
__device__ __forceinline__ bool trace_cta() { return blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0; }
#define TIDAR_TRACE_AT(slot) do { if (trace_cta()) g_tidar_trace[(slot)] = global_ns(); } while (0)
#define TIDAR_TRACE_PH(i, ph) do { if (((i) == 10 || (i) == 11) && lane == 0) TIDAR_TRACE_AT(1700 + 8 * warp + (ph)); } while (0)
#define TIDAR_TRACE_CTA(which) do { const unsigned cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (cta_ < 8192) g_tidar_trace[2048 + 4 * cta_ + (which)] = global_ns(); } while (0)
#else
#define TIDAR_TRACE_AT(slot) do {} while (0)
#define TIDAR_TRACE_PH(i, ph) do {} while (0)
#define TIDAR_TRACE_CTA(which) do {} while (0)
#endif

using namespace tc05;
static_assert((128 * kStageStride + 256) * 4 <= kStages * kTileBytes, "row staging fits the K ring");

// ------------------------------------------------------------------ the kernel
// 18 warps: two SMSPs host five of them, so a thread may hold at most
// 16384 / (5 * 32) -> 96 registers.
__global__ void __maxnreg__(96)
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
  // Set-up that reads nothing the previous kernel on the stream may write
  // (barriers, the tensor maps) runs before the dependency wait, so it
  // overlaps that kernel's tail.
  if (threadIdx.x == 0) {
    TIDAR_TRACE_CTA(0);
    TIDAR_TRACE_AT(0);
#ifdef TIDAR_TRACE
    if (trace_cta()) g_tidar_trace[2] = clock64();
#endif
    for (int i = 0; i < kNumBars; ++i) {
      const bool pfull = i >= BAR_PFULL && i < BAR_PFULL + kStages;
      mbar_init(sb + kOffBar + 8u * i, pfull ? 8u : 1u);
    }
    reinterpret_cast<volatile int*>(smem + kOffMisc)[1] = 0;     // abort flag
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kp);
    prefetch_tmap(&tm_vp);
    prefetch_tmap(&tm_ks);
    prefetch_tmap(&tm_vs);
    const int bq = blockIdx.z / prm.a.Hkv;
    prefetch_l2(prm.a.seq_lens + bq, 4, 0, 1);
    const int pgq = blockIdx.y * prm.a.keys_per_split / 64;   // the last split may start past the table
    if (pgq < prm.a.max_pages)
      prefetch_l2(prm.a.page_table + (size_t)bq * prm.a.max_pages + pgq, min(256, 4 * (prm.a.max_pages - pgq)), 0, 1);
  }
  pdl_wait();       // the previous kernel on the stream is complete from here on
  pdl_trigger();
  // longest sequences first (ragged batches of up to 32 sequences)
  const int b = longest_first(a.seq_lens, a.B, (int)blockIdx.z / a.Hkv);
  // The producer's first two 32-page windows of the page table do not depend on
  // the prefix length, so they load alongside it.
  int win_cur = -1, win_nxt = -1;
  if (warp == 0) {
    const int32_t* tb = a.page_table + (size_t)b * a.max_pages;
    const int pg = blockIdx.y * a.keys_per_split / 64;
    win_cur = pg + lane < a.max_pages ? tb[pg + lane] : -1;
    win_nxt = pg + 32 + lane < a.max_pages ? tb[pg + 32 + lane] : -1;
  }

  const int tile = blockIdx.x, split = blockIdx.y;
  const int g = blockIdx.z % a.Hkv;
  const int rho0 = tile * prm.rho_per_tile;
  const int rho1 = min(a.R, rho0 + prm.rho_per_tile);
  const int rows_valid = (rho1 - rho0) * a.G;

  int P = a.seq_lens[b];
  const bool len_ok = P >= 0 && P <= a.max_prefix;
  if (!len_ok) {
    if (threadIdx.x == 0 && tile == 0 && split == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    P = 0;
  }
  const BlockPlan bp = make_block_plan(a, P, split, rho0, rho1);
  const int32_t* table = a.page_table + (size_t)b * a.max_pages;

  auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  if (warp == 1) {      // every CTA holds TMEM (released at the end), keys or not
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

  // This CTA's share of the output, carried past the role branches: the
  // normalised partial O of 32 columns of one row and its log-sum-exp.
  float ov[32];
  float olse = -INFINITY;
  bool owrite = false;

  if (bp.nb == 0) {
    // This split holds no prefix keys of sequence b (only possible with
    // nsplit > 1): it contributes an empty partial (lse = -inf) to the merge.
  } else if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Separate K and V rings (3 stages each): a K stage is refilled as soon as
    // its S MMA is done, a V stage when its PV is done, so K runs up to three
    // blocks ahead of the scores.  The whole warp runs the loop (lane 0 issues);
    // the page-table entries of this split come from 32-page windows held one
    // entry per lane, with the next window already loading, so no issue waits
    // on a page-table read.
    constexpr unsigned kAll = 0xffffffffu;
    int k_phase[kStages] = {-1, -1, -1}, v_phase[kStages] = {-1, -1, -1};
    if (lane == 0) {
      mbar_expect_tx(bar(BAR_Q), 2u * 128u * (uint32_t)(prm.rho_per_tile * a.G));
      tma_load_4d(sb + kOffQ, &tm_q, 0, g * a.G, rho0, b, bar(BAR_Q));
      tma_load_4d(sb + kOffQ + kChunkBytes, &tm_q, 64, g * a.G, rho0, b, bar(BAR_Q));
    }
    const int pg0 = bp.k0 / 64;                                   // k0 is a multiple of 128
    auto load_win = [&](int base) -> int {
      const int pi = pg0 + base + lane;
      return pi < a.max_pages ? table[pi] : -1;
    };
    int kwb = 0, kcur = win_cur, knxt = win_nxt;
    int vwb = 0, vcur = kcur, vnxt = knxt;
    // table entry of relative page pi (warp-uniform, non-decreasing per ring)
    auto entry = [&](int& base, int& cur, int& nxt, int pi) -> int {
      while (pi >= base + 32) {
        base += 32;
        cur = nxt;
        nxt = load_win(base + 32);
      }
      return __shfl_sync(kAll, cur, pi - base);
    };
    bool bad = false;
    // one ring's tile of block i: two 64-row pages of the cache, or a window
    auto issue = [&](int i, bool is_v) {
      const int s = i % kStages;
      const uint32_t dst = sb + (is_v ? kOffV : kOffK) + s * kTileBytes;
      const uint32_t full = bar((is_v ? BAR_VFULL : BAR_KFULL) + s);
      if (i < bp.npb) {
        const CUtensorMap* map = is_v ? &tm_vp : &tm_kp;
        const int start = bp.k0 + i * 128;
        const bool need_b = start + 64 < bp.kend;
        const int pa = is_v ? entry(vwb, vcur, vnxt, 2 * i) : entry(kwb, kcur, knxt, 2 * i);
        const int pb = is_v ? entry(vwb, vcur, vnxt, 2 * i + 1) : entry(kwb, kcur, knxt, 2 * i + 1);
        const bool oka = page_ok(pa, a.num_pages), okb = need_b && page_ok(pb, a.num_pages);
        if (!oka || (need_b && !okb)) bad = true;
        if (lane == 0) {
          mbar_expect_tx(full, (uint32_t)(oka + okb) * 2u * 8192u);
          if (oka) {
            tma_load_2d(dst, map, 0, (pa * a.Hkv + g) * 64, full);
            tma_load_2d(dst + kChunkBytes, map, 64, (pa * a.Hkv + g) * 64, full);
          }
          if (okb) {
            tma_load_2d(dst + 8192, map, 0, (pb * a.Hkv + g) * 64, full);
            tma_load_2d(dst + kChunkBytes + 8192, map, 64, (pb * a.Hkv + g) * 64, full);
          }
        }
      } else if (lane == 0) {
        const CUtensorMap* map = is_v ? &tm_vs : &tm_ks;
        const int w = bp.wins[i - bp.npb];
        mbar_expect_tx(full, kTileBytes);
        tma_load_4d(dst, map, 0, g, w * 128, b, full);
        tma_load_4d(dst + kChunkBytes, map, 64, g, w * 128, b, full);
      }
      (is_v ? v_phase : k_phase)[s] = i / kStages;
    };
    // lane 0's view of a barrier phase / the abort flag, for the whole warp
    auto test_all = [&](uint32_t bar_addr, uint32_t parity) -> bool {
      const int t = lane == 0 ? (int)mbar_test(bar_addr, parity) : 0;
      return __shfl_sync(kAll, t, 0) != 0;
    };
    auto aborted = [&]() -> bool { return __shfl_sync(kAll, lane == 0 ? *abort_flag : 0, 0) != 0; };
    int ik = prm.starve ? bp.nb : 0, iv = ik;
    uint64_t last = global_ns();
    while ((ik < bp.nb || iv < bp.nb) && !aborted()) {
      bool progress = false;
      if (ik < bp.nb &&
          (ik < kStages || test_all(bar(BAR_KEMPTY + ik % kStages), (uint32_t)((ik / kStages - 1) & 1)))) {
        issue(ik, false);
        if (lane == 0) TIDAR_TRACE_AT(16 + min(ik, 239));
        ++ik;
        progress = true;
      }
      if (iv < ik &&
          (iv < kStages || test_all(bar(BAR_VEMPTY + iv % kStages), (uint32_t)((iv / kStages - 1) & 1)))) {
        issue(iv, true);
        ++iv;
        progress = true;
      }
      if (progress) {
        last = global_ns();
      } else {
        // sleep briefly on the ring that is further behind, then re-check both
        if (lane == 0) {
          if (ik < bp.nb && ik - iv < kStages)
            mbar_try_wait_ns(bar(BAR_KEMPTY + ik % kStages), (uint32_t)((ik / kStages - 1) & 1), 500u);
          else
            mbar_try_wait_ns(bar(BAR_VEMPTY + iv % kStages), (uint32_t)((iv / kStages - 1) & 1), 500u);
          if (global_ns() - last > kWaitLimitNs) {
            *abort_flag = 1;
            raise_error(a.err, TIDAR_DEVERR_TIMEOUT);
          }
        }
        __syncwarp();
      }
    }
    if (lane == 0) {
      if (bad) raise_error(a.err, TIDAR_DEVERR_BAD_PAGE);
      // Drain: on the normal path every load was consumed; after a timeout make
      // sure no copy is still writing shared memory when the CTA exits.
      if (*abort_flag) {
        for (int s2 = 0; s2 < kStages; ++s2) {
          if (k_phase[s2] >= 0) wait_quiet(bar(BAR_KFULL + s2), k_phase[s2] & 1);
          if (v_phase[s2] >= 0) wait_quiet(bar(BAR_VFULL + s2), v_phase[s2] & 1);
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
      // Operand descriptors: a descriptor's start-address field is the shared
      // address / 16 (below 2^14 here), so a tile at base + delta has the
      // descriptor of base plus delta / 16.  Q's eight are fixed; a stage's
      // K and V ones are its ring slot's base plus constants, formed ahead of
      // the eight-MMA asm blocks.
      uint64_t dq[8];
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) dq[kc] = desc_k_sw128(sb + kOffQ + (kc >> 2) * kChunkBytes + (kc & 3) * 32);
      const uint64_t dk0 = desc_k_sw128(sb + kOffK), dv0 = desc_mn_sw128(sb + kOffV, kChunkBytes);
      auto issue_s = [&](int blk) -> bool {
        const int st = blk % kStages, t = blk & 1;
        if (!wait_bar(bar(BAR_KFULL + st), (uint32_t)((blk / kStages) & 1), abort_flag, a.err)) return false;
        TIDAR_TRACE_AT(256 + min(blk, 255));
        fence_after();
        const uint64_t kbase = dk0 + (uint64_t)((st * kTileBytes) >> 4);
        uint64_t dk[8];
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) dk[kc] = kbase + (uint64_t)(((kc >> 2) * kChunkBytes + (kc & 3) * 32) >> 4);
        mma_ss_x8(tmem + col_s(t), dq, dk, kIdescS, 0u);
        mma_commit(bar(BAR_SFULL + t));
        mma_commit(bar(BAR_KEMPTY + st));
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
        const uint64_t vbase = dv0 + (uint64_t)((st * kTileBytes) >> 4);
        uint32_t pa[8];
        uint64_t dv[8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          pa[kk] = tmem + col_s(t) + p_col(kk);
          dv[kk] = vbase + (uint64_t)((kk * 2048) >> 4);
        }
        mma_ts_x8(tmem + col_o(t), pa, dv, kIdescPV, j > 0 ? 1u : 0u);
        mma_commit(bar(BAR_PVDONE + t));
        mma_commit(bar(BAR_VEMPTY + st));
        TIDAR_TRACE_AT(768 + min(b2, 255));
        if (b2 + 2 < bp.nb && !issue_s(b2 + 2)) break;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar(BAR_FINAL));
      wait_quiet(bar(BAR_FINAL), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    // Warps 2..17.  Set t (block parity) = (warp-2)/8 owns S_t and O_t; within a
    // set, half hf = ((warp-2)/4)&1 takes columns [64hf, 64hf+64) of the rows of
    // TMEM lane quarter warp%4.  One thread = one half row.  The two halves of a
    // row swap block maxima at a named barrier (id 1 + 4t + quarter, 64
    // threads); row sums and the two sets are merged in the epilogue.
    const int q4 = warp & 3;
    const int t = (warp - 2) >> 3;
    const int hf = ((warp - 2) >> 2) & 1;
    const int r = 32 * q4 + lane;
    const int rho_c = min(rho0 + r / a.G, a.R - 1);
    const StepVis vis = step_visibility(a.k, rho_c);
    const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
    const int gt = (warp - 2 - 8 * t) * 32 + lane;     // 0..255 within the set
    const bool live = 32 * q4 < rows_valid;             // the warp holds at least one real row
    const float sl2 = prm.scale_log2;
    const int nbt = (bp.nb - t + 1) >> 1;               // blocks of this set
    float* xmax = reinterpret_cast<float*>(smem + kOffRed);          // [2 set][2 half][128]
    int* xok = reinterpret_cast<int*>(smem + kOffOk);                // [2 set][2 half][4 quarter]
    const uint32_t pair_bar = 1 + 4 * t + q4;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nbt; ++j) {
      const int b2 = 2 * j + t;
      if (!warp_wait_bar(bar(BAR_SFULL + t), (uint32_t)(j & 1), abort_flag, a.err)) ok = false;
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
      uint32_t mw[4] = {~0u, ~0u, ~0u, ~0u};
      if (!full) block_mask(window, kb, vis, a.R, lo_valid, hi_valid, mw);
      const uint32_t scol = col_s(t) + 64 * hf;          // this half's 64 score columns
      // pass 1: maximum of this half's raw scores (the positive scale commutes);
      // its 64 columns come in one TMEM round trip
      float mb = -INFINITY;
      if (live && ok) {
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint32_t x[64];
        tmem_ld64(trow + scol, x);
        tmem_wait_ld();
        if (!full) {
          // masked block (rare): invisible keys become -inf in TMEM too, so
          // the exponential pass needs no mask (2^-inf = 0)
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!(mw[2 * hf + (c >> 5)] & (1u << (c & 31)))) x[c] = 0xff800000u;
          tmem_st32(trow + scol, *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
          tmem_st32(trow + scol + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
          tmem_wait_st();
        }
#pragma unroll
        for (int c = 0; c < 64; c += 8) {
          mx[0] = max3(mx[0], __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
          mx[1] = max3(mx[1], __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
          mx[2] = max3(mx[2], __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
          mx[3] = max3(mx[3], __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
        }
        mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
      }
      TIDAR_TRACE_PH(b2, 3);
      // swap block maxima and status with the other half of the row
      const int slot = t * 256;
      xmax[slot + hf * 128 + r] = mb;
      if (lane == 0) xok[t * 8 + hf * 4 + q4] = ok ? 1 : 0;            // ok is warp-uniform
      asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      const float mrow = fmaxf(mb, xmax[slot + (hf ^ 1) * 128 + r]);
      const bool both_ok = ok && xok[t * 8 + (hf ^ 1) * 4 + q4] != 0;
      // the slots are rewritten next block only after the partner has read them:
      // it cannot pass the next barrier before this thread arrives there
      asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      if (!both_ok) { ok = false; break; }               // both halves leave together
      const float m_new = fmaxf(m, mrow);
      const bool need = m_new > m + 8.0f;
      const float f_resc = need ? ex2(m - m_new) : 1.0f;   // factor for O_t and l (m = -inf -> 0)
      if (need) m = m_new;
      const float nbase = m == -INFINITY ? 0.f : -m;
      TIDAR_TRACE_PH(b2, 4);
      // pass 2: P = 2^(score * scale - m) in bf16 for this half's 64 keys, over
      // the first 32 columns of this half's S (one TMEM load, one store)
      float lblk = 0.f;
      if (live) {
        const uint64_t sl2x2 = f2_make(sl2, sl2), nbx2 = f2_make(nbase, nbase);
        uint64_t ls2[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
        uint32_t x[64];
        tmem_ld64(trow + scol, x);
        tmem_wait_ld();
        uint32_t pk[32];
        // The same loop for full and masked blocks (invisible keys hold -inf
        // in S since pass 1, and 2^-inf = 0).  Compiled as two copies, the
        // common full-block one is scheduled without register spills.
        auto exps = [&]() {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float v0, v1;
            f2_split(f2_fma(f2_make(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1])), sl2x2, nbx2), v0, v1);
            const float p0 = ex2(v0), p1 = ex2(v1);
            ls2[c & 1] = f2_add(ls2[c & 1], f2_make(p0, p1));
            pk[c] = cvt_bf16x2(p0, p1);
          }
        };
        if (full) exps();
        else exps();
        tmem_st32(trow + scol, pk);
        float la, lb, lc, ld;
        f2_split(ls2[0], la, lb);
        f2_split(ls2[1], lc, ld);
        lblk = (la + lb) + (lc + ld);
      }
      TIDAR_TRACE_PH(b2, 5);
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O_t holds PV of this set's earlier blocks: wait for the last one and
        // rescale this half's 64 columns before this block's PV is released
        if (!warp_wait_bar(bar(BAR_PVDONE + t), (uint32_t)((j - 1) & 1), abort_flag, a.err)) ok = false;
        fence_after();
        if (ok) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[16];
            tmem_ld16(trow + col_o(t) + 64 * hf + 16 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_resc);
            tmem_st16(trow + col_o(t) + 64 * hf + 16 * c, o);
          }
        }
      }
      l = l * f_resc + lblk;
      if (!window && (lo_valid < 64 || hi_valid < 64)) {
        // keys past the prefix end or on an unmapped page: zero their V rows so
        // that 0 * (whatever the page holds) cannot turn into NaN
        const int st = b2 % kStages;
        if (!warp_wait_bar(bar(BAR_VFULL + st), (uint32_t)((b2 / kStages) & 1), abort_flag, a.err)) ok = false;
        if (ok) {
          uint8_t* vs = smem + kOffV + st * kTileBytes;
          for (int idx = gt; idx < 128 * 16; idx += 256) {
            const int row = idx >> 4, piece = idx & 15;
            const bool inval = row < 64 ? row >= lo_valid : row - 64 >= hi_valid;
            if (inval)
              *reinterpret_cast<uint4*>(vs + (piece >> 3) * kChunkBytes + row * 128 + (piece & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
      }
      tmem_wait_st();
      TIDAR_TRACE_PH(b2, 6);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_PFULL + t));
      if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1280 + min(b2, 255));
    }
    // ---- epilogue: merge sets and halves.  The four warps of a lane quarter
    // (2 sets x 2 halves) meet at barrier 9 + quarter; each then writes 32 of
    // the 128 output columns of its rows.
    const int nb0 = (bp.nb + 1) >> 1, nb1 = bp.nb >> 1;
    // both sets' last PV must be complete before O_0 and O_1 are read; after it
    // no MMA reads shared memory, so the Q tile holds the exchange arrays
    if (ok && nb0 > 0 && !warp_wait_bar(bar(BAR_PVDONE + 0), (uint32_t)((nb0 - 1) & 1), abort_flag, a.err)) ok = false;
    if (ok && nb1 > 0 && !warp_wait_bar(bar(BAR_PVDONE + 1), (uint32_t)((nb1 - 1) & 1), abort_flag, a.err)) ok = false;
    fence_after();
    float* xm = reinterpret_cast<float*>(smem + kOffQ);              // [2 set][128] max
    float* xs = xm + 256;                                            // [2 set][2 half][128] sums
    int* xk = reinterpret_cast<int*>(xs + 512);                      // [2 set][2 half][4] status
    asm volatile("bar.sync %0, 128;" ::"r"(9 + q4) : "memory");
    if (hf == 0) xm[t * 128 + r] = m;
    xs[(t * 2 + hf) * 128 + r] = l;
    if (lane == 0) xk[t * 8 + hf * 4 + q4] = ok ? 1 : 0;
    asm volatile("bar.sync %0, 128;" ::"r"(9 + q4) : "memory");
    const float m0 = xm[r], m1 = xm[128 + r];
    const float l0 = xs[r] + xs[128 + r], l1 = xs[256 + r] + xs[384 + r];
    ok = xk[q4] && xk[4 + q4] && xk[8 + q4] && xk[12 + q4];
    if (warp == 4 && lane == 0) { TIDAR_TRACE_AT(1536); TIDAR_TRACE_CTA(2); }
    const float mt = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : ex2(m0 - mt);
    const float f1 = (m1 == -INFINITY || nb1 == 0) ? 0.f : ex2(m1 - mt);
    const float lt = l0 * f0 + l1 * f1;
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    const float g0 = f0 * inv, g1 = f1 * inv;
    const float lse = lt > 0.f ? (mt + log2f(lt)) * 0.69314718055994531f : -INFINITY;
    const bool write = r < rows_valid && ok;
    const int col0 = 32 * (2 * t + hf);                  // this thread's 32 output columns
    {
      uint32_t o0[32], o1[32];
      tmem_ld32(trow + col_o(0) + col0, o0);
      if (nb1 > 0) tmem_ld32(trow + col_o(1) + col0, o1);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        ov[e] = __uint_as_float(o0[e]) * g0 + (nb1 > 0 ? __uint_as_float(o1[e]) * g1 : 0.f);
    }
    owrite = write;
    olse = lse;
    if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1538);
  }

  // The producer has drained, every MMA is complete and no copy is in flight.
  if (lane == 0) TIDAR_TRACE_AT(1550 + warp);
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TIDAR_TRACE_AT(1542);

  // ------------------------------------------------------------------ write-out
  // The softmax threads stage their normalised O (32 columns of one row each)
  // and the rows' lse in the idle K ring; then every warp stores whole rows:
  // the bf16 output (one split), or this split's fp32 partials, which the
  // splits of a cluster then merge (cluster_merge) or a finalize launch does.
  // A CTA without keys (an empty slice of a prefix-only call, or a split past
  // a short sequence's prefix) contributes O = 0 with lse = -inf.
  float* ost = reinterpret_cast<float*>(smem + kOffK);
  float* lst = ost + 128 * kStageStride;
  int* wst = reinterpret_cast<int*>(lst + 128);
  if (warp >= 2) {
    const int r = 32 * (warp & 3) + lane;
    const int t = (warp - 2) >> 3, hf = ((warp - 2) >> 2) & 1;
    if (bp.nb == 0) {
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] = 0.f;
      olse = -INFINITY;
      owrite = r < rows_valid;
    }
    float4* d = reinterpret_cast<float4*>(ost + r * kStageStride + 32 * (2 * t + hf));
#pragma unroll
    for (int e = 0; e < 32; e += 4) d[e / 4] = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
    if (t == 0 && hf == 0) {
      lst[r] = owrite ? olse : -INFINITY;
      wst[r] = owrite ? 1 : 0;
    }
    if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1543);
  }
  __syncthreads();
  if (threadIdx.x == 0) TIDAR_TRACE_AT(1544);
  auto out_row = [&](int r) -> long long {
    const int rho = rho0 + r / a.G, h = g * a.G + r % a.G;
    return (long long)(b * a.R + rho) * a.Hq + h;
  };
  if (a.nsplit == 1) {
    store_rows_bf16(ost, lst, wst, rows_valid, out_row, static_cast<__nv_bfloat16*>(a.out), a.lse_out);
  } else if (a.cluster_merge) {
    // ---------------------------------------------------------------- split merge
    // The CTAs of this cluster are the splits of one (b, g, tile) (cluster
    // rank = split): once all of them have staged their rows (first cluster
    // barrier), CTA j merges rows j, j + ns, j + 2 ns, ... of the tile from
    // every split's shared memory; the second barrier keeps each CTA's shared
    // memory alive until its peers are done.
    const int ns = a.nsplit;
    const int rank = (int)cluster_rank();
    cluster_sync_all();
    if (threadIdx.x == 0) { TIDAR_TRACE_AT(1540); TIDAR_TRACE_CTA(3); }
    const int owned = rows_valid > rank ? (rows_valid - rank + ns - 1) / ns : 0;
    merge_rows<4, 2>(ost, lst, ns, rank, owned, out_row, static_cast<__nv_bfloat16*>(a.out), a.lse_out);
    if (threadIdx.x == 0) TIDAR_TRACE_AT(1541);
    cluster_sync_all();
  } else {
    const long long stride = (long long)a.B * a.R * a.Hq;
    store_rows_partial(ost, lst, wst, rows_valid, [&](int r) -> long long { return split * stride + out_row(r); },
                       a.part_o, a.part_lse);
    if (warp == 4 && lane == 0) TIDAR_TRACE_AT(1539);
  }

  if (tile == 0 && split == 0 && len_ok && (a.nsplit == 1 || a.cluster_merge) && a.append) {
    // ---------------------------------------------------------------- append
    // Draft rows D_1..D_n of KV head g into cache rows P .. P+n-1 (the keys
    // above read them from k_blk / v_blk, not from the cache).
    for (int c = threadIdx.x; c < a.n * 2 * 16; c += kThreads) {
      const int r = c >> 5, which = (c >> 4) & 1, piece = c & 15;
      const int pos = P + r;
      const int page = table[pos / 64];
      if (!page_ok(page, a.num_pages)) {
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
// The kernel's dynamic shared memory opt-in, once per device.
cudaError_t set_smem_attr() {
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
  return cudaSuccess;
}

}  // namespace

void set_starve_loads(int on) { g_starve_loads = on != 0; }
int tc05_starve_loads() { return g_starve_loads; }

#ifdef TIDAR_TRACE
extern "C" int tidar_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_tidar_trace, bytes);
}
extern "C" int tidar_trace_clear(void) {
  static unsigned long long zeros[2048 + 4 * 8192];
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
  prm.starve = g_starve_loads;

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
  cudaError_t e = set_smem_attr();
  if (e != cudaSuccess) return e;
  const bool clu = a.nsplit > 1 && a.cluster_merge;
  if (a.nsplit > 1 && !clu && (!a.part_o || !a.part_lse)) return cudaErrorInvalidValue;
  if (clu && a.nsplit > kMaxCluster) return cudaErrorNotSupported;
  const dim3 grid(prm.tiles, a.nsplit, a.B * a.Hkv);
  // with the cluster merge, the splits of one (b, g, tile) form a cluster
  const dim3 cluster(1, clu ? a.nsplit : 1, 1);
  return launch_clustered(attn_tc05_kernel, grid, cluster, kThreads, kSmemAlloc, s, tq, tkp, tvp, tks, tvs,
                          prm);
}

int tc05_resident_clusters(int ns) {
  static int cache[64][kMaxCluster + 1];
  if (ns < 1 || ns > kMaxCluster) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev][ns]) return cache[dev][ns] - 1;
  int n = 0;
  if (set_smem_attr() == cudaSuccess &&
      (ns <= 8 || cudaFuncSetAttribute(attn_tc05_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, ns, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = ns;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc05_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache[dev][ns] = n + 1;
  return n;
}

}  // namespace tidar
