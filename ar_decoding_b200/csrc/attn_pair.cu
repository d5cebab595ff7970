// attn_pair.cu -- tensor-core step attention with two query tiles per CTA
// (sm_100a: tcgen05 + TMEM + TMA).
//
// Same operation as the other step-attention kernels (the three-zone
// structured-mask attention of one TiDAR step: "TiDAR: Think in Diffusion,
// Talk in Autoregression", mauroscia.it section 2; nodesdaily.com (fr),
// paragraphs on the three zones and the masking puzzle), for bf16, head_dim
// 128, page 64, on query blocks of more than one 128-row tile per KV head
// (large k: at k = 16 with 4 query heads per KV head a sequence has 272 x 4 =
// 1088 packed rows).  There the step is a dense QK^T / PV contraction over the
// shared prefix, and this kernel is built around keeping the tensor pipe busy.
//
// Work unit (one CTA): sequence b, KV head g, two consecutive query tiles of
// 128 packed rows each (row m of a tile = (rho - rho0) * G + head-in-group), and
// one split of the cached prefix.  Every K/V block staged in shared memory
// feeds both tiles, and the two tiles' softmaxes alternate with each other's
// MMAs in the single in-order tensor pipe:
//
//   S0(b) S1(b) | PV0(b) S0(b+1) | PV1(b) S1(b+1) | PV0(b+1) S0(b+2) | ...
//
// so while warpgroup 0 turns S0(b+1) into probabilities the pipe runs tile 1's
// PV and next scores, and the other way round.  TMEM (512 columns): S0, S1
// (128 fp32 columns each; P, bf16, is written over the first 64), O0, O1.
//
// Roles (12 warps, 384 threads):
//   warps 0..3   softmax of tile 0: thread r owns packed row r (TMEM lane r)
//                and all 128 columns of a block: one tcgen05.ld pass, the
//                row maximum in registers, 2^(score*scale*log2e - max) on the
//                MUFU, P back to TMEM as bf16.  O is rescaled only when the
//                row maximum grows by more than 2^8 (log2 domain).
//   warps 4..7   the same for tile 1.
//   warp 8       TMA producer: Q tiles once; per 128-key block two 64-row
//                pages of K and of V (paged cache, SWIZZLE_128B) or one
//                step-key window; a 3-stage K ring and a 2-stage V ring.
//                No multicast.
//   warp 9       TMEM owner and MMA issuer (one thread).
//   warps 10, 11 only the split merge and the draft-row append.
// The last split also runs the step-key windows holding keys visible to
// either tile, with the zone mask applied in the softmax.  Key splits of one
// (b, g, pair) either form a thread-block cluster and merge in this kernel
// (each CTA stages its normalised rows in shared memory; after a cluster
// barrier CTA `rank` merges a share of the rows over distributed shared
// memory) or write fp32 partials to the workspace for a finalize launch.
// Every mbarrier wait is bounded (~1 s): on expiry the CTA records
// TIDAR_DEVERR_TIMEOUT, stops issuing, drains what it issued, frees TMEM and
// exits through the same cluster barriers as the other CTAs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tc05.cuh"

namespace tidar {

namespace {

using namespace tc05;

constexpr int kPThreads = 384;
constexpr int kKSt = 3;                                    // K ring stages
constexpr int kVSt = 2;                                    // V ring stages
constexpr uint32_t kPChunk = 16384;                        // 128 rows x 128 B (64 bf16)
constexpr uint32_t kPTile = 2 * kPChunk;                   // 128 x 128 bf16
constexpr uint32_t kPOffQ = 0;                             // + t * kPTile
constexpr uint32_t kPOffK = 2 * kPTile;
constexpr uint32_t kPOffV = kPOffK + kKSt * kPTile;
constexpr uint32_t kPOffBar = kPOffV + kVSt * kPTile;
constexpr int PB_Q = 0;
constexpr int PB_KFULL = 1;      // + stage
constexpr int PB_KEMPTY = 4;     // + stage: both tiles' S MMAs of the block are done
constexpr int PB_VFULL = 7;      // + stage
constexpr int PB_VEMPTY = 9;     // + stage: both tiles' PV MMAs of the block are done
constexpr int PB_SFULL = 11;     // + tile
constexpr int PB_PFULL = 13;     // + tile (four warp arrivals)
constexpr int PB_PVDONE = 15;    // + tile
constexpr int PB_FINAL = 17;
constexpr int kPBars = 18;
constexpr uint32_t kPOffMisc = kPOffBar + kPBars * 8;      // [0] TMEM base, [1] abort flag
constexpr uint32_t kPSmem = kPOffMisc + 16;
static_assert(kPSmem <= 232448, "shared memory budget");
static_assert((256 * kStageStride + 512) * 4 <= (kKSt + kVSt) * kPTile, "row staging fits the K/V rings");
// split merge receive area, in the K/V rings once they are idle: [slot][split]
// [32 float4] fp32 partial rows for at most 256 + 16 (slot, split) pairs, then
// their lse

constexpr uint32_t kPTmemCols = 512;
__device__ __forceinline__ uint32_t pcol_s(int t) { return 128u * (uint32_t)t; }
__device__ __forceinline__ uint32_t pcol_o(int t) { return 256u + 128u * (uint32_t)t; }
// kind::f16 instruction descriptors: fp32 accumulate, bf16 A and B, M = N = 128.
constexpr uint32_t kPIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kPIdescPV = kPIdescS | (1u << 16);     // B (= V) is MN-major

// Optional timeline of CTA (0, 0, 0) (build with -DTIDAR_TRACE; absent from
// normal builds): [0] setup, [1] TMEM ready, [16 + 4 i + t] S_t(i) issued,
// [512 + 4 i + t] PV_t(i) issued, [1024 + 4 i + t] softmax t sees S_t(i),
// [1536 + 4 i + t] P_t(i) handed over, [2048 + 8 i + ph] warp 0's phases of
// block i (0 wait done, 1 loaded, 2 max, 3 exps, 4 stored), [2600] epilogue,
// [2601] end; [4096 + 2 cta] start / end of every CTA.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_pair_trace[4096 + 4 * 8192];
__device__ __forceinline__ bool ptrace_cta() { return blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0; }
#define PAIR_TRACE(slot) do { if (ptrace_cta() && (slot) < 4096) g_pair_trace[(slot)] = global_ns(); } while (0)
#define PAIR_TRACE_CTA(w) do { const unsigned c_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (c_ < 8192) g_pair_trace[4096 + 4 * c_ + (w)] = global_ns(); } while (0)
#else
#define PAIR_TRACE(slot) do {} while (0)
#define PAIR_TRACE_CTA(w) do {} while (0)
#endif

struct PairParams {
  AttnArgs a;
  int rho_per_tile;   // query rows per tile (128 / G)
  int tiles;          // tiles per (b, g)
  int pairs;          // CTAs per (b, g, split): ceil(tiles / 2)
  float scale_log2;   // softmax scale * log2(e)
  int starve;         // test hook: issue no K/V copies (the waits for them run out)
};

__global__ void __launch_bounds__(kPThreads, 1)
attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                 const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                 const __grid_constant__ CUtensorMap tm_vs, const PairParams prm) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const AttnArgs& a = prm.a;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool cluster = a.nsplit > 1 && a.cluster_merge;
  // A CTA whose layout check fails does no work but still meets its cluster.
  const bool layout_ok = (sb & 1023u) == 0;
  const int pair = blockIdx.x, split = blockIdx.y;
  const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
  const int tile0 = 2 * pair;
  const int ntile = min(2, prm.tiles - tile0);            // 1 or 2 tiles in this CTA
  int rho0[2], rho1[2], rows_valid[2];
  for (int t = 0; t < 2; ++t) {
    rho0[t] = (tile0 + t) * prm.rho_per_tile;
    rho1[t] = min(a.R, rho0[t] + prm.rho_per_tile);
    rows_valid[t] = t < ntile ? (rho1[t] - rho0[t]) * a.G : 0;
  }
  auto bar = [&](int i) -> uint32_t { return sb + kPOffBar + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kPOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  if (threadIdx.x == 0) {
    PAIR_TRACE_CTA(0);
    PAIR_TRACE(0);
    *abort_flag = layout_ok ? 0 : 1;
    if (layout_ok) {
      for (int i = 0; i < kPBars; ++i) mbar_init(bar(i), (i == PB_PFULL || i == PB_PFULL + 1) ? 4u : 1u);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kp);
      prefetch_tmap(&tm_vp);
      prefetch_tmap(&tm_ks);
      prefetch_tmap(&tm_vs);
      prefetch_l2(a.seq_lens + b, 4, 0, 1);
      const int pgq = split * a.keys_per_split / 64;     // the last split may start past the table
      if (pgq < a.max_pages)
        prefetch_l2(a.page_table + (size_t)b * a.max_pages + pgq, min(256, 4 * (a.max_pages - pgq)), 0, 1);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    } else {
      raise_error(a.err, TIDAR_DEVERR_LAYOUT);
    }
  }
  if (layout_ok && warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kPOffMisc),
                 "r"(kPTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = layout_ok ? misc[0] : 0u;
  if (threadIdx.x == 0) PAIR_TRACE(1);

  pdl_wait();       // the previous kernel on the stream is complete from here on
  pdl_trigger();

  int P = a.seq_lens[b];
  const bool len_ok = P >= 0 && P <= a.max_prefix;
  if (!len_ok) {
    if (threadIdx.x == 0 && pair == 0 && split == 0) raise_error(a.err, TIDAR_DEVERR_BAD_LEN);
    P = 0;
  }
  const BlockPlan bp = make_block_plan(a, P, split, rho0[0], ntile == 2 ? rho1[1] : rho1[0]);
  const int nb = layout_ok ? bp.nb : 0;
  const int32_t* table = a.page_table + (size_t)b * a.max_pages;

  // This thread's row of the output (softmax warps), carried past the roles.
  float ov[128];
  float olse = -INFINITY;
  bool owrite = false;

  if (nb == 0) {
    // no keys for this split (or a failed layout check): an empty partial
  } else if (warp == 8) {
    // ---------------------------------------------------------------- producer
    constexpr unsigned kAll = 0xffffffffu;
    int k_phase[kKSt], v_phase[kVSt];
    for (int s2 = 0; s2 < kKSt; ++s2) k_phase[s2] = -1;
    for (int s2 = 0; s2 < kVSt; ++s2) v_phase[s2] = -1;
    if (lane == 0) {
      // a tile box holds rho_per_tile * G packed rows (126 of 128 when G = 6)
      mbar_expect_tx(bar(PB_Q), (uint32_t)ntile * 2u * 128u * (uint32_t)(prm.rho_per_tile * a.G));
      for (int t = 0; t < ntile; ++t) {
        tma_load_4d(sb + kPOffQ + t * kPTile, &tm_q, 0, g * a.G, rho0[t], b, bar(PB_Q));
        tma_load_4d(sb + kPOffQ + t * kPTile + kPChunk, &tm_q, 64, g * a.G, rho0[t], b, bar(PB_Q));
      }
    }
    // page-table entries of this split, 32 at a time, one per lane, the next
    // window already loading
    const int pg0 = bp.k0 / 64;                                   // k0 is a multiple of 128
    auto load_win = [&](int base) -> int {
      const int pi = pg0 + base + lane;
      return pi < a.max_pages ? table[pi] : -1;
    };
    int kwb = 0, kcur = load_win(0), knxt = load_win(32);
    int vwb = 0, vcur = kcur, vnxt = knxt;
    auto entry = [&](int& base, int& cur, int& nxt, int pi) -> int {
      while (pi >= base + 32) {
        base += 32;
        cur = nxt;
        nxt = load_win(base + 32);
      }
      return __shfl_sync(kAll, cur, pi - base);
    };
    bool bad = false;
    auto issue = [&](int i, bool is_v) {
      const int s = is_v ? i % kVSt : i % kKSt;
      const uint32_t dst = sb + (is_v ? kPOffV : kPOffK) + s * kPTile;
      const uint32_t full = bar((is_v ? PB_VFULL : PB_KFULL) + s);
      if (i < bp.npb) {
        const CUtensorMap* map = is_v ? &tm_vp : &tm_kp;
        const int start = bp.k0 + i * 128;
        const bool need_b = start + 64 < bp.kend;
        const int pa = is_v ? entry(vwb, vcur, vnxt, 2 * i) : entry(kwb, kcur, knxt, 2 * i);
        const int pb2 = is_v ? entry(vwb, vcur, vnxt, 2 * i + 1) : entry(kwb, kcur, knxt, 2 * i + 1);
        const bool oka = page_ok(pa, a.num_pages), okb = need_b && page_ok(pb2, a.num_pages);
        if (!oka || (need_b && !okb)) bad = true;
        if (lane == 0) {
          mbar_expect_tx(full, (uint32_t)(oka + okb) * 2u * 8192u);
          if (oka) {
            tma_load_2d(dst, map, 0, (pa * a.Hkv + g) * 64, full);
            tma_load_2d(dst + kPChunk, map, 64, (pa * a.Hkv + g) * 64, full);
          }
          if (okb) {
            tma_load_2d(dst + 8192, map, 0, (pb2 * a.Hkv + g) * 64, full);
            tma_load_2d(dst + kPChunk + 8192, map, 64, (pb2 * a.Hkv + g) * 64, full);
          }
        }
      } else if (lane == 0) {
        const CUtensorMap* map = is_v ? &tm_vs : &tm_ks;
        const int w = bp.wins[i - bp.npb];
        mbar_expect_tx(full, kPTile);
        tma_load_4d(dst, map, 0, g, w * 128, b, full);
        tma_load_4d(dst + kPChunk, map, 64, g, w * 128, b, full);
      }
      if (is_v) v_phase[s] = i / kVSt;
      else k_phase[s] = i / kKSt;
    };
    auto test_all = [&](uint32_t bar_addr, uint32_t parity) -> bool {
      const int t = lane == 0 ? (int)mbar_test(bar_addr, parity) : 0;
      return __shfl_sync(kAll, t, 0) != 0;
    };
    auto aborted = [&]() -> bool { return __shfl_sync(kAll, lane == 0 ? *abort_flag : 0, 0) != 0; };
    int ik = prm.starve ? nb : 0, iv = ik;
    uint64_t last = global_ns();
    while ((ik < nb || iv < nb) && !aborted()) {
      bool progress = false;
      if (ik < nb && (ik < kKSt || test_all(bar(PB_KEMPTY + ik % kKSt), (uint32_t)((ik / kKSt - 1) & 1)))) {
        issue(ik, false);
        ++ik;
        progress = true;
      }
      if (iv < ik && (iv < kVSt || test_all(bar(PB_VEMPTY + iv % kVSt), (uint32_t)((iv / kVSt - 1) & 1)))) {
        issue(iv, true);
        ++iv;
        progress = true;
      }
      if (progress) {
        last = global_ns();
      } else {
        if (lane == 0) {
          if (ik < nb && ik - iv < kKSt)
            mbar_try_wait_ns(bar(PB_KEMPTY + ik % kKSt), (uint32_t)((ik / kKSt - 1) & 1), 500u);
          else
            mbar_try_wait_ns(bar(PB_VEMPTY + iv % kVSt), (uint32_t)((iv / kVSt - 1) & 1), 500u);
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
      if (*abort_flag) {
        // drain: no copy may still write shared memory when the CTA moves on
        for (int s2 = 0; s2 < kKSt; ++s2)
          if (k_phase[s2] >= 0) wait_quiet(bar(PB_KFULL + s2), k_phase[s2] & 1);
        for (int s2 = 0; s2 < kVSt; ++s2)
          if (v_phase[s2] >= 0) wait_quiet(bar(PB_VFULL + s2), v_phase[s2] & 1);
        wait_quiet(bar(PB_Q), 0);
      }
    }
  } else if (warp == 9) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = wait_bar(bar(PB_Q), 0, abort_flag, a.err);
      fence_after();
      // S_t(blk) = Q_t K_blk^T into S_t; the K stage is released once the last
      // tile's S of the block is issued
      auto issue_s = [&](int t, int blk) -> bool {
        const int st = blk % kKSt;
        if (t == 0) {
          if (!wait_bar(bar(PB_KFULL + st), (uint32_t)((blk / kKSt) & 1), abort_flag, a.err)) return false;
          fence_after();
        }
        const uint32_t qa = sb + kPOffQ + t * kPTile, ka = sb + kPOffK + st * kPTile;
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const uint32_t off = (kc >> 2) * kPChunk + (kc & 3) * 32;
          mma_ss(tmem + pcol_s(t), desc_k_sw128(qa + off), desc_k_sw128(ka + off), kPIdescS, kc > 0);
        }
        mma_commit(bar(PB_SFULL + t));
        if (t == ntile - 1) mma_commit(bar(PB_KEMPTY + st));
        PAIR_TRACE(16 + 4 * min(blk, 120) + t);
        return true;
      };
      for (int t = 0; ok && t < ntile; ++t) ok = issue_s(t, 0);
      for (int b2 = 0; ok && b2 < nb; ++b2) {
        const int vs = b2 % kVSt;
        if (!wait_bar(bar(PB_VFULL + vs), (uint32_t)((b2 / kVSt) & 1), abort_flag, a.err)) break;
        const uint32_t va = sb + kPOffV + vs * kPTile;
        for (int t = 0; ok && t < ntile; ++t) {
          if (!wait_bar(bar(PB_PFULL + t), (uint32_t)(b2 & 1), abort_flag, a.err)) { ok = false; break; }
          fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + pcol_o(t), tmem + pcol_s(t) + 8u * kk, desc_mn_sw128(va + kk * 2048, kPChunk), kPIdescPV,
                   (b2 > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(PB_PVDONE + t));
          PAIR_TRACE(512 + 4 * min(b2, 120) + t);
          if (t == ntile - 1) mma_commit(bar(PB_VEMPTY + vs));
          if (b2 + 1 < nb && !issue_s(t, b2 + 1)) ok = false;
        }
      }
      // every MMA issued above has completed before TMEM is read or released
      mma_commit(bar(PB_FINAL));
      wait_quiet(bar(PB_FINAL), 0);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- softmax
    const int t = warp >> 2;                             // tile of this warpgroup
    const int r = threadIdx.x & 127;                     // packed row = TMEM lane
    if (t < ntile) {
      const int rho_c = min(rho0[t] + r / a.G, a.R - 1);
      const StepVis vis = step_visibility(a.k, rho_c);
      const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      const float sl2 = prm.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int b2 = 0; b2 < nb; ++b2) {
        if (!warp_wait_bar(bar(PB_SFULL + t), (uint32_t)(b2 & 1), abort_flag, a.err)) { ok = false; break; }
        fence_after();
        if (r == 0) PAIR_TRACE(1024 + 4 * min(b2, 120) + t);
        if (threadIdx.x == 0) PAIR_TRACE(2048 + 8 * min(b2, 60) + 0);
        int lo_valid = 64, hi_valid = 64, kb = 0;
        const bool window = b2 >= bp.npb;
        if (!window) {
          const int start = bp.k0 + b2 * 128;
          lo_valid = min(64, bp.kend - start);
          hi_valid = max(0, min(64, bp.kend - start - 64));
          if (lo_valid < 64 || hi_valid < 64) {          // page checks only where a page may be absent
            if (!page_ok(table[start / 64], a.num_pages)) lo_valid = 0;
            if (hi_valid > 0 && !page_ok(table[start / 64 + 1], a.num_pages)) hi_valid = 0;
          }
        } else {
          kb = bp.wins[b2 - bp.npb] * 128;
        }
        const bool full = !window && lo_valid == 64 && hi_valid == 64;
        uint32_t x[128];
        tmem_ld32(trow + pcol_s(t), *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
        tmem_ld32(trow + pcol_s(t) + 32, *reinterpret_cast<uint32_t(*)[32]>(&x[32]));
        tmem_ld32(trow + pcol_s(t) + 64, *reinterpret_cast<uint32_t(*)[32]>(&x[64]));
        tmem_ld32(trow + pcol_s(t) + 96, *reinterpret_cast<uint32_t(*)[32]>(&x[96]));
        tmem_wait_ld();
        if (threadIdx.x == 0) PAIR_TRACE(2048 + 8 * min(b2, 60) + 1);
        if (!full) {
          // invisible keys (zone mask, past the prefix end, unmapped page) get
          // -inf: their probability is 2^-inf = 0
          uint32_t mw[4];
          block_mask(window, kb, vis, a.R, lo_valid, hi_valid, mw);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!(mw[c >> 5] & (1u << (c & 31)))) x[c] = 0xff800000u;
        }
        // row maximum: eight independent chains
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 16)
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = max3(mx[i], __uint_as_float(x[c + 2 * i]), __uint_as_float(x[c + 2 * i + 1]));
        const float mrow = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
        if (threadIdx.x == 0) PAIR_TRACE(2048 + 8 * min(b2, 60) + 2);
        const float m_new = fmaxf(m, mrow);
        const bool need = m_new > m + 8.0f;
        const float f_resc = need ? ex2(m - m_new) : 1.0f;  // factor for O and l (m = -inf -> 0)
        if (need) m = m_new;
        const float nbase = m == -INFINITY ? 0.f : -m;
        // P = 2^(score * scale - m), bf16 pairs packed in place over x[0..63]
        // (every exponential on the MUFU: moving a share to an FMA-pipe
        // polynomial and the bf16 packing to integer operations was measured
        // slower -- the softmax warp is issue-bound, not MUFU-bound)
        const uint64_t sl2x2 = f2_make(sl2, sl2), nbx2 = f2_make(nbase, nbase);
        uint64_t ls2[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          float v0, v1;
          f2_split(f2_fma(f2_make(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1])), sl2x2, nbx2), v0, v1);
          const float p0 = ex2(v0), p1 = ex2(v1);
          ls2[c & 1] = f2_add(ls2[c & 1], f2_make(p0, p1));
          x[c] = cvt_bf16x2(p0, p1);
        }
        if (threadIdx.x == 0) PAIR_TRACE(2048 + 8 * min(b2, 60) + 3);
        tmem_st32(trow + pcol_s(t), *reinterpret_cast<const uint32_t(*)[32]>(&x[0]));
        tmem_st32(trow + pcol_s(t) + 32, *reinterpret_cast<const uint32_t(*)[32]>(&x[32]));
        float la, lb, lc, ld;
        f2_split(ls2[0], la, lb);
        f2_split(ls2[1], lc, ld);
        const float lblk = (la + lb) + (lc + ld);
        if (__any_sync(0xffffffffu, need) && b2 > 0) {
          // O_t holds PV of the earlier blocks: wait for the last one and
          // rescale this row before this block's PV is released
          if (!warp_wait_bar(bar(PB_PVDONE + t), (uint32_t)((b2 - 1) & 1), abort_flag, a.err)) ok = false;
          fence_after();
          if (ok) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(trow + pcol_o(t) + 32 * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f_resc);
              tmem_st32(trow + pcol_o(t) + 32 * c, o);
            }
          }
        }
        l = l * f_resc + lblk;
        if (t == 0 && !window && (lo_valid < 64 || hi_valid < 64)) {
          // keys past the prefix end or on an unmapped page: zero their V rows
          // so that 0 * (whatever the page holds) cannot turn into NaN.  Tile
          // 0's warpgroup does it before it releases P0, and PV1 of the block
          // is issued after PV0.
          const int vs = b2 % kVSt;
          if (!warp_wait_bar(bar(PB_VFULL + vs), (uint32_t)((b2 / kVSt) & 1), abort_flag, a.err)) ok = false;
          if (ok) {
            uint8_t* vsm = smem + kPOffV + vs * kPTile;
            for (int idx = r; idx < 128 * 16; idx += 128) {
              const int row = idx >> 4, piece = idx & 15;
              const bool inval = row < 64 ? row >= lo_valid : row - 64 >= hi_valid;
              if (inval)
                *reinterpret_cast<uint4*>(vsm + (piece >> 3) * kPChunk + row * 128 + (piece & 7) * 16) =
                    make_uint4(0, 0, 0, 0);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          }
          // no barrier here: PV0 of the block waits for all four warps' P0
          // arrivals, each made after that warp's share of the zeroing (and
          // a named barrier could strand a warp that gave up on a wait)
        }
        tmem_wait_st();
        fence_before();
        __syncwarp();
        if (!__all_sync(0xffffffffu, ok)) { ok = false; }
        if (lane == 0) mbar_arrive(bar(PB_PFULL + t));
        if (r == 0) PAIR_TRACE(1536 + 4 * min(b2, 120) + t);
        if (threadIdx.x == 0) PAIR_TRACE(2048 + 8 * min(b2, 60) + 4);
        if (!ok) break;
      }
      if (threadIdx.x == 0) { PAIR_TRACE(2600); PAIR_TRACE_CTA(2); }
      // ---- this tile's row of O: wait for the last PV, normalise
      if (ok && nb > 0 && !warp_wait_bar(bar(PB_PVDONE + t), (uint32_t)((nb - 1) & 1), abort_flag, a.err)) ok = false;
      ok = __all_sync(0xffffffffu, ok && !*abort_flag);
      fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      olse = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(trow + pcol_o(t) + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[32 * c + e] = __uint_as_float(o[e]) * inv;
        }
      }
      owrite = ok && r < rows_valid[t];
      if (threadIdx.x == 0) PAIR_TRACE(2602);
    }
  }

  // The producer has drained, every MMA is complete and no copy is in flight.
  if (lane == 0) PAIR_TRACE(2610 + warp);
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0) PAIR_TRACE(2606);

  // ------------------------------------------------------------------ write-out
  // Staged row i = t * 128 + r (tile t) in the idle K/V rings, then whole-row
  // stores: the bf16 output (one split) or this split's fp32 partials, merged
  // by the cluster (cluster_merge) or a finalize launch.  A pair without keys
  // (an empty slice of a prefix-only call, or a split past a short sequence's
  // prefix) contributes O = 0 with lse = -inf.
  float* ost = reinterpret_cast<float*>(smem + kPOffK);
  float* lst = ost + 256 * kStageStride;
  int* wst = reinterpret_cast<int*>(lst + 256);
  if (warp < 8) {
    const int t = warp >> 2, r = threadIdx.x & 127;
    if (nb == 0) {
#pragma unroll
      for (int e = 0; e < 128; ++e) ov[e] = 0.f;
      olse = -INFINITY;
      owrite = layout_ok && r < rows_valid[t];
    }
    float4* d = reinterpret_cast<float4*>(ost + (t * 128 + r) * kStageStride);
#pragma unroll
    for (int e = 0; e < 128; e += 4) d[e / 4] = make_float4(ov[e], ov[e + 1], ov[e + 2], ov[e + 3]);
    lst[t * 128 + r] = owrite ? olse : -INFINITY;
    wst[t * 128 + r] = owrite ? 1 : 0;
    if (threadIdx.x == 0) PAIR_TRACE(2607);
  }
  __syncthreads();
  if (threadIdx.x == 0) PAIR_TRACE(2608);
  auto out_row = [&](int i) -> long long {
    const int t = i >> 7, rr = i & 127;
    if (t >= ntile || rr >= rows_valid[t]) return -1;
    const int rho = rho0[t] + rr / a.G, h = g * a.G + rr % a.G;
    return (long long)(b * a.R + rho) * a.Hq + h;
  };
  if (a.nsplit == 1) {
    store_rows_bf16(ost, lst, wst, 256, out_row, static_cast<__nv_bfloat16*>(a.out), a.lse_out);
  } else if (cluster) {
    // ---------------------------------------------------------------- split merge
    // Staged row i of the pair is merged by CTA i % ns from every split's
    // shared memory once all have staged (first cluster barrier); the second
    // keeps each CTA's shared memory alive until its peers are done.
    const int ns = a.nsplit;
    const int rank = (int)cluster_rank();
    cluster_sync_all();
    if (threadIdx.x == 0) { PAIR_TRACE(2604); PAIR_TRACE_CTA(3); }
    const int owned = (256 - rank + ns - 1) / ns;
    merge_rows<4, 4>(ost, lst, ns, rank, owned, out_row, static_cast<__nv_bfloat16*>(a.out), a.lse_out);
    if (threadIdx.x == 0) PAIR_TRACE(2605);
    cluster_sync_all();
  } else {
    const long long stride = (long long)a.B * a.R * a.Hq;
    store_rows_partial(ost, lst, wst, 256, [&](int i) -> long long {
                         const long long r = out_row(i);
                         return r < 0 ? -1 : split * stride + r;
                       },
                       a.part_o, a.part_lse);
    if (threadIdx.x == 0) PAIR_TRACE(2603);
  }

  if (pair == 0 && split == 0 && len_ok && (a.nsplit == 1 || cluster) && a.append) {
    // ---------------------------------------------------------------- append
    // Draft rows D_1..D_n of KV head g into cache rows P .. P+n-1 (the keys
    // above read them from k_blk / v_blk, not from the cache).
    for (int c = threadIdx.x; c < a.n * 2 * 16; c += kPThreads) {
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

  if (threadIdx.x == 0) { PAIR_TRACE(2601); PAIR_TRACE_CTA(1); }
  if (layout_ok && warp == 9) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPTmemCols) : "memory");
  }
}

// The kernel's dynamic shared memory opt-in, once per device.
cudaError_t pair_smem_attr() {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return cudaSuccess;
}

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_pair_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_pair_trace, bytes);
}
extern "C" int tidar_pair_trace_clear(void) {
  static unsigned long long zeros[4096 + 4 * 8192];
  return (int)cudaMemcpyToSymbol(g_pair_trace, zeros, sizeof zeros);
}
#endif

cudaError_t launch_attn_pair(const AttnArgs& a, cudaStream_t s) {
  if (!a.bf16 || a.D != 128 || a.page_size != 64 || a.G > 128) return cudaErrorNotSupported;
  PairParams prm;
  prm.a = a;
  prm.rho_per_tile = 128 / a.G;
  prm.tiles = (a.R + prm.rho_per_tile - 1) / prm.rho_per_tile;
  prm.pairs = (prm.tiles + 1) / 2;
  prm.scale_log2 = a.scale * 1.4426950408889634f;
  prm.starve = tc05_starve_loads();

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
  cudaError_t e = pair_smem_attr();
  if (e != cudaSuccess) return e;
  const bool clu = a.nsplit > 1 && a.cluster_merge;
  if (a.nsplit > 1 && !clu && (!a.part_o || !a.part_lse)) return cudaErrorInvalidValue;
  if (clu && a.nsplit > kMaxCluster) return cudaErrorNotSupported;
  const dim3 grid(prm.pairs, a.nsplit, a.B * a.Hkv);
  const dim3 cluster(1, clu ? a.nsplit : 1, 1);
  return launch_clustered(attn_pair_kernel, grid, cluster, kPThreads, kPSmem, s, tq, tkp, tvp, tks, tvs, prm);
}

int pair_resident_clusters(int ns) {
  static int cache[64][kMaxCluster + 1];
  if (ns < 1 || ns > kMaxCluster) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev][ns]) return cache[dev][ns] - 1;
  int n = 0;
  if (pair_smem_attr() == cudaSuccess &&
      (ns <= 8 || cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, ns, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = kPSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = ns;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_pair_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache[dev][ns] = n + 1;
  return n;
}

}  // namespace tidar
