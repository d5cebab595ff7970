// linear_tc05.cu -- the projections on either side of the step attention, on
// the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// At the level of one transformer layer a TiDAR step is: project the R step
// rows' hidden states to queries, keys and values, rotate queries and keys to
// their positions, run the three-zone attention, project the result back
// ("TiDAR: Think in Diffusion, Talk in Autoregression", mauroscia.it section
// 2: one forward pass over the three zones; engineer-news.pages.dev, section
// "為什麼 GPU 在 AR 推論時是閒置的": every decode step reloads the weights,
// so a memory-bound step leaves compute idle for the extra rows).  Both
// projections are y = x w^T with the weights [N][K] bf16 and the rows x [T][K]
// bf16; with T in the tens to hundreds they stream the weights from HBM.
//
// Work unit (one CTA): 128 output features (one head of 128 dims for the
// query/key/value projection) x a tile of up to 288 tokens x a range of the
// reduction.  The weights are the MMA's A operand (M = 128 features in the
// TMEM lanes), the rows the B operand (N = tokens in the TMEM columns: one MMA
// of N = tile, or two of N = tile / 2 above 256), so every token count from 1
// up fills the 128-wide M dimension.  The K ranges of one (feature tile, token
// tile) form a thread-block cluster; each CTA writes its fp32 partial sums to
// the workspace (they stay in L2) and, after a cluster barrier, CTA `rank`
// adds the splits' partials of its share of the tokens (in split order, so the
// sum is deterministic) and writes them.  The split count is the largest
// whose clusters all fit on the device at once (one wave).
//
// Epilogues:
//   plain   y [T][N] bf16.
//   qkv     features [0, Hq D) are queries, then Hkv D keys, then Hkv D values;
//           queries and keys get the rotate-half rotary embedding at the zone
//           position of their row (draft d_r at P + r - 1, slot s of block j
//           at P + j + s - 1, the single row of k = 0 at P; P = seq_lens[b]),
//           angle pos * base^(-2f/D) formed in fp64; the results go to
//           q [B][R][Hq][D], k_blk and v_blk [B][R][Hkv][D], the layouts
//           tidar_step_attn reads.
//
// Roles (6 warps): warp 0 TMA producer (the weight tiles of the first stages
// are issued before the wait on the previous kernel: they do not depend on
// it); warp 1 TMEM owner and MMA issuer; warps 2..5 move the accumulator from
// TMEM (lane quarter warp % 4) to the workspace (to shared memory with one
// split); all six warps then reduce and write, one warp per token and several
// tokens' loads in flight.  Every mbarrier wait is bounded (~1 s): on expiry
// the CTA records TIDAR_DEVERR_TIMEOUT, skips the rest of its work, marks its
// partials invalid (the other splits of its cluster then write nothing for
// the tile), still meets its cluster at the barrier, frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace tidar {

namespace {

constexpr int kLinThreads = 192;
constexpr int kLinMaxStages = 8;
constexpr uint32_t kLinATile = 128u * 128u;              // 128 features x 64 bf16 (128 B rows)
constexpr uint32_t kLinSmemBudget = 225u * 1024u;        // ring + barriers, under the 227 KB limit
constexpr int kLinMaxTile = 288;                         // tokens per CTA (TMEM columns)
constexpr int kLinMaxSplit = 8;                          // K splits (cluster size)

struct LinParams {
  int T, K, N;        // tokens, reduction length, output features
  int nt;             // tokens per tile (multiple of 16; of 32 when two MMAs)
  int nsub;           // MMAs per 16-wide K step: 1 (nt <= 256) or 2
  int stages;
  int ksplit;         // cluster size along the reduction
  int kb_total;       // K / 64
  uint32_t stage_bytes;
  int mode;           // 0 plain, 1 qkv + rotary embedding
  void* y;
  void* q;
  void* kb;
  void* vb;
  const int32_t* seq_lens;
  int Hq, Hkv, R, kdraft, max_prefix;
  double log2_base;
  unsigned int* err;
  float* part;        // [tiles][N / 128][ksplit][nt][128] fp32 split partials (ksplit > 1)
  int* stat;          // [tiles][N / 128][ksplit]: 0 when that split's partials are valid
};

// Optional timeline of CTA (0, 0, 0) (build with -DTIDAR_TRACE; absent from
// normal builds): [0] setup, [1] weights of the first stages issued, [2]
// after the wait on the previous kernel, [16 + i] producer issues k-block i,
// [144 + i] the MMA thread sees k-block i, [272] accumulator done, [273]
// partials in shared memory, [274] merged and written; [512 + 2 cta] start /
// end of every CTA.
#ifdef TIDAR_TRACE
__device__ unsigned long long g_lin_trace[512 + 2 * 4096];
#define LIN_TRACE(slot) do { if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (slot) < 512) \
    g_lin_trace[(slot)] = global_ns(); } while (0)
#define LIN_TRACE_CTA(w) do { const unsigned c_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
    if (c_ < 4096) g_lin_trace[512 + 2 * c_ + (w)] = global_ns(); } while (0)
#else
#define LIN_TRACE(slot) do {} while (0)
#define LIN_TRACE_CTA(w) do {} while (0)
#endif

__device__ __forceinline__ void lin_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void lin_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major SWIZZLE_128B shared-memory matrix descriptor (8-row groups 1024 B
// apart, sm_100 descriptor version); the K offset inside the 128-byte row is
// added to the start address.
__device__ __forceinline__ uint64_t lin_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both K-major.
__device__ __forceinline__ uint32_t lin_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void lin_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void lin_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ uint32_t lin_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
#define LIN_R16(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
    "=r"(r[i + 6]), "=r"(r[i + 7]), "=r"(r[i + 8]), "=r"(r[i + 9]), "=r"(r[i + 10]), "=r"(r[i + 11]),         \
    "=r"(r[i + 12]), "=r"(r[i + 13]), "=r"(r[i + 14]), "=r"(r[i + 15])
// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void lin_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : LIN_R16(0)
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Position of query row `row` of a sequence whose settled prefix is P.
__device__ __forceinline__ long long zone_position(int k, int row, int P) {
  if (k == 0 || row < k) return (long long)P + row;     // d_r (r = row + 1) at P + r - 1
  const int j = (row - k) / k + 1, s = (row - k) % k + 1;
  return (long long)P + j + s - 1;
}

// (token tile, feature tile) group of a CTA, and the first float of split
// `split`'s partials in the workspace.
__device__ __forceinline__ int lin_group(const LinParams& prm, int tt, int ft) { return tt * (prm.N / 128) + ft; }
__device__ __forceinline__ size_t lin_part_offset(const LinParams& prm, int tt, int ft, int split) {
  return ((size_t)lin_group(prm, tt, ft) * prm.ksplit + split) * (size_t)prm.nt * 128;
}

// Sum of the KS splits' partials of tokens [tlo, thi) of the tile and the
// epilogue.  One warp per token, lane l holding features 4l .. 4l+3; each warp
// has U tokens' loads (KS float4 each, from L2 -- other SMs wrote them -- or
// from shared memory with one split) in flight before it adds them in split
// order.  The rotary pairs (f, f + 64) sit in lanes l and l ^ 16.
template <int KS>
__device__ __forceinline__ void lin_reduce(const LinParams& prm, const float* part, int tlo, int thi, int t0,
                                           int ft, int warp, int lane, const double* invf) {
  constexpr int U = KS == 1 ? 4 : (KS <= 2 ? 8 : (KS <= 4 ? 4 : 2));
  constexpr int W = kLinThreads / 32;
  const size_t split_stride = (size_t)prm.nt * 128;
  for (int tb = tlo + warp; tb < thi; tb += W * U) {
    float4 v[U][KS];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = tb + W * u;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        if (t < thi) {
          const float4* src = reinterpret_cast<const float4*>(part + s * split_stride + (size_t)t * 128) + lane;
          v[u][s] = KS == 1 ? *src : __ldcg(src);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = tb + W * u;
      if (t >= thi) break;                                // warp-uniform
      float acc[4] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w};
#pragma unroll
      for (int s = 1; s < KS; ++s) {
        acc[0] += v[u][s].x; acc[1] += v[u][s].y; acc[2] += v[u][s].z; acc[3] += v[u][s].w;
      }
      const int tg = t0 + t;
      __nv_bfloat16* dst;
      if (prm.mode == 0) {
        dst = static_cast<__nv_bfloat16*>(prm.y) + (size_t)tg * prm.N + ft * 128;
      } else {
        const int b = tg / prm.R, row = tg % prm.R;
        bool rotate = true;
        if (ft < prm.Hq) {
          dst = static_cast<__nv_bfloat16*>(prm.q) + ((size_t)tg * prm.Hq + ft) * 128;
        } else if (ft < prm.Hq + prm.Hkv) {
          dst = static_cast<__nv_bfloat16*>(prm.kb) + ((size_t)tg * prm.Hkv + (ft - prm.Hq)) * 128;
        } else {
          dst = static_cast<__nv_bfloat16*>(prm.vb) + ((size_t)tg * prm.Hkv + (ft - prm.Hq - prm.Hkv)) * 128;
          rotate = false;
        }
        if (rotate) {                                     // warp-uniform
          int P = prm.seq_lens[b];
          if (P < 0 || P > prm.max_prefix) {
            if (lane == 0 && row == 0 && ft == 0 && blockIdx.y == 0) raise_error(prm.err, TIDAR_DEVERR_BAD_LEN);
            P = 0;
          }
          const double pos = (double)zone_position(prm.kdraft, row, P);
          const bool hi = lane >= 16;                     // features 64 .. 127: the second of each pair
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float other = __shfl_xor_sync(0xffffffffu, acc[e], 16);
            const double ang = pos * invf[4 * (lane & 15) + e];
            const double red = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
            float sn, cs;
            sincosf((float)red, &sn, &cs);
            // (x_f, x_{f+64}) -> (x_f cos - x_{f+64} sin, x_f sin + x_{f+64} cos)
            acc[e] = hi ? other * sn + acc[e] * cs : acc[e] * cs - other * sn;
          }
        }
      }
      uint2 u2;
      u2.x = lin_bf16x2(acc[0], acc[1]);
      u2.y = lin_bf16x2(acc[2], acc[3]);
      *reinterpret_cast<uint2*>(dst + 4 * lane) = u2;
    }
  }
}

__global__ void __launch_bounds__(kLinThreads, 1)
linear_tc05_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                   const LinParams prm) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Every CTA of the cluster must reach both cluster barriers: a CTA whose
  // layout check fails still takes part in them (doing no work).
  const bool layout_ok = (sb & 1023u) == 0;
  const int ft = blockIdx.x, split = blockIdx.y, tt = blockIdx.z;
  const int t0 = tt * prm.nt;
  const int nvalid = min(prm.nt, prm.T - t0);             // real tokens in this tile
  const int kb0 = (int)((long long)split * prm.kb_total / prm.ksplit);
  const int kb1 = (int)((long long)(split + 1) * prm.kb_total / prm.ksplit);
  const int nkb = kb1 - kb0;                              // >= 1 (ksplit <= kb_total)
  const uint32_t ring = (uint32_t)prm.stages * prm.stage_bytes;
  auto bar = [&](int i) -> uint32_t { return sb + ring + 8u * i; };   // full[s], empty[s], done
  const int BAR_FULL = 0, BAR_EMPTY = kLinMaxStages, BAR_DONE = 2 * kLinMaxStages;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + ring + 8u * (2 * kLinMaxStages + 1));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  double* invf = reinterpret_cast<double*>(smem + ring + 8u * (2 * kLinMaxStages + 1) + 16);   // [64]

  if (threadIdx.x == 0) { LIN_TRACE_CTA(0); LIN_TRACE(0); }
  if (threadIdx.x == 0) {
    // the other CTAs of the cluster read this flag before trusting this CTA's
    // partials, so it is set even when the layout check fails
    *abort_flag = layout_ok ? 0 : 1;
    if (layout_ok) {
      prefetch_tmap(&tm_w);      // kernel parameters: safe before the dependency wait
      prefetch_tmap(&tm_x);
      for (int i = 0; i < 2 * kLinMaxStages + 1; ++i) mbar_init(bar(i), 1u);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
  }
  if (layout_ok && prm.mode == 1 && threadIdx.x < 64) {
    // inverse frequencies base^(-2f/128) of the rotary pairs, fp64
    invf[threadIdx.x] = exp2(-(2.0 * threadIdx.x / 128.0) * prm.log2_base);
  }
  if (layout_ok && warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + ring + 8u * (2 * kLinMaxStages + 1)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  lin_fence_before();
  __syncthreads();
  lin_fence_after();
  const uint32_t tmem = layout_ok ? misc[0] : 0u;
  if (!layout_ok && threadIdx.x == 0) raise_error(prm.err, TIDAR_DEVERR_LAYOUT);

  const int nsubn = prm.nt / prm.nsub;                    // tokens per MMA
  const uint32_t a_bytes = kLinATile, b_bytes = (uint32_t)prm.nt * 128u;

  if (!layout_ok) {
    pdl_wait();
    pdl_trigger();
  } else if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // The weight tiles of the first stages do not depend on the previous
    // kernel: they are issued before the wait, the token tiles after it.
    const int pre = min(prm.stages, nkb);
    if (lane == 0) {
      for (int i = 0; i < pre; ++i) {
        const uint32_t dst = sb + (uint32_t)i * prm.stage_bytes;
        mbar_expect_tx(bar(BAR_FULL + i), a_bytes + b_bytes);
        tma_load_2d(dst, &tm_w, (kb0 + i) * 64, ft * 128, bar(BAR_FULL + i));
      }
      LIN_TRACE(1);
    }
    pdl_wait();
    pdl_trigger();
    if (lane == 0) LIN_TRACE(2);
    if (lane == 0) {
      int issued = pre;          // stages whose copies were (at least partly) issued
      for (int i = 0; i < nkb; ++i) {
        const int s = i % prm.stages;
        const uint32_t dst = sb + (uint32_t)s * prm.stage_bytes;
        if (i >= pre) {
          if (!wait_bar(bar(BAR_EMPTY + s), (uint32_t)((i / prm.stages - 1) & 1), abort_flag, prm.err)) break;
          mbar_expect_tx(bar(BAR_FULL + s), a_bytes + b_bytes);
          tma_load_2d(dst, &tm_w, (kb0 + i) * 64, ft * 128, bar(BAR_FULL + s));
          issued = i + 1;
        }
        LIN_TRACE(16 + min(i, 127));
        for (int u = 0; u < prm.nsub; ++u)
          tma_load_2d(dst + a_bytes + (uint32_t)u * nsubn * 128u, &tm_x, (kb0 + i) * 64, t0 + u * nsubn,
                      bar(BAR_FULL + s));
      }
      if (*abort_flag) {
        // drain: no copy may still write shared memory when the CTA moves on
        // (every issued stage got both its weight and its token tiles)
        for (int i = max(0, issued - prm.stages); i < issued; ++i)
          wait_quiet(bar(BAR_FULL + i % prm.stages), (uint32_t)((i / prm.stages) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {
      const uint32_t idesc = lin_idesc(nsubn);
      int i = 0;
      for (; i < nkb; ++i) {
        const int s = i % prm.stages;
        if (!wait_bar(bar(BAR_FULL + s), (uint32_t)((i / prm.stages) & 1), abort_flag, prm.err)) break;
        LIN_TRACE(144 + min(i, 127));
        lin_fence_after();
        const uint32_t a = sb + (uint32_t)s * prm.stage_bytes, b = a + a_bytes;
#pragma unroll
        for (int kc = 0; kc < 4; ++kc)
          for (int u = 0; u < prm.nsub; ++u)
            lin_mma(tmem + (uint32_t)(u * nsubn), lin_desc(a + kc * 32), lin_desc(b + (uint32_t)u * nsubn * 128u + kc * 32),
                    idesc, (i > 0 || kc > 0) ? 1u : 0u);
        lin_commit(bar(BAR_EMPTY + s));
      }
      // every MMA issued above has completed before the accumulator is read
      lin_commit(bar(BAR_DONE));
    }
  } else {
    // ---------------------------------------------------------------- TMEM -> partials
    pdl_wait();
    pdl_trigger();
    const int q4 = warp & 3;
    const int f = 32 * q4 + lane;
    bool ok = warp_wait_bar(bar(BAR_DONE), 0, abort_flag, prm.err);
    ok = __all_sync(0xffffffffu, ok && !*abort_flag);     // tcgen05.ld needs the whole warp
    if (threadIdx.x == 64) LIN_TRACE(272);
    lin_fence_after();
    if (ok) {
      // one split: [nt][128] in shared memory (the ring is idle now); several:
      // this split's slice of the workspace, token-major, so a warp's 32
      // features of one token are one 128-byte line
      float* part = prm.ksplit > 1 ? prm.part + lin_part_offset(prm, tt, ft, split) : reinterpret_cast<float*>(smem);
      const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
      for (int c = 0; c < nvalid; c += 16) {
        uint32_t r[16];
        lin_tmem_ld16(trow + (uint32_t)c, r);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (c + e < nvalid) part[(c + e) * 128 + f] = __uint_as_float(r[e]);
      }
    }
  }
  lin_fence_before();
  __syncthreads();
  const bool cta_ok = layout_ok && !*abort_flag;
  if (threadIdx.x == 0) LIN_TRACE(273);
  const int ks = prm.ksplit;
  if (ks > 1) {
    // every split's partials and status word are written before any CTA of
    // the cluster reads them (release / acquire at cluster scope)
    if (threadIdx.x == 0) prm.stat[lin_group(prm, tt, ft) * ks + split] = cta_ok ? 0 : 1;
    cluster_sync_all();
  }

  // ------------------------------------------------------------------ reduce + write
  // CTA `rank` owns tokens [rank * per, (rank + 1) * per) of the tile.  A
  // split that timed out or failed its layout check leaves garbage, so every
  // CTA checks all status words first and writes nothing for the tile if one
  // is set (the error word already says why).
  const uint32_t rank = ks > 1 ? cluster_rank() : 0u;
  const int per = (nvalid + ks - 1) / ks;
  const int tlo = (int)rank * per, thi = min(nvalid, tlo + per);
  bool all_ok = cta_ok;
  if (ks > 1) {
    const int* st = prm.stat + lin_group(prm, tt, ft) * ks;
    for (int r2 = 0; r2 < ks; ++r2) all_ok = all_ok && __ldcg(st + r2) == 0;
  }
  if (all_ok) {
    switch (ks) {
      case 1: lin_reduce<1>(prm, reinterpret_cast<const float*>(smem), tlo, thi, t0, ft, warp, lane, invf); break;
      case 2: lin_reduce<2>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      case 3: lin_reduce<3>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      case 4: lin_reduce<4>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      case 5: lin_reduce<5>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      case 6: lin_reduce<6>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      case 7: lin_reduce<7>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
      default: lin_reduce<8>(prm, prm.part + lin_part_offset(prm, tt, ft, 0), tlo, thi, t0, ft, warp, lane, invf); break;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) { LIN_TRACE(274); LIN_TRACE_CTA(1); }
  if (layout_ok && warp == 1) {
    lin_fence_after();
    if (lane == 0) wait_quiet(bar(BAR_DONE), 0);
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u) : "memory");
  }
}

// Largest dynamic shared memory of any launch (set once per device).
cudaError_t lin_smem_attr() {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorNotSupported;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(linear_tc05_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLinSmemBudget);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return cudaSuccess;
}

// Clusters of `ks` CTAs (the K splits of one output tile) with `smem` bytes
// each that this device holds at once; 0 if none (or no device).
int lin_resident_clusters(int ks, size_t smem) {
  static int cache[64][kLinMaxSplit + 1][4];
  static size_t cache_smem[64][kLinMaxSplit + 1][4];
  if (ks < 1 || ks > kLinMaxSplit) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) { cudaGetLastError(); return 0; }
  for (int i = 0; i < 4; ++i)
    if (cache[dev][ks][i] && cache_smem[dev][ks][i] == smem) return cache[dev][ks][i] - 1;
  int n = 0;
  if (lin_smem_attr() == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, ks, 1);
    cfg.blockDim = dim3(kLinThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = ks;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, linear_tc05_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  for (int i = 0; i < 4; ++i)
    if (!cache[dev][ks][i]) { cache[dev][ks][i] = n + 1; cache_smem[dev][ks][i] = smem; break; }
  return n;
}

}  // namespace

#ifdef TIDAR_TRACE
extern "C" int tidar_lin_trace_read(void* dst, size_t bytes) {
  return (int)cudaMemcpyFromSymbol(dst, g_lin_trace, bytes);
}
extern "C" int tidar_lin_trace_clear() {
  static unsigned long long zero[512 + 2 * 4096];
  return (int)cudaMemcpyToSymbol(g_lin_trace, zero, sizeof zero);
}
#endif

LinearPlan plan_linear(int T, int K, int N) {
  LinearPlan p{};
  if (T <= 0 || K <= 0 || N <= 0 || K % 64 || N % 128) return p;
  const int pad16 = (T + 15) / 16 * 16;
  if (T <= kLinMaxTile) {
    p.nt = pad16 <= 256 ? pad16 : (T + 31) / 32 * 32;
  } else {
    p.nt = 256;
  }
  p.nsub = p.nt > 256 ? 2 : 1;
  p.tiles = (T + p.nt - 1) / p.nt;
  p.stage_bytes = kLinATile + (uint32_t)p.nt * 128u;
  const uint32_t extra = 8u * (2 * kLinMaxStages + 1) + 16u + 64u * 8u;
  p.stages = (int)((kLinSmemBudget - extra) / p.stage_bytes);
  if (p.stages > kLinMaxStages) p.stages = kLinMaxStages;
  p.smem = p.stages * p.stage_bytes + extra;
  // Split count: the waves of clusters the launch needs times (the k-blocks
  // of one split + a fixed per-CTA cost: ramp-up, partials, the wait for the
  // slowest split of the cluster), plus the reduction through L2, in units of
  // one 64-wide k-block (about 0.5 us with every SM streaming).  Without a
  // device (host-only planning) the occupancy is taken as one cluster per ks
  // SMs.
  const int kb = K / 64;
  const long long base = (long long)(N / 128) * p.tiles;
  constexpr double kFixed = 10.0, kReduce = 1.5;
  double best = 1e300;
  int best_ks = 1;
  for (int ks = 1; ks <= kLinMaxSplit && ks <= kb; ++ks) {
    int resident = ks == 1 ? 148 : lin_resident_clusters(ks, p.smem);
    if (resident <= 0) resident = 148 / ks;
    const long long waves = (base + resident - 1) / resident;
    const double cost = (double)waves * ((double)kb / ks + kFixed) + (ks > 1 ? kReduce : 0.0);
    if (cost < best - 1e-9) { best = cost; best_ks = ks; }
  }
  p.ksplit = best_ks;
  p.ws_bytes = p.ksplit > 1 ? ((base * p.ksplit * (size_t)p.nt * 128 * sizeof(float) + 255) / 256 * 256 +
                                (base * p.ksplit * sizeof(int) + 255) / 256 * 256)
                            : 0;
  p.ok = p.stages >= 4 && (uint32_t)p.nt * 512u <= (uint32_t)p.stages * p.stage_bytes;
  return p;
}

cudaError_t launch_linear(const LinearArgs& a, cudaStream_t s) {
  const LinearPlan p = plan_linear(a.T, a.K, a.N);
  if (!p.ok) return cudaErrorNotSupported;
  if (p.ws_bytes && (!a.ws || (reinterpret_cast<uintptr_t>(a.ws) & 255u))) return cudaErrorInvalidValue;
  LinParams prm{};
  prm.T = a.T; prm.K = a.K; prm.N = a.N;
  prm.nt = p.nt; prm.nsub = p.nsub; prm.stages = p.stages; prm.ksplit = p.ksplit;
  prm.kb_total = a.K / 64; prm.stage_bytes = p.stage_bytes;
  prm.mode = a.mode; prm.y = a.y; prm.q = a.q; prm.kb = a.k_blk; prm.vb = a.v_blk;
  prm.seq_lens = a.seq_lens; prm.Hq = a.Hq; prm.Hkv = a.Hkv; prm.R = a.R; prm.kdraft = a.k;
  prm.max_prefix = a.max_prefix; prm.log2_base = a.log2_base; prm.err = a.err;
  if (p.ws_bytes) {
    const size_t groups = (size_t)(a.N / 128) * p.tiles;
    prm.part = static_cast<float*>(a.ws);
    prm.stat = reinterpret_cast<int*>(static_cast<char*>(a.ws) +
                                      (groups * p.ksplit * (size_t)p.nt * 128 * sizeof(float) + 255) / 256 * 256);
  }
  CUtensorMap tw, tx;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.N};
    const cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    const cuuint32_t box[2] = {64, 128};
    if (!encode(&tw, a.w, 2, dims, str, box)) return cudaErrorNotSupported;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.T};
    const cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(p.nt / p.nsub)};
    if (!encode(&tx, a.x, 2, dims, str, box)) return cudaErrorNotSupported;
  }
  cudaError_t e = lin_smem_attr();
  if (e != cudaSuccess) return e;
  const dim3 grid(a.N / 128, p.ksplit, p.tiles), cluster(1, p.ksplit, 1);
  return launch_clustered(linear_tc05_kernel, grid, cluster, kLinThreads, p.smem, s, tw, tx, prm);
}

}  // namespace tidar
