// api.cu -- the C ABI of libtidar.so: argument checks, launch plans, launches.
//
// Every host-checkable condition is tested before anything is queued; the
// kernels only re-check what depends on device-resident values (page ids,
// lengths, accept counts) and report it through the per-device error word.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "../../include/tidar.h"
#include "common.cuh"
#include "kernels.h"

// Per-device error word (one instance per device that loads the library).
__device__ unsigned int g_tidar_error_word = 0;

namespace {

thread_local char g_cuda_msg[256] = "";
constexpr int kMaxDevices = 64;
// Per-device address of the error word.  Filled under g_err_mutex, so two host
// threads making their first call on a device at once look it up once.
unsigned int* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_err_mutex;

tidar_status cuda_fail(cudaError_t e) {
  snprintf(g_cuda_msg, sizeof g_cuda_msg, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return TIDAR_ERR_CUDA;
}

// Device address of this device's error word (looked up once per device).
tidar_status error_word(unsigned int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return TIDAR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_err_mutex);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_tidar_error_word);
    if (e != cudaSuccess) return cuda_fail(e);
    g_err_ptr[dev] = static_cast<unsigned int*>(p);
  }
  *out = g_err_ptr[dev];
  return TIDAR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace tidar {
unsigned int* device_error_word() {
  unsigned int* p = nullptr;
  return error_word(&p) == TIDAR_OK ? p : nullptr;
}
tidar_status error_word_status(unsigned int** out) { return error_word(out); }
tidar_status cuda_status(cudaError_t e) { return cuda_fail(e); }
}  // namespace tidar

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Shape checks shared by step_attn and commit.
tidar_status check_desc(const tidar_step_desc* d) {
  if (!d) return TIDAR_ERR_INVALID_ARG;
  if (d->batch < 0 || d->num_q_heads <= 0 || d->num_kv_heads <= 0 ||
      d->num_q_heads % d->num_kv_heads != 0 || d->k < 0 || d->max_prefix_len < 0 ||
      d->page_size <= 0)
    return TIDAR_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return TIDAR_ERR_UNSUPPORTED;
  if (d->k > 16) return TIDAR_ERR_UNSUPPORTED;
  if (d->page_size != 16 && d->page_size != 32 && d->page_size != 64 && d->page_size != 128)
    return TIDAR_ERR_UNSUPPORTED;
  if (d->dtype != TIDAR_F32 && d->dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (d->path != TIDAR_PATH_AUTO && d->path != TIDAR_PATH_SIMT && d->path != TIDAR_PATH_TC05 &&
      d->path != TIDAR_PATH_DEC && d->path != TIDAR_PATH_PAIR)
    return TIDAR_ERR_INVALID_ARG;
  return TIDAR_OK;
}

tidar_status check_cache(const tidar_step_desc* d, const tidar_kv_cache* c) {
  if (!c) return TIDAR_ERR_INVALID_ARG;
  const int n = d->k > 0 ? d->k : 1;
  if (c->num_pages <= 0 || c->max_pages_per_seq <= 0) return TIDAR_ERR_INVALID_ARG;
  const long long need = ((long long)d->max_prefix_len + n + d->page_size - 1) / d->page_size;
  if (c->max_pages_per_seq < need) return TIDAR_ERR_INVALID_ARG;
  if (!c->k_pages || !c->v_pages || !c->page_table || !c->seq_lens) return TIDAR_ERR_INVALID_ARG;
  if (!aligned16(c->k_pages) || !aligned16(c->v_pages)) return TIDAR_ERR_INVALID_ARG;
  return TIDAR_OK;
}

constexpr bool kTc05Built = true;

bool tc05_supported(const tidar_step_desc* d) {
  return kTc05Built && d->dtype == TIDAR_BF16 && d->head_dim == 128 && d->page_size == 64;
}

// Warp-MMA decode kernel: at most 16 packed query rows per KV head.
bool dec_supported(const tidar_step_desc* d) {
  return tc05_supported(d) &&
         (long long)tidar::rows_per_seq(d->k) * (d->num_q_heads / d->num_kv_heads) <= 16;
}

constexpr int kNumSMs = 148;

int g_force_partials = 0;   // TIDAR_DEBUG_FORCE_SPLIT_PARTIALS

struct Plan {
  int path;    // 1 SIMT, 2 TC05, 3 DEC, 4 PAIR
  int nsplit;
  int keys_per_split;
  bool cluster_merge;   // splits of a tile form one cluster and merge in the attention kernel
};

// Step-key windows (128 step keys each) the last split of the busiest query
// tile runs on the tensor-core paths (PAIR: a pair of tiles): window 0 (the
// drafts) plus those holding the tile's own mask blocks -- the windows the
// kernels' block plans add, at most 4.
int max_step_windows(const tidar_step_desc* d, int path) {
  const int k = d->k, R = tidar::rows_per_seq(k);
  const int G = d->num_q_heads / d->num_kv_heads;
  const int rows = (path == 4 ? 2 : 1) * (128 / G);
  int most = 1;
  for (int rho0 = 0; rho0 < R; rho0 += rows) {
    const int rho1 = rho0 + rows < R ? rho0 + rows : R;
    int nw = 1;
    if (k > 0 && rho1 - 1 >= k) {
      const int jlo = ((rho0 > k ? rho0 : k) - k) / k + 1;
      const int jhi = (rho1 - 1 - k) / k + 1;
      const int lo = k + (jlo - 1) * k, hi = k + jhi * k;
      for (int w = lo / 128; w <= (hi - 1) / 128 && nw < 4; ++w)
        if (w != 0) ++nw;
    }
    if (nw > most) most = nw;
  }
  return most;
}

// Key ranges are multiples of 128 keys (64 on the decode path).  SIMT: aim for
// ~2 waves of 4-warp CTAs.  TC05 / PAIR / DEC: one CTA per SM and per (b, kv
// head, query tile or pair of tiles, split), split count from a cost model.
Plan make_plan(const tidar_step_desc* d, int path) {
  Plan p;
  p.path = path;
  const int R = tidar::rows_per_seq(d->k);
  const int G = d->num_q_heads / d->num_kv_heads;
  const int M = R * G;
  const int maxP = d->max_prefix_len;
  const int blocks128 = (maxP + 127) / 128;
  long long units;
  int target;
  if (path == 2 || path == 4) {
    const int rows_per_tile = (128 / G) * G;
    const int tiles = (M + rows_per_tile - 1) / rows_per_tile;
    units = (long long)d->batch * d->num_kv_heads * (path == 4 ? (tiles + 1) / 2 : tiles);
    target = kNumSMs;
  } else if (path == 3) {
    units = (long long)d->batch * d->num_kv_heads;
    target = kNumSMs;
  } else {
    units = (long long)d->batch * d->num_kv_heads * ((M + 3) / 4);
    target = 2 * kNumSMs * 4;
  }
  // at least 2 key blocks of 128 per split (tensor-core paths), 2 pages of 64
  // (decode path), 1 block for SIMT
  const int max_ns = path == 3 ? ((maxP + 63) / 64 / 2 > 0 ? (maxP + 63) / 64 / 2 : 1)
                               : ((path == 2 || path == 4) ? (blocks128 / 2 > 0 ? blocks128 / 2 : 1)
                                                           : (blocks128 > 0 ? blocks128 : 1));
  auto split_keys = [&](int n) {
    if (path == 3) {                                  // pages of 64 keys
      const int pages = (maxP + 63) / 64;
      const int pps = (pages + n - 1) / n;
      p.keys_per_split = (pps > 0 ? pps : 1) * 64;
      p.nsplit = maxP > 0 ? (maxP + p.keys_per_split - 1) / p.keys_per_split : 1;
      if (p.nsplit < 1) p.nsplit = 1;
      return;
    }
    // tensor-core paths: the last split also runs the tile's step-key windows
    // (blocks of 128 step keys; a masked block costs about what a prefix block
    // does), so the blocks are dealt out with the busiest tile's windows counted
    // as the last ones: every split holds at most bps blocks, and the last
    // split holds what remains of the prefix (possibly nothing) and the windows
    const int wins = ((path == 2 || path == 4) && n > 1) ? max_step_windows(d, path) : 0;
    const int bps = (blocks128 + wins + n - 1) / n;
    p.keys_per_split = (bps > 0 ? bps : 1) * 128;
    p.nsplit = maxP > 0 ? (blocks128 + wins + bps - 1) / (bps > 0 ? bps : 1) : 1;
    if (p.nsplit < 1) p.nsplit = 1;
  };
  p.cluster_merge = false;
  if (path == 1) {
    // SIMT: aim for ~2 waves of 4-warp CTAs
    int ns = 1;
    if (units > 0 && units < target) ns = (int)((target + units - 1) / units);
    if (ns > max_ns) ns = max_ns;
    if (ns > 64) ns = 64;
    split_keys(ns < 1 ? 1 : ns);
    return p;
  }
  // Tensor-core and decode paths (one CTA per SM): choose the split count by a
  // cost model in units of 128-key blocks per CTA -- the waves of CTAs the
  // launch needs times (the keys of one split + a fixed per-CTA cost), plus
  // the merge: a second launch, or (the splits of a tile forming a cluster of
  // nsplit CTAs) an on-chip merge at the end of the attention kernel, whose
  // waves count the clusters that can be resident at once.
  // A launch that already fills the device (units >= one wave) keeps one split:
  // with ragged batches the longest sequence, not the wave count, sets its time.
  constexpr double kFixedBlocks = 3.0, kFinalizeBlocks = 2.0, kClusterMergeBlocks = 1.0;
  double best = 1e300;
  int best_n = 1;
  bool best_cluster = false;
  int last_ns = -1;
  const int n_hi = units >= target ? 1 : (max_ns < 64 ? max_ns : 64);
  for (int n = 1; n <= n_hi; ++n) {
    split_keys(n);
    if (p.nsplit == last_ns) continue;
    last_ns = p.nsplit;
    const double per = (double)p.keys_per_split / 128.0 + kFixedBlocks;
    const long long ctas = units * p.nsplit;
    const double cost_p = (double)((ctas + target - 1) / target) * per + (p.nsplit > 1 ? kFinalizeBlocks : 0.0);
    if (cost_p < best) { best = cost_p; best_n = n; best_cluster = false; }
    if (p.nsplit > 1 && p.nsplit <= 16 && !g_force_partials) {
      const int resident = path == 2 ? tidar::tc05_resident_clusters(p.nsplit)
                                     : (path == 4 ? tidar::pair_resident_clusters(p.nsplit)
                                                  : tidar::dec_resident_clusters(p.nsplit, M));
      if (resident > 0) {
        const double cost_c = (double)((units + resident - 1) / resident) * per + kClusterMergeBlocks;
        if (cost_c <= best) { best = cost_c; best_n = n; best_cluster = true; }   // ties: on chip
      }
    }
  }
  split_keys(best_n);
  p.cluster_merge = best_cluster && p.nsplit > 1;
  return p;
}

int choose_path(const tidar_step_desc* d) {
  if (d->path == TIDAR_PATH_SIMT) return 1;
  if (d->path == TIDAR_PATH_TC05) return 2;
  if (d->path == TIDAR_PATH_DEC) return 3;
  if (d->path == TIDAR_PATH_PAIR) return 4;
  return dec_supported(d) ? 3 : (tc05_supported(d) ? 2 : 1);
}

}  // namespace

extern "C" {

const char* tidar_status_string(tidar_status s) {
  switch (s) {
    case TIDAR_OK: return "ok";
    case TIDAR_ERR_INVALID_ARG: return "invalid argument";
    case TIDAR_ERR_UNSUPPORTED: return "unsupported configuration";
    case TIDAR_ERR_CUDA: return "CUDA error";
    case TIDAR_ERR_TIMEOUT: return "device-side wait timed out";
    case TIDAR_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

const char* tidar_last_cuda_error(void) { return g_cuda_msg; }

tidar_status tidar_step_attn_plan(const tidar_step_desc* desc, int32_t* path, int32_t* splits,
                                  int32_t* merge) {
  tidar_status st = check_desc(desc);
  if (st != TIDAR_OK) return st;
  const int pth = choose_path(desc);
  if ((pth == 2 || pth == 4) && !tc05_supported(desc)) return TIDAR_ERR_UNSUPPORTED;
  if (pth == 3 && !dec_supported(desc)) return TIDAR_ERR_UNSUPPORTED;
  const Plan p = make_plan(desc, pth);
  if (path) *path = p.path;
  if (splits) *splits = p.nsplit;
  if (merge) *merge = p.nsplit <= 1 ? 0 : (p.cluster_merge ? 1 : 2);
  return TIDAR_OK;
}

size_t tidar_step_attn_workspace_bytes(const tidar_step_desc* d) {
  if (check_desc(d) != TIDAR_OK) return 0;
  const int pth = choose_path(d);
  const Plan p = make_plan(d, pth);
  if (p.nsplit <= 1 || p.cluster_merge) return 0;     // one split, or merged in the kernel
  const size_t rows = (size_t)d->batch * tidar::rows_per_seq(d->k) * d->num_q_heads;
  return align256((size_t)p.nsplit * rows * d->head_dim * sizeof(float)) +
         align256((size_t)p.nsplit * rows * sizeof(float));
}

}  // extern "C"

namespace {

// The step attention; step_keys = 0 restricts every row to the cache's prefix
// (a slice of a longer sequence), append = 0 leaves the cache untouched.
tidar_status step_attn_impl(const tidar_step_desc* d, const tidar_kv_cache* c, const void* q,
                            const void* k_blk, const void* v_blk, void* out, float* lse_out,
                            void* workspace, size_t workspace_bytes, tidar_stream_t stream, int step_keys,
                            int append) {
  tidar_status st = check_desc(d);
  if (st != TIDAR_OK) return st;
  if (d->batch == 0) return TIDAR_OK;
  if ((st = check_cache(d, c)) != TIDAR_OK) return st;
  if (!q || !k_blk || !v_blk || !out) return TIDAR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_blk) || !aligned16(v_blk) || !aligned16(out))
    return TIDAR_ERR_INVALID_ARG;
  const int pth = choose_path(d);
  if ((pth == 2 || pth == 4) && !tc05_supported(d)) return TIDAR_ERR_UNSUPPORTED;
  if (pth == 3 && !dec_supported(d)) return TIDAR_ERR_UNSUPPORTED;
  const Plan p = make_plan(d, pth);
  const size_t need = tidar_step_attn_workspace_bytes(d);
  if (workspace_bytes < need) return TIDAR_ERR_INVALID_ARG;
  if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
    return TIDAR_ERR_INVALID_ARG;
  unsigned int* err = nullptr;
  if ((st = error_word(&err)) != TIDAR_OK) return st;

  tidar::AttnArgs a;
  memset(&a, 0, sizeof a);
  a.q = q; a.k_blk = k_blk; a.v_blk = v_blk;
  a.k_pages = c->k_pages; a.v_pages = c->v_pages;
  a.page_table = c->page_table; a.seq_lens = c->seq_lens;
  a.out = out; a.lse_out = lse_out; a.err = err;
  a.B = d->batch; a.Hq = d->num_q_heads; a.Hkv = d->num_kv_heads; a.G = a.Hq / a.Hkv;
  a.D = d->head_dim; a.k = d->k; a.R = tidar::rows_per_seq(d->k); a.n = d->k > 0 ? d->k : 1;
  a.page_size = d->page_size; a.max_pages = c->max_pages_per_seq; a.num_pages = c->num_pages;
  a.max_prefix = d->max_prefix_len;
  a.nsplit = p.nsplit; a.keys_per_split = p.keys_per_split;
  a.bf16 = d->dtype == TIDAR_BF16;
  a.scale = d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)d->head_dim);
  a.step_keys = step_keys;
  a.append = append;
  a.cluster_merge = p.cluster_merge ? 1 : 0;
  if (p.nsplit > 1 && !p.cluster_merge) {
    const size_t rows = (size_t)a.B * a.R * a.Hq;
    a.part_o = static_cast<float*>(workspace);
    a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          align256((size_t)p.nsplit * rows * a.D * sizeof(float)));
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = pth == 2   ? tidar::launch_attn_tc05(a, s)
                  : pth == 3 ? tidar::launch_attn_dec(a, s)
                  : pth == 4 ? tidar::launch_attn_pair(a, s)
                             : tidar::launch_attn_simt(a, s);
  if (e == cudaErrorNotSupported) return TIDAR_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return cuda_fail(e);
  // Split merge and draft-row append: a second launch for the CUDA-core path
  // and for split partials; the tensor-core and decode kernels do both
  // themselves with one split or with the on-chip cluster merge.
  if ((pth == 1 && append) || (p.nsplit > 1 && !p.cluster_merge)) {
    e = tidar::launch_finalize(a, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return TIDAR_OK;
}

}  // namespace

extern "C" {

tidar_status tidar_step_attn(const tidar_step_desc* d, const tidar_kv_cache* c, const void* q,
                             const void* k_blk, const void* v_blk, void* out, float* lse_out,
                             void* workspace, size_t workspace_bytes, tidar_stream_t stream) {
  return step_attn_impl(d, c, q, k_blk, v_blk, out, lse_out, workspace, workspace_bytes, stream, 1, 1);
}

tidar_status tidar_step_attn_part(const tidar_step_desc* d, const tidar_kv_cache* c, const void* q,
                                  const void* k_blk, const void* v_blk, int32_t flags, void* out,
                                  float* lse_out, void* workspace, size_t workspace_bytes,
                                  tidar_stream_t stream) {
  if (flags & ~(TIDAR_PART_STEP_KEYS | TIDAR_PART_APPEND)) return TIDAR_ERR_INVALID_ARG;
  if (!lse_out) return TIDAR_ERR_INVALID_ARG;
  return step_attn_impl(d, c, q, k_blk, v_blk, out, lse_out, workspace, workspace_bytes, stream,
                        (flags & TIDAR_PART_STEP_KEYS) ? 1 : 0, (flags & TIDAR_PART_APPEND) ? 1 : 0);
}

tidar_status tidar_merge_attn(int32_t nparts, int64_t rows, int32_t head_dim, tidar_dtype dtype,
                              const void* part_o, const float* part_lse, void* out, float* lse_out,
                              tidar_stream_t stream) {
  if (nparts <= 0 || rows < 0) return TIDAR_ERR_INVALID_ARG;
  if (nparts > 64 || (head_dim != 64 && head_dim != 128)) return TIDAR_ERR_UNSUPPORTED;
  if (dtype != TIDAR_F32 && dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (rows == 0) return TIDAR_OK;
  if (!part_o || !part_lse || !out || !aligned16(part_o) || !aligned16(out)) return TIDAR_ERR_INVALID_ARG;
  const cudaError_t e = tidar::launch_merge_parts(nparts, rows, head_dim, dtype == TIDAR_BF16, part_o, part_lse,
                                                  out, lse_out, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

size_t tidar_verify_workspace_bytes(int32_t batch, int32_t k, int32_t vocab, tidar_accept_mode mode) {
  if (batch <= 0 || k < 0 || k > 16 || vocab <= 0) return 0;
  return tidar::verify_workspace_bytes(batch, k, vocab, mode);
}

}  // extern "C"

namespace {

// Shared by tidar_verify and tidar_verify_blockq: draft_block null means
// draft_logits is [B][k-1][V]; else it is the previous step's [B][k][k][V]
// block logits, read through draft_block.
// Host checks of a verification and its launch arguments (nothing queued).
tidar_status verify_prepare(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                            tidar_accept_mode mode, const void* logits, const int32_t* drafts,
                            const void* draft_logits, const int32_t* draft_block,
                            const float* uniforms, const int32_t* block_guesses,
                            int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                            int32_t* selected_block, void* workspace, size_t workspace_bytes,
                            tidar::VerifyArgs& a) {
  if (batch < 0 || k < 0 || vocab <= 0) return TIDAR_ERR_INVALID_ARG;
  if (k > 16) return TIDAR_ERR_UNSUPPORTED;
  if (dtype != TIDAR_F32 && dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (mode != TIDAR_GREEDY && mode != TIDAR_REJECTION) return TIDAR_ERR_INVALID_ARG;
  if (batch == 0) return TIDAR_OK;
  if (!logits || !accept_count || !out_tokens) return TIDAR_ERR_INVALID_ARG;
  if (k > 1 && !drafts) return TIDAR_ERR_INVALID_ARG;
  if (mode == TIDAR_REJECTION && (!uniforms || (k > 1 && !draft_logits)))
    return TIDAR_ERR_INVALID_ARG;
  if (!tidar::verify_grid_ok(batch, k, mode)) return TIDAR_ERR_UNSUPPORTED;
  const size_t need = tidar::verify_workspace_bytes(batch, k, vocab, mode);
  if (workspace_bytes < need ||
      (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))))
    return TIDAR_ERR_INVALID_ARG;
  a = tidar::VerifyArgs{};
  a.B = batch; a.k = k; a.n = k > 0 ? k : 1; a.V = vocab; a.bf16 = dtype == TIDAR_BF16; a.mode = mode;
  a.logits = logits; a.drafts = drafts; a.draft_logits = draft_logits; a.uniforms = uniforms;
  a.draft_block = k > 1 ? draft_block : nullptr;
  a.block_guesses = block_guesses; a.accept_count = accept_count; a.out_tokens = out_tokens;
  a.next_drafts = next_drafts; a.selected_block = selected_block; a.workspace = workspace;
  return error_word(&a.err);
}

tidar_status verify_launch(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                           tidar_accept_mode mode, const void* logits, const int32_t* drafts,
                           const void* draft_logits, const int32_t* draft_block,
                           const float* uniforms, const int32_t* block_guesses,
                           int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                           int32_t* selected_block, void* workspace, size_t workspace_bytes,
                           tidar_stream_t stream) {
  tidar::VerifyArgs a;
  tidar_status st = verify_prepare(batch, k, vocab, dtype, mode, logits, drafts, draft_logits, draft_block,
                                   uniforms, block_guesses, accept_count, out_tokens, next_drafts,
                                   selected_block, workspace, workspace_bytes, a);
  if (st != TIDAR_OK || batch == 0) return st;
  cudaError_t e = tidar::launch_verify(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

// Host checks of a commit and its launch arguments (nothing queued).
tidar_status commit_prepare(const tidar_step_desc* d, const tidar_kv_cache* c, const int32_t* accept_count,
                            int32_t* released_pages, int32_t* num_released, tidar::CommitArgs& a) {
  tidar_status st = check_desc(d);
  if (st != TIDAR_OK) return st;
  if (d->batch == 0) return TIDAR_OK;
  if ((st = check_cache(d, c)) != TIDAR_OK) return st;
  if (!accept_count || !released_pages || !num_released) return TIDAR_ERR_INVALID_ARG;
  if (!tidar::commit_batch_ok(d->batch, d->k, d->page_size)) return TIDAR_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  if ((st = error_word(&err)) != TIDAR_OK) return st;
  a.B = d->batch; a.Hkv = d->num_kv_heads; a.D = d->head_dim; a.k = d->k; a.n = d->k > 0 ? d->k : 1;
  a.page_size = d->page_size; a.elem_bytes = d->dtype == TIDAR_BF16 ? 2 : 4;
  a.max_pages = c->max_pages_per_seq; a.num_pages = c->num_pages;
  a.k_pages = c->k_pages; a.v_pages = c->v_pages; a.page_table = c->page_table;
  a.seq_lens = c->seq_lens; a.accept_count = accept_count; a.released = released_pages;
  a.num_released = num_released; a.err = err;
  return TIDAR_OK;
}

}  // namespace

extern "C" {

tidar_status tidar_verify(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                          tidar_accept_mode mode, const void* logits, const int32_t* drafts,
                          const void* draft_logits, const float* uniforms,
                          const int32_t* block_guesses, int32_t* accept_count,
                          int32_t* out_tokens, int32_t* next_drafts, int32_t* selected_block,
                          void* workspace, size_t workspace_bytes, tidar_stream_t stream) {
  return verify_launch(batch, k, vocab, dtype, mode, logits, drafts, draft_logits, nullptr,
                       uniforms, block_guesses, accept_count, out_tokens, next_drafts,
                       selected_block, workspace, workspace_bytes, stream);
}

tidar_status tidar_verify_blockq(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                 const void* logits, const int32_t* drafts,
                                 const void* prev_block_logits, const int32_t* draft_block,
                                 const float* uniforms, const int32_t* block_guesses,
                                 int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                                 int32_t* selected_block, void* workspace, size_t workspace_bytes,
                                 tidar_stream_t stream) {
  if (k > 1 && batch > 0 && (!prev_block_logits || !draft_block)) return TIDAR_ERR_INVALID_ARG;
  return verify_launch(batch, k, vocab, dtype, TIDAR_REJECTION, logits, drafts, prev_block_logits,
                       draft_block, uniforms, block_guesses, accept_count, out_tokens, next_drafts,
                       selected_block, workspace, workspace_bytes, stream);
}

size_t tidar_verify_sampled_workspace_bytes(int32_t batch, int32_t k, int32_t vocab,
                                            tidar_accept_mode mode) {
  if (batch <= 0 || k < 0 || k > 16 || vocab <= 0) return 0;
  if (mode == TIDAR_GREEDY) return tidar_verify_workspace_bytes(batch, k, vocab, mode);   // tidar_verify's
  return align256(tidar::sampled_verify_workspace_bytes(batch, k));
}

static bool sampling_ok(const tidar_sampling* sp) {
  return sp && sp->temperature > 0.f && sp->top_p > 0.f;   // NaN fails both
}

tidar_status tidar_verify_sampled(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                  tidar_accept_mode mode, const tidar_sampling* sampling,
                                  const void* logits, const int32_t* drafts, const void* draft_logits,
                                  const void* prev_block_logits, const int32_t* draft_block,
                                  const float* uniforms, const int32_t* block_guesses,
                                  int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                                  int32_t* selected_block, void* workspace, size_t workspace_bytes,
                                  tidar_stream_t stream) {
  if (!sampling_ok(sampling)) return TIDAR_ERR_INVALID_ARG;
  if (mode == TIDAR_GREEDY)
    return verify_launch(batch, k, vocab, dtype, mode, logits, drafts, nullptr, nullptr, uniforms,
                         block_guesses, accept_count, out_tokens, next_drafts, selected_block, workspace,
                         workspace_bytes, stream);
  if (batch < 0 || k < 0 || vocab <= 0) return TIDAR_ERR_INVALID_ARG;
  if (k > 16) return TIDAR_ERR_UNSUPPORTED;
  if (dtype != TIDAR_F32 && dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (mode != TIDAR_REJECTION) return TIDAR_ERR_INVALID_ARG;
  if (batch == 0) return TIDAR_OK;
  if (batch > 65535) return TIDAR_ERR_UNSUPPORTED;
  if (!logits || !accept_count || !out_tokens || !uniforms) return TIDAR_ERR_INVALID_ARG;
  const bool blockq = prev_block_logits != nullptr;
  if (k > 1 && (!drafts || (!blockq && !draft_logits) || (blockq && !draft_block)))
    return TIDAR_ERR_INVALID_ARG;
  const size_t need = tidar_verify_sampled_workspace_bytes(batch, k, vocab, mode);
  if (workspace_bytes < need || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return TIDAR_ERR_INVALID_ARG;
  tidar::VerifyArgs a{};
  a.B = batch; a.k = k; a.n = k > 0 ? k : 1; a.V = vocab; a.bf16 = dtype == TIDAR_BF16; a.mode = mode;
  a.logits = logits; a.drafts = drafts; a.uniforms = uniforms;
  a.draft_logits = k > 1 ? (blockq ? prev_block_logits : draft_logits) : nullptr;
  a.draft_block = (k > 1 && blockq) ? draft_block : nullptr;
  a.block_guesses = block_guesses; a.accept_count = accept_count; a.out_tokens = out_tokens;
  a.next_drafts = next_drafts; a.selected_block = selected_block; a.workspace = workspace;
  tidar_status st = error_word(&a.err);
  if (st != TIDAR_OK) return st;
  const cudaError_t e = tidar::launch_sampled_verify(a, (double)sampling->temperature,
                                                     (double)sampling->top_p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

tidar_status tidar_sample_drafts(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                 tidar_accept_mode mode, const tidar_sampling* sampling,
                                 const void* block_logits, const int32_t* selected_block,
                                 const float* uniforms, int32_t* next_drafts, tidar_stream_t stream) {
  if (!sampling_ok(sampling)) return TIDAR_ERR_INVALID_ARG;
  if (batch < 0 || k < 0 || vocab <= 0) return TIDAR_ERR_INVALID_ARG;
  if (k > 16) return TIDAR_ERR_UNSUPPORTED;
  if (dtype != TIDAR_F32 && dtype != TIDAR_BF16) return TIDAR_ERR_UNSUPPORTED;
  if (mode != TIDAR_GREEDY && mode != TIDAR_REJECTION) return TIDAR_ERR_INVALID_ARG;
  if (batch == 0 || k < 2) return TIDAR_OK;
  if (batch > 65535) return TIDAR_ERR_UNSUPPORTED;
  if (!block_logits || !selected_block || !next_drafts || (mode == TIDAR_REJECTION && !uniforms))
    return TIDAR_ERR_INVALID_ARG;
  unsigned int* err = nullptr;
  tidar_status st = error_word(&err);
  if (st != TIDAR_OK) return st;
  const cudaError_t e = tidar::launch_sample_drafts(
      batch, k, vocab, dtype == TIDAR_BF16, mode, (double)sampling->temperature, (double)sampling->top_p,
      block_logits, selected_block, uniforms, next_drafts, err, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

tidar_status tidar_commit(const tidar_step_desc* d, const tidar_kv_cache* c,
                          const int32_t* accept_count, int32_t* released_pages,
                          int32_t* num_released, tidar_stream_t stream) {
  tidar::CommitArgs a{};
  const tidar_status st = commit_prepare(d, c, accept_count, released_pages, num_released, a);
  if (st != TIDAR_OK || d->batch == 0) return st;
  cudaError_t e = tidar::launch_commit(a, nullptr, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

tidar_status tidar_verify_commit(const tidar_step_desc* d, const tidar_kv_cache* c, int32_t vocab,
                                 tidar_dtype dtype, tidar_accept_mode mode, const void* logits,
                                 const int32_t* drafts, const void* draft_logits, const float* uniforms,
                                 const int32_t* block_guesses, int32_t* accept_count, int32_t* out_tokens,
                                 int32_t* next_drafts, int32_t* selected_block, int32_t* released_pages,
                                 int32_t* num_released, void* workspace, size_t workspace_bytes,
                                 tidar_stream_t stream) {
  // every host check of both halves before anything is queued
  tidar::CommitArgs ca{};
  tidar_status st = commit_prepare(d, c, accept_count, released_pages, num_released, ca);
  if (st != TIDAR_OK) return st;
  tidar::VerifyArgs va;
  st = verify_prepare(d->batch, d->k, vocab, dtype, mode, logits, drafts, draft_logits, nullptr, uniforms,
                      block_guesses, accept_count, out_tokens, next_drafts, selected_block, workspace,
                      workspace_bytes, va);
  if (st != TIDAR_OK || d->batch == 0) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (mode == TIDAR_REJECTION) {
    cudaError_t e = tidar::launch_verify(va, s);
    if (e == cudaSuccess) e = tidar::launch_commit(ca, nullptr, s);
    return e == cudaSuccess ? TIDAR_OK : cuda_fail(e);
  }
  // greedy: the chunk statistics, then acceptance and commit in one launch
  cudaError_t e = tidar::launch_greedy_stats(va, s);
  if (e != cudaSuccess) return cuda_fail(e);
  tidar::GreedyAcceptArgs f{};
  f.stats = static_cast<const tidar::ChunkStat*>(workspace);
  f.nchunk = tidar::verify_chunks(vocab);
  f.drafts = drafts; f.block_guesses = block_guesses; f.accept_count = accept_count;
  f.out_tokens = out_tokens; f.next_drafts = next_drafts; f.selected_block = selected_block;
  e = tidar::launch_commit(ca, &f, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

tidar_status tidar_reserve(const tidar_step_desc* d, const tidar_kv_cache* c,
                           const tidar_page_pool* pool, const int32_t* returned_pages,
                           const int32_t* num_returned, tidar_stream_t stream) {
  tidar_status st = check_desc(d);
  if (st != TIDAR_OK) return st;
  if (d->batch == 0) return TIDAR_OK;
  if ((st = check_cache(d, c)) != TIDAR_OK) return st;
  if (!pool || !pool->free_count || pool->capacity < 0 || (pool->capacity > 0 && !pool->free_pages))
    return TIDAR_ERR_INVALID_ARG;
  if (!returned_pages != !num_returned) return TIDAR_ERR_INVALID_ARG;
  if (!tidar::reserve_batch_ok(d->batch)) return TIDAR_ERR_UNSUPPORTED;
  unsigned int* err = nullptr;
  if ((st = error_word(&err)) != TIDAR_OK) return st;
  tidar::ReserveArgs a;
  a.B = d->batch; a.n = d->k > 0 ? d->k : 1; a.page_size = d->page_size;
  a.max_prefix = d->max_prefix_len; a.max_pages = c->max_pages_per_seq; a.num_pages = c->num_pages;
  a.capacity = pool->capacity; a.page_table = c->page_table; a.seq_lens = c->seq_lens;
  a.free_pages = pool->free_pages; a.free_count = pool->free_count;
  a.returned = returned_pages; a.num_returned = num_returned; a.err = err;
  cudaError_t e = tidar::launch_reserve(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

size_t tidar_linear_workspace_bytes(int32_t rows, int32_t out_features, int32_t in_features) {
  if (rows <= 0 || out_features <= 0 || in_features <= 0) return 0;
  const tidar::LinearPlan p = tidar::plan_linear(rows, in_features, out_features);
  return p.ok ? p.ws_bytes : 0;
}

tidar_status tidar_linear(int32_t rows, int32_t out_features, int32_t in_features, tidar_dtype dtype,
                          const void* x, const void* w, void* y, void* workspace, size_t workspace_bytes,
                          tidar_stream_t stream) {
  if (rows < 0 || out_features <= 0 || in_features <= 0) return TIDAR_ERR_INVALID_ARG;
  if (dtype != TIDAR_BF16 || in_features % 64 || out_features % 128) return TIDAR_ERR_UNSUPPORTED;
  if (rows == 0) return TIDAR_OK;
  if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y)) return TIDAR_ERR_INVALID_ARG;
  const tidar::LinearPlan p = tidar::plan_linear(rows, in_features, out_features);
  if (!p.ok) return TIDAR_ERR_UNSUPPORTED;
  if (workspace_bytes < p.ws_bytes || (p.ws_bytes && !workspace) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return TIDAR_ERR_INVALID_ARG;
  tidar::LinearArgs a{};
  a.T = rows; a.K = in_features; a.N = out_features; a.mode = 0;
  a.x = x; a.w = w; a.y = y; a.ws = workspace;
  tidar_status st = error_word(&a.err);
  if (st != TIDAR_OK) return st;
  const cudaError_t e = tidar::launch_linear(a, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return TIDAR_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

size_t tidar_qkv_rope_workspace_bytes(const tidar_step_desc* d, int32_t d_model) {
  if (check_desc(d) != TIDAR_OK || d_model <= 0 || d->batch <= 0) return 0;
  const long long T = (long long)d->batch * tidar::rows_per_seq(d->k);
  if (T > 0x7fffffffLL) return 0;
  return tidar_linear_workspace_bytes((int32_t)T, (d->num_q_heads + 2 * d->num_kv_heads) * 128, d_model);
}

tidar_status tidar_qkv_rope(const tidar_step_desc* d, int32_t d_model, const void* x, const void* w_qkv,
                            const int32_t* seq_lens, float rope_base, void* q, void* k_blk, void* v_blk,
                            void* workspace, size_t workspace_bytes, tidar_stream_t stream) {
  tidar_status st = check_desc(d);
  if (st != TIDAR_OK) return st;
  if (d_model <= 0 || !(rope_base > 1.0f)) return TIDAR_ERR_INVALID_ARG;
  if (d->dtype != TIDAR_BF16 || d->head_dim != 128 || d_model % 64) return TIDAR_ERR_UNSUPPORTED;
  if (d->batch == 0) return TIDAR_OK;
  if (!x || !w_qkv || !seq_lens || !q || !k_blk || !v_blk) return TIDAR_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q) || !aligned16(k_blk) || !aligned16(v_blk))
    return TIDAR_ERR_INVALID_ARG;
  const int R = tidar::rows_per_seq(d->k);
  const long long T = (long long)d->batch * R;
  if (T > 0x7fffffffLL) return TIDAR_ERR_UNSUPPORTED;
  const int N = (d->num_q_heads + 2 * d->num_kv_heads) * 128;
  const tidar::LinearPlan p = tidar::plan_linear((int)T, d_model, N);
  if (!p.ok) return TIDAR_ERR_UNSUPPORTED;
  if (workspace_bytes < p.ws_bytes || (p.ws_bytes && !workspace) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return TIDAR_ERR_INVALID_ARG;
  tidar::LinearArgs a{};
  a.T = (int)T; a.K = d_model; a.N = N; a.mode = 1; a.ws = workspace;
  a.x = x; a.w = w_qkv; a.q = q; a.k_blk = k_blk; a.v_blk = v_blk; a.seq_lens = seq_lens;
  a.Hq = d->num_q_heads; a.Hkv = d->num_kv_heads; a.R = R; a.k = d->k; a.max_prefix = d->max_prefix_len;
  a.log2_base = log2((double)rope_base);
  if ((st = error_word(&a.err)) != TIDAR_OK) return st;
  const cudaError_t e = tidar::launch_linear(a, reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return TIDAR_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return cuda_fail(e);
  return TIDAR_OK;
}

}  // extern "C"

namespace {
// Byte offsets of the layer step's workspace: q, k_blk, v_blk, attention
// output, the projections' split partials (the two projections run one after
// the other and share them), then the step attention's own workspace.
struct LayerWs {
  size_t q, kb, vb, o, lin, attn, total;
};
LayerWs layer_ws(const tidar_step_desc* d, int d_model) {
  LayerWs w{};
  const size_t rows = (size_t)d->batch * tidar::rows_per_seq(d->k);
  const size_t qb = rows * d->num_q_heads * 128 * 2, kvb = rows * d->num_kv_heads * 128 * 2;
  const size_t lin_qkv = tidar_qkv_rope_workspace_bytes(d, d_model);
  const size_t lin_o = tidar_linear_workspace_bytes((int32_t)rows, d_model, d->num_q_heads * 128);
  w.q = 0;
  w.kb = w.q + align256(qb);
  w.vb = w.kb + align256(kvb);
  w.o = w.vb + align256(kvb);
  w.lin = w.o + align256(qb);
  w.attn = w.lin + align256(lin_qkv > lin_o ? lin_qkv : lin_o);
  w.total = w.attn + align256(tidar_step_attn_workspace_bytes(d));
  return w;
}
}  // namespace

extern "C" {

size_t tidar_layer_step_workspace_bytes(const tidar_step_desc* d, int32_t d_model) {
  if (check_desc(d) != TIDAR_OK || d_model <= 0) return 0;
  return layer_ws(d, d_model).total;
}

tidar_status tidar_layer_step(const tidar_step_desc* d, const tidar_kv_cache* c, int32_t d_model,
                              const void* x, const void* w_qkv, const void* w_o, float rope_base, void* y,
                              float* lse_out, void* workspace, size_t workspace_bytes,
                              tidar_stream_t stream) {
  tidar_status st = check_desc(d);
  if (st != TIDAR_OK) return st;
  if (d_model <= 0) return TIDAR_ERR_INVALID_ARG;
  if (d->dtype != TIDAR_BF16 || d->head_dim != 128 || d_model % 128) return TIDAR_ERR_UNSUPPORTED;
  if (d->batch == 0) return TIDAR_OK;
  if ((st = check_cache(d, c)) != TIDAR_OK) return st;
  if (!w_o || !y || !aligned16(w_o) || !aligned16(y)) return TIDAR_ERR_INVALID_ARG;
  const LayerWs w = layer_ws(d, d_model);
  if (workspace_bytes < w.total || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return TIDAR_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  const int rows = d->batch * tidar::rows_per_seq(d->k);
  if (!tidar::plan_linear(rows, d->num_q_heads * 128, d_model).ok) return TIDAR_ERR_UNSUPPORTED;
  st = tidar_qkv_rope(d, d_model, x, w_qkv, c->seq_lens, rope_base, ws + w.q, ws + w.kb, ws + w.vb,
                      ws + w.lin, w.attn - w.lin, stream);
  if (st != TIDAR_OK) return st;
  st = tidar_step_attn(d, c, ws + w.q, ws + w.kb, ws + w.vb, ws + w.o, lse_out, ws + w.attn,
                       workspace_bytes - w.attn, stream);
  if (st != TIDAR_OK) return st;
  return tidar_linear(rows, d_model, d->num_q_heads * 128, TIDAR_BF16, ws + w.o, w_o, y, ws + w.lin,
                      w.attn - w.lin, stream);
}

tidar_status tidar_debug_set(tidar_debug_knob knob, int32_t value) {
  switch (knob) {
    case TIDAR_DEBUG_STARVE_ATTENTION_LOADS: tidar::set_starve_loads(value != 0); return TIDAR_OK;
    case TIDAR_DEBUG_FORCE_SPLIT_PARTIALS: g_force_partials = value != 0; return TIDAR_OK;
  }
  return TIDAR_ERR_INVALID_ARG;
}

tidar_status tidar_get_device_status(tidar_stream_t stream, uint32_t* bits_out) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int bits = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&bits, g_tidar_error_word, sizeof bits);
  if (e != cudaSuccess) return cuda_fail(e);
  if (bits) {
    e = cudaMemcpyToSymbol(g_tidar_error_word, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (bits_out) *bits_out = bits;
  if (bits & TIDAR_DEVERR_TIMEOUT) return TIDAR_ERR_TIMEOUT;
  if (bits) return TIDAR_ERR_DEVICE;
  return TIDAR_OK;
}

}  // extern "C"
