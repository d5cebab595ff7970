// kernels.h -- host-side launch interface between api.cu and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tidar.h"

namespace tidar {

// Everything a step-attention kernel needs, in device pointers and sizes.
struct AttnArgs {
  const void* q;
  const void* k_blk;
  const void* v_blk;
  const void* k_pages;
  const void* v_pages;
  const int32_t* page_table;
  const int32_t* seq_lens;
  void* out;
  float* lse_out;        // may be null
  float* part_o;         // [nsplit][B][R][Hq][D] fp32 (nsplit > 1)
  float* part_lse;       // [nsplit][B][R][Hq]  fp32 (nsplit > 1)
  unsigned int* err;     // device error word
  int B, Hq, Hkv, G, D, k, R, n, page_size, max_pages, num_pages, max_prefix;
  int nsplit, keys_per_split;
  int bf16;              // 1: bf16 tensors, 0: fp32
  float scale;           // softmax scale (natural-log domain)
  int step_keys;         // 1: the last split also attends the step keys (the zone mask); 0: prefix only
  int append;            // 1: write the draft rows' K/V into the cache
  int cluster_merge;     // nsplit > 1: the splits of a tile are one cluster and merge in the kernel
                         // (part_o unused); 0: partials in part_o / part_lse, a finalize launch merges
};

// Warp-MMA kernel for query blocks of at most 16 packed rows per KV head
// (bf16, D 128, page 64; splits in multiples of 64 keys).  With cluster_merge
// its nsplit CTAs form a cluster and merge over distributed shared memory (and
// the kernel appends the draft rows itself); without it the splits write
// part_o / part_lse and launch_finalize merges and appends.
cudaError_t launch_attn_dec(const AttnArgs& a, cudaStream_t s);
int dec_resident_clusters(int ns, int M);   // M = packed query rows per KV head
// CUDA-core kernel (fp32 or bf16, D 64 or 128).
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s);
// tcgen05/TMEM kernel (bf16, D 128, page 64).  Returns cudaErrorNotSupported if
// the tensor maps cannot be built.
cudaError_t launch_attn_tc05(const AttnArgs& a, cudaStream_t s);
// How many clusters of `ns` tcgen05 attention CTAs (one per key split) this
// device holds at once; 0 if none.  With cluster_merge the splits form such a
// cluster and merge over distributed shared memory (and the kernel performs
// the draft-row append), else they write part_o / part_lse and
// launch_finalize merges and appends.
int tc05_resident_clusters(int ns);
// Tensor-core kernel with two 128-row query tiles per CTA sharing each staged
// K/V block (bf16, D 128, page 64), for query blocks of more than one tile per
// KV head.  Split merge and append as launch_attn_tc05.
cudaError_t launch_attn_pair(const AttnArgs& a, cudaStream_t s);
int pair_resident_clusters(int ns);
// Test hook: launches issue no K/V copies (their bounded waits run out).
void set_starve_loads(int on);
int tc05_starve_loads();
// Split merge (when nsplit > 1) and the draft-row append, in one launch
// (CUDA-core path).
cudaError_t launch_finalize(const AttnArgs& a, cudaStream_t s);
// Log-sum-exp merge of attention results over disjoint key sets: part_o
// [nparts][rows][D] (dtype), part_lse [nparts][rows] -> out, lse_out.
cudaError_t launch_merge_parts(int nparts, long long rows, int D, int bf16, const void* part_o,
                               const float* part_lse, void* out, float* lse_out, cudaStream_t s);

struct VerifyArgs {
  int B, k, n, V, bf16, mode;
  const void* logits;
  const int32_t* drafts;
  const void* draft_logits;
  // Rejection: null when draft_logits is [B][k-1][V] (q_i in row i-1); else
  // draft_logits is the previous step's block logits [B][k][k][V] and q_i is
  // block draft_block[b] (1..k; outside -> block 1, TIDAR_DEVERR_BAD_COUNT),
  // slot i+1.
  const int32_t* draft_block;
  const float* uniforms;
  const int32_t* block_guesses;
  int32_t* accept_count;
  int32_t* out_tokens;
  int32_t* next_drafts;
  int32_t* selected_block;
  void* workspace;
  unsigned int* err;     // device error word (a bounded wait that ran out)
};
// This device's error word (looked up once per device); nullptr on failure.
unsigned int* device_error_word();
// The same lookup as a status (TIDAR_ERR_CUDA with the message recorded for
// tidar_last_cuda_error on failure).
tidar_status error_word_status(unsigned int** out);
// Records a CUDA error's name and text for tidar_last_cuda_error and returns
// TIDAR_ERR_CUDA.
tidar_status cuda_status(cudaError_t e);
size_t verify_workspace_bytes(int B, int k, int V, int mode);
bool verify_grid_ok(int B, int k, int mode);   // launch grid fits (grid.y <= 65535)
cudaError_t launch_verify(const VerifyArgs& a, cudaStream_t s);
// Rejection verification under temperature / nucleus truncation: per-row
// distribution descriptors into a.workspace, then one CTA per sequence.
size_t sampled_verify_workspace_bytes(int B, int k);
cudaError_t launch_sampled_verify(const VerifyArgs& a, double temp, double top_p, cudaStream_t s);
// The next drafts from slots 2..k of each sequence's selected mask block.
cudaError_t launch_sample_drafts(int B, int k, int V, int bf16, int mode, double temp, double top_p,
                                 const void* block_logits, const int32_t* selected_block,
                                 const float* uniforms, int32_t* next_drafts, unsigned int* err,
                                 cudaStream_t s);

// Exact (max, argmax) of one 4096-wide chunk of a logits row (lowest index on
// ties) and, in rejection mode, the fp64 sum of exp(x - max) over it.
struct ChunkStat {
  float max;
  int arg;
  double sum;
};
// Launches the per-chunk statistics of the B n logits rows of a greedy
// verification into a.workspace ([B n][chunks] ChunkStat).
cudaError_t launch_greedy_stats(const VerifyArgs& a, cudaStream_t s);
int verify_chunks(int V);
// Greedy acceptance from those statistics, for the commit kernel to run it in
// the same launch (tidar_verify_commit): its outputs as tidar_verify's.
struct GreedyAcceptArgs {
  const ChunkStat* stats;
  int nchunk;
  const int32_t* drafts;
  const int32_t* block_guesses;
  int32_t* accept_count;
  int32_t* out_tokens;
  int32_t* next_drafts;
  int32_t* selected_block;
};

struct CommitArgs {
  int B, Hkv, D, k, n, page_size, elem_bytes, max_pages, num_pages;
  void* k_pages;
  void* v_pages;
  int32_t* page_table;
  int32_t* seq_lens;
  const int32_t* accept_count;
  int32_t* released;
  int32_t* num_released;
  unsigned int* err;
};
bool commit_batch_ok(int B, int k, int page_size);   // per-sequence records fit shared memory
// fused == nullptr: the accept counts come from a.accept_count; else the
// kernel computes them (greedy) from fused->stats and writes the
// verification outputs too.
cudaError_t launch_commit(const CommitArgs& a, const GreedyAcceptArgs* fused, cudaStream_t s);

struct ReserveArgs {
  int B, n, page_size, max_prefix, max_pages, num_pages, capacity;
  int32_t* page_table;
  const int32_t* seq_lens;
  int32_t* free_pages;
  int32_t* free_count;
  const int32_t* returned;       // may be null (then num_returned is null too)
  const int32_t* num_returned;
  unsigned int* err;
};
// One CTA keeps a byte per sequence in shared memory.
constexpr int kReserveMaxBatch = 65536;
bool reserve_batch_ok(int B);
cudaError_t launch_reserve(const ReserveArgs& a, cudaStream_t s);

// Projections on either side of the step attention (tcgen05 GEMM, weights
// [N][K] bf16 as the A operand, token rows [T][K] bf16 as B).  mode 0: y
// [T][N] bf16.  mode 1: the query/key/value projection of the R rows of each
// sequence (T = B R, N = (Hq + 2 Hkv) 128), rotary embedding of queries and
// keys at their zone positions, outputs q / k_blk / v_blk.
struct LinearArgs {
  int T, K, N, mode;
  const void* x;
  const void* w;
  void* y;
  void* q;
  void* k_blk;
  void* v_blk;
  const int32_t* seq_lens;
  int Hq, Hkv, R, k, max_prefix;
  double log2_base;
  unsigned int* err;
  void* ws;          // plan.ws_bytes of device scratch (split partials), 256-byte aligned
};
struct LinearPlan {
  bool ok;
  int nt, nsub, tiles, stages, ksplit;
  uint32_t stage_bytes;
  size_t smem;
  size_t ws_bytes;   // split-K partials and status words (0 with one split)
};
// Tile plan of one projection: ok is false for shapes the kernel does not
// take (K not a multiple of 64, N not a multiple of 128).  The split count
// depends on the current device's cluster occupancy (queried once).
LinearPlan plan_linear(int T, int K, int N);
cudaError_t launch_linear(const LinearArgs& a, cudaStream_t s);

}  // namespace tidar
