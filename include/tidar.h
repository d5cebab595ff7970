/*
 * tidar.h -- C ABI of libtidar.so, the GPU hot path of one TiDAR decode step.
 *
 * The method ("TiDAR: Think in Diffusion, Talk in Autoregression", arXiv
 * 2511.08923) is described on these pages, cited below by tag:
 *   [MS]   "TiDAR: Think in Diffusion, Talk in Autoregression" (mauroscia.it)
 *   [NDfr] "TiDAR : l'hybride de NVIDIA qui rédige par diffusion et parle de
 *          manière autorégressive" (nodesdaily.com, French)
 *   [FG]   "論文の概要: TiDAR: Think in Diffusion, Talk in Autoregression"
 *          (fugumt.com; the paper's abstract)
 *   [EN]   "TiDAR：Nvidia 的擴散＋自回歸混合架構——把閒置的 GPU 算力換成推論加速"
 *          (engineer-news.pages.dev)
 *
 * One step = tidar_step_attn (one attention pass over three zones, plus the
 * speculative write of the draft rows' K/V), then tidar_verify (left-to-right
 * acceptance and selection of the matching pre-drafted block), then
 * tidar_commit (keep the accepted drafts' cache rows, evict the rest).
 * Around it, for a loop of steps that never returns to the host:
 * tidar_reserve (the next step's draft pages from a device stack of free
 * pages, fed with the pages the commit released) and tidar_verify_blockq
 * (rejection verification whose draft distributions are read from the
 * previous step's mask-block logits through its selected block).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated otherwise, on the device
 *     that is current when the call is made.  The caller owns every buffer
 *     (cache, tables, inputs, outputs, workspace); the library allocates no
 *     device memory.  Its device state is a per-device error word (see
 *     tidar_get_device_status) and the fixed scratch of tidar_verify_noalloc;
 *     on the host it caches per-device kernel attributes and cluster
 *     occupancy, looked up on the first call made with each device current.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and returns after the launches are queued.  Kernels are
 *     launched as programmatic dependents of the preceding kernel on the
 *     stream: they may start early but wait for it to complete before they
 *     touch global memory, so stream order is kept.
 *   - Argument errors the host can see are returned before anything is
 *     launched.  Errors that depend on device-resident values (page ids, prefix
 *     lengths, accept counts) set bits in the device error word; the affected
 *     work is skipped (outputs of that row/sequence are unspecified but
 *     finite) and tidar_get_device_status reports them.  Nothing traps.
 *   - Floating-point tensors are fp32 (TIDAR_F32) or bf16 (TIDAR_BF16),
 *     row-major, contiguous, 16-byte aligned.
 *
 * Shapes (B batch, Hq query heads, Hkv KV heads, G = Hq/Hkv, D head_dim,
 * k draft length in 0..16, n = max(k,1), R = k + k*k rows per sequence, R = 1
 * when k = 0):
 *   query rows of a sequence, in order: the k carried-over drafts d_1..d_k
 *   (row r-1 for d_r), then mask block j = 1..k, slot s = 1..k at row
 *   k + (j-1)k + (s-1).  The step keys/values use the same row indices.
 */
#ifndef TIDAR_H
#define TIDAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tidar_stream_t; /* identical to cudaStream_t */

typedef enum {
  TIDAR_OK = 0,
  TIDAR_ERR_INVALID_ARG = 1, /* a host-checkable argument is wrong; nothing launched */
  TIDAR_ERR_UNSUPPORTED = 2, /* valid but not implemented (dtype/head_dim/page size/path) */
  TIDAR_ERR_CUDA = 3,        /* a CUDA runtime call failed (message via tidar_last_cuda_error) */
  TIDAR_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (device error word) */
  TIDAR_ERR_DEVICE = 5       /* a device-side check failed (device error word) */
} tidar_status;

typedef enum { TIDAR_F32 = 0, TIDAR_BF16 = 1 } tidar_dtype;
typedef enum { TIDAR_GREEDY = 0, TIDAR_REJECTION = 1 } tidar_accept_mode;

/* Kernel family for the step attention.  AUTO picks, for bf16, head_dim 128,
 * page 64: the warp-MMA decode kernel (DEC) when the query block packs into at
 * most 16 rows per KV head (R * G <= 16, e.g. plain decode k = 0), else the
 * tcgen05/TMEM tensor-core kernel with one 128-row query tile per CTA (TC05);
 * the CUDA-core kernel (SIMT) otherwise.  PAIR is the tensor-core kernel with
 * two query tiles per CTA sharing each staged K/V block (same inputs as
 * TC05).  Asking for DEC with R * G > 16 returns TIDAR_ERR_UNSUPPORTED. */
typedef enum {
  TIDAR_PATH_AUTO = 0,
  TIDAR_PATH_SIMT = 1,
  TIDAR_PATH_TC05 = 2,
  TIDAR_PATH_DEC = 3,
  TIDAR_PATH_PAIR = 4
} tidar_attn_path;

/* Bits of the device error word. */
#define TIDAR_DEVERR_BAD_PAGE 0x1u      /* a needed page-table entry is -1 or >= num_pages */
#define TIDAR_DEVERR_BAD_LEN 0x2u       /* seq_lens[b] < 0 or > max_prefix_len */
#define TIDAR_DEVERR_BAD_COUNT 0x4u     /* accept_count[b] outside 0..n (commit); draft_block[b] outside 1..k (tidar_verify_blockq) */
#define TIDAR_DEVERR_TIMEOUT 0x8u       /* a bounded mbarrier wait ran out */
#define TIDAR_DEVERR_LAYOUT 0x10u       /* a kernel's shared-memory layout check failed (no work done) */
#define TIDAR_DEVERR_POOL 0x20u         /* tidar_reserve: too few free pages, or no room for the returned ids */

typedef struct {
  int32_t batch;          /* B >= 0 (0: every call is a no-op) */
  int32_t num_q_heads;    /* Hq */
  int32_t num_kv_heads;   /* Hkv, divides Hq; query head h reads KV head h / (Hq/Hkv) */
  int32_t head_dim;       /* D: 64 or 128 */
  int32_t k;              /* draft length, 0..16 */
  int32_t page_size;      /* rows per cache page: 16, 32, 64 or 128 (tensor-core path: 64) */
  int32_t max_prefix_len; /* upper bound on every seq_lens[b]; sizes the KV split */
  tidar_dtype dtype;      /* of q, k_blk, v_blk, out and the cache */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim) */
  tidar_attn_path path;   /* TIDAR_PATH_AUTO unless a test pins a kernel family */
} tidar_step_desc;

typedef struct {
  void* k_pages;             /* [num_pages][Hkv][page_size][D], dtype */
  void* v_pages;             /* same layout */
  int32_t* page_table;       /* [batch][max_pages_per_seq]: page id of rows
                                [i*page_size, (i+1)*page_size) of sequence b, -1 = none */
  int32_t* seq_lens;         /* [batch]: P_b, the committed (settled) prefix length */
  int32_t num_pages;
  int32_t max_pages_per_seq; /* >= ceil((max_prefix_len + n) / page_size) */
} tidar_kv_cache;

/* ---------------------------------------------------------------------------
 * Step attention.  [MS] §2 "Single Forward Pass & Structured Attention Mask"
 * (three zones: causal prefix, verified drafts, bidirectional pre-drafts);
 * [NDfr] paragraphs on the three zones, on betting on every outcome (one mask
 * block per possible accept count) and on the masking puzzle (drafts strictly
 * causal, each block fully visible inside and seeing the whole settled past;
 * the mask depends only on zone-relative positions, so it slides forward).
 *
 * For sequence b, query head h (KV head g = h / G) and row rho:
 *   out[b][rho][h] = sum over visible keys x of softmax_x(<q, K_x> * scale) V_x
 * where the visible keys are the prefix rows 0..P_b-1 of the paged cache and
 * the step keys chosen by the mask:
 *   draft row r (rho = r-1):          D_1..D_r
 *   slot (j, s) of mask block j:      D_1..D_j and M_{j,1..k} (its whole block)
 *   k = 0 (one row):                  D_1 (itself)
 * lse_out (optional) receives the natural-log normaliser log(sum exp(score)).
 *
 * The same call writes the step rows' K/V of the drafts (rows 0..n-1 of k_blk,
 * v_blk) into cache rows P_b .. P_b+n-1 (the pages must already be reserved in
 * page_table); tidar_commit later keeps the accepted ones.  The attention
 * itself reads only cache rows < P_b.
 *
 *   q        [B][R][Hq][D]     k_blk, v_blk [B][R][Hkv][D]     (dtype)
 *   out      [B][R][Hq][D]     (dtype)     lse_out [B][R][Hq] fp32 or NULL
 *   workspace: device scratch of at least tidar_step_attn_workspace_bytes(desc)
 *     bytes, 256-byte aligned (may be NULL when that size is 0: one split, or
 *     splits merged inside the kernel); it holds split partials for the
 *     second launch.  Contents on entry are ignored.  Calls that share a
 *     workspace must be stream-ordered.
 * Device errors: BAD_PAGE (prefix or draft page unmapped), BAD_LEN; the TC05
 * and DEC kernels also TIMEOUT (a bounded wait on a copy or on a cluster
 * peer ran out) and LAYOUT.  Splits of a long prefix merge inside the
 * attention kernel (the splits of a query tile form a thread-block cluster and
 * read each other's rows over distributed shared memory) when such clusters
 * can be scheduled, else through workspace partials in a second launch.  That second launch also writes the
 * draft rows; without it the tensor-core and decode kernels write them (SIMT
 * always takes the second launch).
 * ------------------------------------------------------------------------- */
size_t tidar_step_attn_workspace_bytes(const tidar_step_desc* desc);
tidar_status tidar_step_attn(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                             const void* q, const void* k_blk, const void* v_blk, void* out,
                             float* lse_out, void* workspace, size_t workspace_bytes,
                             tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Context parallelism: one long sequence whose prefix pages are spread over
 * several GPUs (no counterpart on the pages, which speak of one standalone
 * model on one device; the split follows from softmax attention over a union
 * of disjoint key sets being the log-sum-exp merge of the attention over each
 * set).  Each GPU runs tidar_step_attn_part on its slice -- a tidar_kv_cache
 * holding its share of the prefix rows, seq_lens = the slice's length -- and
 * the GPUs exchange (out, lse) and merge them with tidar_merge_attn.  Exactly
 * one slice, the one holding the sequence's tail pages, takes the step keys
 * and appends the draft rows.
 *
 * tidar_step_attn_part: tidar_step_attn with
 *   flags & TIDAR_PART_STEP_KEYS: also attend the step keys (the zone mask);
 *                                 else every row sees only the slice's prefix;
 *   flags & TIDAR_PART_APPEND:    write the draft rows' K/V at the slice's
 *                                 rows P_b .. P_b+n-1 (its pages reserved);
 *   lse_out is required.  A row with no key in the call (an empty slice
 *   without step keys) gets out = 0 and lse = -inf.
 *   tidar_step_attn is flags = TIDAR_PART_STEP_KEYS | TIDAR_PART_APPEND.
 * tidar_merge_attn: out[i] = sum_r w_r part_o[r][i] / sum_r w_r with
 *   w_r = exp(part_lse[r][i] - max_r part_lse[r][i]); lse_out[i] = max +
 *   log(sum w) (fp32; may be NULL).  part_o [nparts][rows][head_dim] and out
 *   [rows][head_dim] of `dtype`; part_lse [nparts][rows] fp32.  A part with
 *   lse -inf gets no weight.  nparts <= 64, head_dim 64 or 128.
 * ------------------------------------------------------------------------- */
#define TIDAR_PART_STEP_KEYS 0x1
#define TIDAR_PART_APPEND 0x2
tidar_status tidar_step_attn_part(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                                  const void* q, const void* k_blk, const void* v_blk,
                                  int32_t flags, void* out, float* lse_out, void* workspace,
                                  size_t workspace_bytes, tidar_stream_t stream);
tidar_status tidar_merge_attn(int32_t nparts, int64_t rows, int32_t head_dim, tidar_dtype dtype,
                              const void* part_o, const float* part_lse, void* out,
                              float* lse_out, tidar_stream_t stream);

/* The launch plan the library would use: kernel family (1 SIMT, 2 TC05,
 * 3 DEC, 4 PAIR), number of KV splits, and how the splits merge (0: one
 * split; 1: in the attention kernel, its splits forming a thread-block
 * cluster; 2: a second launch).  Any pointer may be NULL.  Host only; with a
 * GPU present the first call per device queries its cluster occupancy. */
tidar_status tidar_step_attn_plan(const tidar_step_desc* desc, int32_t* path, int32_t* splits,
                                  int32_t* merge);

/* ---------------------------------------------------------------------------
 * Verification, acceptance and selection.  [NDfr] paragraph on betting on
 * every outcome (strict left-to-right scoring of the carried drafts; a guess
 * block is waiting for whichever outcome verification confirms); [MS] §1
 * (a good draft is accepted, a bad one corrected); [EN] section "TiDAR 在做什麼"
 * and [NDfr] last paragraph (output identical to AR sampling).  The rejection
 * rule is the speculative-sampling rule of the work [MS] lists as TiDAR's
 * lineage (Leviathan et al., Chen et al.).
 *
 * With n = max(k,1) and row i of `logits` the AR distribution p_i of the token
 * after d_1..d_i:
 *   j = 1; for i = 1..n-1, accept d_{i+1} iff
 *     greedy:    d_{i+1} == argmax logits_i (lowest index on ties)
 *     rejection: u[i-1] * q_i(d_{i+1}) < p_i(d_{i+1})       (fp64)
 *   and stop at the first rejection; j = 1 + accepted count.
 *   t* at row j: greedy argmax; rejection: inverse CDF (smallest t with
 *   u[n-1]*sum(w) < sum_{x<=t} w) of w = max(0, p_j - q_j) after a rejection
 *   (w = p_j if that is all zero) or w = p_j when every draft was accepted.
 *   accept_count[b] = j; out_tokens[b] = d_2..d_j, t*, then -1 up to n;
 *   selected_block[b] = j (0 when k = 0); next_drafts[b] = t*, g_{j,2..k}.
 * Probabilities in the rejection test and the inverse CDF are computed in
 * fp64 (softmax with the row maximum subtracted).  Logits must be finite.
 *
 *   logits        [B][n][V] dtype         drafts [B][k] int32 (NULL if k == 0)
 *   draft_logits  [B][k-1][V] dtype, rejection only (q_i is row i-1)
 *   uniforms      [B][n] fp32 in [0,1), rejection only
 *   block_guesses [B][k][k] int32 slot guesses of each mask block, or NULL
 *   accept_count  [B] int32      out_tokens [B][n] int32
 *   next_drafts   [B][k] int32 or NULL      selected_block [B] int32 or NULL
 *   workspace: at least tidar_verify_workspace_bytes(...) bytes, 256-aligned
 *     (per-chunk statistics of the logits rows).
 * A draft token outside [0, V) is never accepted.  TIDAR_ERR_UNSUPPORTED when
 * the launch grid does not fit: greedy B*n > 65535, rejection B*(2n-1) > 65535.
 * ------------------------------------------------------------------------- */
size_t tidar_verify_workspace_bytes(int32_t batch, int32_t k, int32_t vocab,
                                    tidar_accept_mode mode);
tidar_status tidar_verify(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                          tidar_accept_mode mode, const void* logits, const int32_t* drafts,
                          const void* draft_logits, const float* uniforms,
                          const int32_t* block_guesses, int32_t* accept_count,
                          int32_t* out_tokens, int32_t* next_drafts, int32_t* selected_block,
                          void* workspace, size_t workspace_bytes, tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Rejection verification whose draft distributions are read in place from the
 * previous step's mask-block logits.  [NDfr] paragraph on betting on every
 * outcome (one guess block per possible accept count, waiting for the
 * verification that confirms it); [MS] §2 (the pre-drafts come from the
 * diffusion predictions of the mask slots).  The block j selected last step
 * supplied this step's drafts [t*, g_{j,2}, .., g_{j,k}], so draft d_{i+1}
 * (i >= 1) was drawn from slot i+1 of block j: q_i is row
 * (b, j-1, i) of prev_block_logits.  Nothing is gathered or copied; j comes
 * from draft_block on the device (last step's selected_block), so a loop of
 * steps needs no host round-trip.
 *
 *   prev_block_logits [B][k][k][V] dtype (block j-1, slot s-1), 16-byte aligned
 *   draft_block       [B] int32, 1..k (a value outside: block 1 is read and
 *                     TIDAR_DEVERR_BAD_COUNT is set)
 * Both may be NULL when k <= 1.  Every other argument, the workspace
 * (tidar_verify_workspace_bytes(..., TIDAR_REJECTION)) and the results are
 * those of tidar_verify in TIDAR_REJECTION mode with draft_logits row i-1 =
 * that block row.
 * ------------------------------------------------------------------------- */
tidar_status tidar_verify_blockq(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                 const void* logits, const int32_t* drafts,
                                 const void* prev_block_logits, const int32_t* draft_block,
                                 const float* uniforms, const int32_t* block_guesses,
                                 int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                                 int32_t* selected_block, void* workspace, size_t workspace_bytes,
                                 tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Verification without a caller workspace (no counterpart in the paper; a
 * convenience of this library).
 *
 * Same arguments, results and device-side behaviour as tidar_verify, minus
 * the workspace.  It is for callers that cannot allocate device memory at the
 * point where they verify: a decode loop being captured into a CUDA graph, or
 * a host runtime that only passes in tensors it already owns.  The scratch is
 * a fixed array inside the library of TIDAR_VERIFY_NOALLOC_MAX_SCRATCH_BYTES
 * (4 MiB) on every GPU that loads the library, held until the process exits.
 * The call allocates nothing.
 *   - Returns TIDAR_ERR_UNSUPPORTED, before any launch, when the call needs
 *     more scratch than that (tidar_verify_workspace_bytes(...) > the maximum).
 *   - The first call made with a given device current looks the array's
 *     address up (cudaGetSymbolAddress); make that first call before any
 *     stream capture.
 *   - All calls share the array and it keeps the previous call's contents
 *     (verification reads nothing it did not write).  Calls that can overlap
 *     on the GPU -- different streams with no ordering between them -- race
 *     on it; order them on one stream.
 * ------------------------------------------------------------------------- */
#define TIDAR_VERIFY_NOALLOC_MAX_SCRATCH_BYTES ((size_t)4 << 20)
tidar_status tidar_verify_noalloc(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                  tidar_accept_mode mode, const void* logits,
                                  const int32_t* drafts, const void* draft_logits,
                                  const float* uniforms, const int32_t* block_guesses,
                                  int32_t* accept_count, int32_t* out_tokens,
                                  int32_t* next_drafts, int32_t* selected_block,
                                  tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Sampling controls: verification and the next drafts under a temperature and
 * a nucleus (top-p) truncation.  The pages fix neither; they speak of sampling
 * from the AR distribution ([EN] section "TiDAR 在做什麼") and of drafting from
 * the mask blocks' predictions ([MS] §2; [NDfr] paragraph on betting on every
 * outcome).  The speculative-sampling rule is exact for any pair (p, q), so the
 * same transform is applied to the AR rows and to the draft rows:
 *   temperature T > 0:  p(x) proportional to exp(l(x) / T);
 *   top_p in (0, 1]:    order the tokens larger logit first, lower index first
 *                       on equal logits; keep token x iff the probability of
 *                       the tokens before it is below top_p (the shortest run
 *                       reaching top_p); renormalise the kept tokens.
 *                       top_p >= 1 keeps every token.
 * Probabilities, the cut and the sums are fp64 (the cut is exact up to
 * summation order: a cut within ~1e-15 of top_p may fall either way).
 * ------------------------------------------------------------------------- */
typedef struct {
  float temperature; /* > 0 */
  float top_p;       /* > 0; >= 1 disables the truncation */
} tidar_sampling;

/* tidar_verify / tidar_verify_blockq with the transform.
 *   Greedy mode ignores the transform (the most likely token is always kept
 *   and T keeps the order) and runs tidar_verify's greedy kernel; draft rows
 *   and uniforms are not read.
 *   Rejection mode: draft_logits [B][k-1][V] (q_i in row i-1), or -- when
 *   prev_block_logits is non-NULL -- q_i read in place from the previous
 *   step's mask blocks as tidar_verify_blockq does (draft_logits then unused).
 *   workspace: at least tidar_verify_sampled_workspace_bytes(batch, k, vocab,
 *   mode) bytes, 256-byte aligned.  Everything else as tidar_verify.
 * TIDAR_ERR_INVALID_ARG for a NULL `sampling`, T <= 0 or top_p <= 0 (or NaN).
 */
size_t tidar_verify_sampled_workspace_bytes(int32_t batch, int32_t k, int32_t vocab,
                                            tidar_accept_mode mode);
tidar_status tidar_verify_sampled(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                  tidar_accept_mode mode, const tidar_sampling* sampling,
                                  const void* logits, const int32_t* drafts,
                                  const void* draft_logits, const void* prev_block_logits,
                                  const int32_t* draft_block, const float* uniforms,
                                  const int32_t* block_guesses, int32_t* accept_count,
                                  int32_t* out_tokens, int32_t* next_drafts,
                                  int32_t* selected_block, void* workspace,
                                  size_t workspace_bytes, tidar_stream_t stream);

/* The next step's drafts from the selected mask block, on the device.  With
 * j = selected_block[b] (a value outside 1..k reads block 1 and sets
 * TIDAR_DEVERR_BAD_COUNT), slot s = 2..k of block j -- row
 * block_logits[b][j-1][s-1] -- gives next_drafts[b][s-1]:
 *   TIDAR_GREEDY:    its argmax (lowest index on ties);
 *   TIDAR_REJECTION: a draw from its transformed distribution, the smallest t
 *                    with uniforms[b][s-1] * sum(q) < sum_{x<=t} q(x) (index
 *                    order), so that next step's tidar_verify_sampled /
 *                    tidar_verify_blockq, reading q from the same rows, sees
 *                    drafts drawn from q.
 * next_drafts[b][0] (t*, written by verification) is not touched.  k < 2: no
 * work.  block_logits [B][k][k][V] dtype, 16-byte aligned; uniforms [B][k]
 * fp32 in [0,1) (TIDAR_REJECTION only; entry 0 unused).  No workspace.
 */
tidar_status tidar_sample_drafts(int32_t batch, int32_t k, int32_t vocab, tidar_dtype dtype,
                                 tidar_accept_mode mode, const tidar_sampling* sampling,
                                 const void* block_logits, const int32_t* selected_block,
                                 const float* uniforms, int32_t* next_drafts,
                                 tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * KV commit / evict, in place.  [NDfr] paragraph on the three zones (the
 * settled cache is reused, rejected entries are evicted); [MS] "KV Cache" and
 * [FG] abstract (exact KV cache).  Accepted drafts are a prefix of the draft
 * zone ([NDfr]: the futures run from only the first kept to all kept), so no row
 * moves.  For each b with c = accept_count[b] in 0..n and P = seq_lens[b]:
 *   cache rows P+c .. P+n-1 (every KV head, K and V) are zeroed;
 *   seq_lens[b] = P + c;
 *   page_table[b][i] for i in [ceil((P+c)/ps), ceil((P+n)/ps)) -- pages that
 *   held only rejected draft rows -- are set to -1 and their ids returned.
 *   released_pages: [B * (ceil(n/ps) + 1)] int32, the released ids in
 *     (b, i) order, then -1; num_released: [1] int32.
 * tidar_verify produces c in 1..n; c = 0 (evict every draft row) is allowed.
 * Device errors: BAD_COUNT (c out of range) or BAD_PAGE (a draft row without
 * a valid page): that sequence is left untouched.  TIDAR_ERR_UNSUPPORTED when
 * the per-sequence bookkeeping of the one launch (a single thread-block
 * cluster) exceeds its shared memory: B * (4 + min(n, ceil(n/ps) + 1)) * 4
 * bytes > 8 * 200 KiB (B > 68266 at page 64).
 * ------------------------------------------------------------------------- */
tidar_status tidar_commit(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                          const int32_t* accept_count, int32_t* released_pages,
                          int32_t* num_released, tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * tidar_verify followed by tidar_commit on the accept counts it produces, as
 * one call: the verification after a step's forward pass and the eviction it
 * implies ([NDfr] paragraphs on betting on every outcome and on the three
 * zones).  Arguments as the two calls (batch and k from desc; dtype is the
 * logits' type), accept_count both the verification's output and the
 * commit's input; workspace as tidar_verify's
 * (tidar_verify_workspace_bytes(batch, k, vocab, mode)).  Every host check of
 * both runs before anything is queued.  Greedy mode computes the acceptance
 * inside the commit's launch (two launches: the chunk statistics, then
 * acceptance + commit); rejection mode queues tidar_verify's launches and
 * then the commit's.  Results and device errors are those of the two calls.
 * ------------------------------------------------------------------------- */
tidar_status tidar_verify_commit(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                                 int32_t vocab, tidar_dtype dtype, tidar_accept_mode mode,
                                 const void* logits, const int32_t* drafts,
                                 const void* draft_logits, const float* uniforms,
                                 const int32_t* block_guesses, int32_t* accept_count,
                                 int32_t* out_tokens, int32_t* next_drafts,
                                 int32_t* selected_block, int32_t* released_pages,
                                 int32_t* num_released, void* workspace, size_t workspace_bytes,
                                 tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Page reservation for the next step's draft rows, from a device stack of
 * free pages (the step the commit's release implies; the pages do not
 * describe a page pool).  [NDfr] paragraph on the three zones: the candidates
 * carried from the previous step follow the settled tokens, the settled cache
 * is reused and rejected entries are evicted.  With the ids that tidar_commit
 * released passed back in, reserve -> tidar_step_attn -> tidar_verify ->
 * tidar_commit repeats on the device with no host round-trip, so many steps
 * can be one CUDA graph.
 *
 * The pool is a stack: free_pages[0 .. *free_count) are free page ids, the
 * last one on top.  In one launch:
 *   1. the returned ids (*num_returned of them) are pushed in order on top;
 *      if *num_returned < 0 or they do not fit in `capacity` (or *free_count
 *      is outside 0..capacity), NOTHING changes and TIDAR_DEVERR_POOL is set;
 *   2. for each b, with P = seq_lens[b] and n = max(k,1), the draft rows
 *      P .. P+n-1 lie on page-table entries floor(P/ps) .. ceil((P+n)/ps)-1.
 *      An entry below ceil(P/ps) also holds prefix rows and must be a valid
 *      page; an entry at or above it is kept if valid and needs a page if -1.
 *      P < 0 or P > max_prefix_len sets BAD_LEN, any other entry BAD_PAGE; that
 *      sequence is skipped;
 *   3. if the stack holds fewer ids than the entries that need one, no entry
 *      changes, TIDAR_DEVERR_POOL is set and *free_count is the count after the
 *      push;
 *   4. otherwise the needing entries, in (b, i) order, pop the stack: the t-th
 *      takes free_pages[count-1-t]; *free_count drops by their number.
 *      Entries at or above the new count keep the ids they held.
 * Popped ids are not range-checked here (tidar_step_attn reports BAD_PAGE).
 * With page_size >= 16 and k <= 16 a sequence needs at most one page a step.
 *
 *   pool->free_pages [capacity] int32, pool->free_count [1] int32 (device)
 *   returned_pages [*num_returned] int32 and num_returned [1] int32 (device),
 *     e.g. tidar_commit's released_pages / num_released; both NULL to push
 *     nothing, else both non-NULL (TIDAR_ERR_INVALID_ARG).
 * Only page_table (and the pool) are written; dtype, head counts, head_dim and
 * path of `desc` are not used beyond validation.  TIDAR_ERR_UNSUPPORTED when
 * batch > 65536 (one CTA with a byte of shared memory per sequence).
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t* free_pages; /* [capacity] page ids; [0, *free_count) are free */
  int32_t* free_count; /* [1] */
  int32_t capacity;    /* >= 0 */
} tidar_page_pool;

tidar_status tidar_reserve(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                           const tidar_page_pool* pool, const int32_t* returned_pages,
                           const int32_t* num_returned, tidar_stream_t stream);

/* ---------------------------------------------------------------------------
 * Layer-level step: the projections on either side of the step attention.
 * [MS] §2 (one forward pass of the model over the three zones); [EN] section
 * "為什麼 GPU 在 AR 推論時是閒置的" (each AR decode step reloads every weight,
 * so a memory-bound step leaves the compute units idle); [NDfr] paragraph on
 * the masking puzzle (the extra blocks cost a small constant factor on that
 * idle capacity) and [FG] abstract ("free token slots").  Weights are bf16
 * rows of their output features (a linear layer y = x w^T); the library
 * computes in fp32 and stores bf16.  The weights here are the caller's
 * (random ones in this repository's tests and benchmark).
 *
 * tidar_linear: y [rows][out_features] = x [rows][in_features] . w^T with
 *   w [out_features][in_features].  dtype must be TIDAR_BF16, in_features a
 *   multiple of 64 and out_features a multiple of 128 (else
 *   TIDAR_ERR_UNSUPPORTED); x, w, y 16-byte aligned.  rows >= 0.
 *   workspace: device scratch of at least tidar_linear_workspace_bytes(rows,
 *   out_features, in_features) bytes, 256-byte aligned (NULL when that is 0):
 *   the fp32 partial sums of the reduction's splits.  Contents on entry are
 *   ignored; calls sharing a workspace must be stream-ordered.  The size
 *   depends on the current device (its cluster occupancy sets the number of
 *   splits): query it on the device that runs the call.
 *
 * tidar_qkv_rope: the query/key/value projection of the R step rows of each
 *   sequence and the rotary embedding at their zone positions.
 *   x      [B][R][d_model] bf16 hidden states of the step rows (row order as
 *          tidar_step_attn: drafts, then mask blocks)
 *   w_qkv  [(Hq + 2 Hkv) D][d_model] bf16: query features of head h at rows
 *          [h D, h D + D), then the Hkv key heads, then the Hkv value heads
 *   seq_lens [B] int32 (device): P_b, which places the rows:
 *          draft d_r at position P_b + r - 1, slot s of mask block j at
 *          P_b + j + s - 1 (where t* and the next drafts land once j drafts
 *          are accepted), the single row of k = 0 at P_b
 *   queries and keys are rotated pairwise (dims f and f + D/2) by the angle
 *   position * rope_base^(-2f/D) (formed in fp64); values are not rotated.
 *   q [B][R][Hq][D], k_blk / v_blk [B][R][Hkv][D]: tidar_step_attn's inputs.
 *   Needs dtype TIDAR_BF16, head_dim 128, d_model a multiple of 64
 *   (TIDAR_ERR_UNSUPPORTED otherwise), rope_base > 1.  Device error BAD_LEN
 *   (seq_lens[b] outside 0..max_prefix_len: position P_b = 0 is used).
 *   workspace as tidar_linear's, sized by tidar_qkv_rope_workspace_bytes.
 *
 * tidar_layer_step: tidar_qkv_rope, tidar_step_attn (which also appends the
 *   drafts' rotated K/V to the cache) and the output projection
 *   y [B][R][d_model] = attn_out . w_o^T with w_o [d_model][Hq D], as one
 *   call.  lse_out as tidar_step_attn's.  workspace: at least
 *   tidar_layer_step_workspace_bytes(desc, d_model) bytes, 256-byte aligned,
 *   holding q, k_blk, v_blk, the attention output, the projections' and the
 *   attention's own workspaces.  d_model must also be a multiple of 128.
 * Device errors: those of the calls it makes; TIMEOUT if a bounded wait in a
 * projection ran out.
 * ------------------------------------------------------------------------- */
size_t tidar_linear_workspace_bytes(int32_t rows, int32_t out_features, int32_t in_features);
tidar_status tidar_linear(int32_t rows, int32_t out_features, int32_t in_features,
                          tidar_dtype dtype, const void* x, const void* w, void* y,
                          void* workspace, size_t workspace_bytes, tidar_stream_t stream);
size_t tidar_qkv_rope_workspace_bytes(const tidar_step_desc* desc, int32_t d_model);
tidar_status tidar_qkv_rope(const tidar_step_desc* desc, int32_t d_model, const void* x,
                            const void* w_qkv, const int32_t* seq_lens, float rope_base,
                            void* q, void* k_blk, void* v_blk, void* workspace,
                            size_t workspace_bytes, tidar_stream_t stream);
size_t tidar_layer_step_workspace_bytes(const tidar_step_desc* desc, int32_t d_model);
tidar_status tidar_layer_step(const tidar_step_desc* desc, const tidar_kv_cache* cache,
                              int32_t d_model, const void* x, const void* w_qkv,
                              const void* w_o, float rope_base, void* y, float* lse_out,
                              void* workspace, size_t workspace_bytes, tidar_stream_t stream);

/* Synchronises `stream`, reads and clears this device's error word.  Returns
 * TIDAR_ERR_TIMEOUT if the timeout bit was set, TIDAR_ERR_DEVICE for any other
 * bit, TIDAR_ERR_CUDA if the synchronisation failed, else TIDAR_OK.  bits_out
 * (host pointer, may be NULL) receives the raw bits. */
tidar_status tidar_get_device_status(tidar_stream_t stream, uint32_t* bits_out);

const char* tidar_status_string(tidar_status status);
/* Text of the last CUDA error seen by this thread's calls (host string). */
const char* tidar_last_cuda_error(void);

/* ---------------------------------------------------------------------------
 * Test hooks (no counterpart in the paper).  Process-wide host flags, read
 * when a call is launched; all off by default.
 *   TIDAR_DEBUG_STARVE_ATTENTION_LOADS: tensor-core step attentions issue no
 *     K/V copies, so their bounded mbarrier waits run out (after about 1 s):
 *     the CTAs record TIDAR_DEVERR_TIMEOUT, release TMEM and exit, the
 *     outputs are unspecified, tidar_get_device_status returns
 *     TIDAR_ERR_TIMEOUT and the CUDA context stays usable (failure injection).
 *   TIDAR_DEBUG_FORCE_SPLIT_PARTIALS: the TC05, PAIR and DEC paths merge key
 *     splits in a second launch even where they would merge them in the
 *     attention kernel (so tests reach both merges).  May change the split
 *     count, and with it the size tidar_step_attn_workspace_bytes reports.
 * Returns TIDAR_ERR_INVALID_ARG for an unknown knob.
 * ------------------------------------------------------------------------- */
typedef enum {
  TIDAR_DEBUG_STARVE_ATTENTION_LOADS = 1,
  TIDAR_DEBUG_FORCE_SPLIT_PARTIALS = 2
} tidar_debug_knob;
tidar_status tidar_debug_set(tidar_debug_knob knob, int32_t value);

#ifdef __cplusplus
}
#endif
#endif /* TIDAR_H */
