/*
 * tidar_oracle.c -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, CPU restatement of one TiDAR decode step, written from the
 * description of the method on these web pages (cited below by tag):
 *
 *   [EN]   "TiDAR：Nvidia 的擴散＋自回歸混合架構——把閒置的 GPU 算力換成推論加速"
 *          (engineer-news.pages.dev)
 *   [MS]   "TiDAR: Think in Diffusion, Talk in Autoregression" (mauroscia.it)
 *   [NDfr] "TiDAR : l'hybride de NVIDIA qui rédige par diffusion et parle de
 *          manière autorégressive" (nodesdaily.com, French)
 *   [FG]   "論文の概要: TiDAR: Think in Diffusion, Talk in Autoregression"
 *          (fugumt.com, arXiv 2511.08923 abstract)
 *
 * Only tests/, the smoke check and the CPU-baseline leg of the benchmark may
 * load this code.  It shares no source with the CUDA library and never links it.
 *
 * Arithmetic: inputs are fp32 or bf16 (bf16 is widened exactly to fp64); every
 * sum, exponential and division is in fp64.  Loops are unfused and unsplit:
 * scores for all visible keys, then the maximum, then the normaliser, then the
 * weighted sum of values, in key order.
 *
 * Notation (the pages give none in symbols; this is the plainest reading):
 *   B batch, Hq query heads, Hkv KV heads, G = Hq/Hkv, D head_dim, P_b the
 *   settled prefix length of sequence b, k the draft length, n = max(k,1),
 *   R = k + k*k query rows per sequence (R = 1 when k = 0).
 *   Rows of a step: draft rows r = 1..k (row index r-1), then mask block
 *   j = 1..k, slot s = 1..k (row index k + (j-1)k + (s-1)).
 *   Step keys use the same indices: D_1..D_k are step keys 0..k-1 and
 *   M_{j,s} is step key k + (j-1)k + (s-1).
 *
 * Parity pins: every function here is checked by tests/test_oracle_*.py against
 * closed forms, independent formulations (dense attention over explicitly
 * concatenated key sets, numpy/torch library routines), invariants and
 * chi-squared / exact-enumeration tests of the acceptance rule.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_PAGE 2
#define ORACLE_ERR_COUNT 3

/* bf16 -> fp64, exact: a bf16 value is the upper half of an fp32 value. */
static double widen_bf16(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Element idx of a buffer stored as fp32 (dtype 0) or bf16 (dtype 1). */
static double elem(const void* base, int64_t idx, int dtype) {
  if (dtype == 0) return (double)((const float*)base)[idx];
  return widen_bf16(((const uint16_t*)base)[idx]);
}

/*
 * Structured mask over the step keys ([MS] §2 "Single Forward Pass &
 * Structured Attention Mask": three zones, causal for the verified drafts,
 * bidirectional for the pre-drafts; [NDfr] paragraph on the masking puzzle:
 * settled tokens strictly causal, each guess block fully visible inside and
 * seeing the whole settled past; [NDfr] paragraph on betting on every outcome:
 * one guess block per future "first survives / two survive / all survive").
 *
 * Returns 1 if query row `row` may attend step key `key`.  The prefix keys are
 * visible to every row and are not decided here.  The predicate depends on
 * zone-relative indices only, never on P_b ([NDfr] masking paragraph: the same
 * mask slides forward as the text grows).
 */
int tidar_oracle_step_key_visible(int k, int row, int key) {
  if (k == 0) return key == 0;           /* plain AR decode: the newest token sees itself */
  if (row < k) return key <= row;         /* draft row r sees D_1..D_r (causal) */
  {
    int j = (row - k) / k + 1;            /* mask block j in 1..k */
    int first = k + (j - 1) * k;          /* its slots M_{j,1..k} */
    if (key < j) return 1;                /* D_1..D_j: the j drafts of this future */
    return key >= first && key < first + k; /* its own block, bidirectional */
  }
}

static int rows_per_seq(int k) { return k == 0 ? 1 : k + k * k; }

/* Address (in elements) of cache row `pos` of KV head g for sequence b, or -1
 * if the page table does not map it to a valid page. */
static int64_t cache_row(const int32_t* page_table, int max_pages, int num_pages,
                         int page_size, int Hkv, int D, int b, int g, int64_t pos) {
  int64_t pi = pos / page_size;
  int32_t page;
  if (pi >= max_pages) return -1;
  page = page_table[(int64_t)b * max_pages + pi];
  if (page < 0 || page >= num_pages) return -1;
  return (((int64_t)page * Hkv + g) * page_size + pos % page_size) * D;
}

/*
 * One output row of the step attention: softmax over every visible key of the
 * scaled dot products, applied to the values (the plain definition of
 * attention; the prefix zone comes from the KV cache, [MS] "KV Cache",
 * [NDfr] paragraph on the three zones).  Query head h reads KV head h / G.
 * Returns ORACLE_ERR_PAGE if a needed prefix page is unmapped.
 */
static int attend_one(int b, int rho, int h, int Hq, int Hkv, int D, int k, int page_size,
                      int dtype, double scale, const void* k_pages, const void* v_pages,
                      const int32_t* page_table, int max_pages, int num_pages, int P,
                      const void* q, const void* k_blk, const void* v_blk, int with_step_keys,
                      double* s /* scratch, P + R */, double* out, double* lse) {
  const int R = rows_per_seq(k);
  const int G = Hq / Hkv;
  const int g = h / G;
  const int64_t qoff = (((int64_t)b * R + rho) * Hq + h) * D;
  int nkeys = 0, i, d;
  double m = -INFINITY, z = 0.0;

  /* scores: prefix keys 0..P-1, then the visible step keys in index order */
  for (i = 0; i < P; ++i) {
    int64_t ko = cache_row(page_table, max_pages, num_pages, page_size, Hkv, D, b, g, i);
    double dot = 0.0;
    if (ko < 0) return ORACLE_ERR_PAGE;
    for (d = 0; d < D; ++d) dot += elem(q, qoff + d, dtype) * elem(k_pages, ko + d, dtype);
    s[nkeys++] = dot * scale;
  }
  for (i = 0; with_step_keys && i < R; ++i) {
    if (tidar_oracle_step_key_visible(k, rho, i)) {
      int64_t ko = (((int64_t)b * R + i) * Hkv + g) * D;
      double dot = 0.0;
      for (d = 0; d < D; ++d) dot += elem(q, qoff + d, dtype) * elem(k_blk, ko + d, dtype);
      s[nkeys++] = dot * scale;
    }
  }
  for (i = 0; i < nkeys; ++i) if (s[i] > m) m = s[i];
  for (i = 0; i < nkeys; ++i) { s[i] = exp(s[i] - m); z += s[i]; }

  for (d = 0; d < D; ++d) out[d] = 0.0;
  nkeys = 0;
  for (i = 0; i < P; ++i) {
    int64_t vo = cache_row(page_table, max_pages, num_pages, page_size, Hkv, D, b, g, i);
    double w = s[nkeys++] / z;
    for (d = 0; d < D; ++d) out[d] += w * elem(v_pages, vo + d, dtype);
  }
  for (i = 0; with_step_keys && i < R; ++i) {
    if (tidar_oracle_step_key_visible(k, rho, i)) {
      int64_t vo = (((int64_t)b * R + i) * Hkv + g) * D;
      double w = s[nkeys++] / z;
      for (d = 0; d < D; ++d) out[d] += w * elem(v_blk, vo + d, dtype);
    }
  }
  *lse = nkeys > 0 ? m + log(z) : -INFINITY;   /* no key: out = 0, lse = -inf */
  return ORACLE_OK;
}

/*
 * Step attention over the three zones.
 *   q      [B][R][Hq][D]      k_blk, v_blk [B][R][Hkv][D]  (dtype)
 *   k_pages, v_pages [num_pages][Hkv][page_size][D]; page_table [B][max_pages]
 *   seq_lens [B] (P_b).
 * If n_sel < 0 every (b, rho, h) is computed into out [B][R][Hq][D] and
 * lse [B][R][Hq]; otherwise only the n_sel triples sel[3i..3i+2] = (b, rho, h),
 * into out [n_sel][D], lse [n_sel].  lse is the natural log of the softmax
 * normaliser including the maximum.  scale <= 0 selects 1/sqrt(D).
 */
int tidar_oracle_step_attn_keys(int B, int Hq, int Hkv, int D, int k, int page_size, int dtype,
                                double scale, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, int max_pages, int num_pages,
                                const int32_t* seq_lens, const void* q, const void* k_blk,
                                const void* v_blk, int with_step_keys, int n_sel,
                                const int32_t* sel, double* out, double* lse, int num_threads);

int tidar_oracle_step_attn(int B, int Hq, int Hkv, int D, int k, int page_size, int dtype,
                           double scale, const void* k_pages, const void* v_pages,
                           const int32_t* page_table, int max_pages, int num_pages,
                           const int32_t* seq_lens, const void* q, const void* k_blk,
                           const void* v_blk, int n_sel, const int32_t* sel, double* out,
                           double* lse, int num_threads) {
  return tidar_oracle_step_attn_keys(B, Hq, Hkv, D, k, page_size, dtype, scale, k_pages, v_pages,
                                     page_table, max_pages, num_pages, seq_lens, q, k_blk, v_blk, 1,
                                     n_sel, sel, out, lse, num_threads);
}

/*
 * The same with the step keys optional: with_step_keys = 0 restricts every row
 * to the cache's prefix rows (attention over one slice of a longer sequence's
 * keys; a row with no key gets out = 0, lse = -inf).
 */
int tidar_oracle_step_attn_keys(int B, int Hq, int Hkv, int D, int k, int page_size, int dtype,
                                double scale, const void* k_pages, const void* v_pages,
                                const int32_t* page_table, int max_pages, int num_pages,
                                const int32_t* seq_lens, const void* q, const void* k_blk,
                                const void* v_blk, int with_step_keys, int n_sel,
                                const int32_t* sel, double* out, double* lse, int num_threads) {
  const int R = rows_per_seq(k);
  int64_t total, t;
  int Pmax = 0, b, status = ORACLE_OK;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || k < 0 || page_size <= 0)
    return ORACLE_ERR_ARG;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  for (b = 0; b < B; ++b) {
    if (seq_lens[b] < 0) return ORACLE_ERR_ARG;
    if (seq_lens[b] > Pmax) Pmax = seq_lens[b];
  }
  total = n_sel < 0 ? (int64_t)B * R * Hq : n_sel;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel
#endif
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)(Pmax + R + 1));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
    for (t = 0; t < total; ++t) {
      int bb, rho, h, st;
      if (n_sel < 0) {
        h = (int)(t % Hq);
        rho = (int)((t / Hq) % R);
        bb = (int)(t / ((int64_t)Hq * R));
      } else {
        bb = sel[3 * t]; rho = sel[3 * t + 1]; h = sel[3 * t + 2];
      }
      if (!s || bb < 0 || bb >= B || rho < 0 || rho >= R || h < 0 || h >= Hq) {
        st = ORACLE_ERR_ARG;
      } else {
        st = attend_one(bb, rho, h, Hq, Hkv, D, k, page_size, dtype, scale, k_pages, v_pages,
                        page_table, max_pages, num_pages, seq_lens[bb], q, k_blk, v_blk,
                        with_step_keys, s, out + t * D, lse + t);
      }
      if (st != ORACLE_OK) {
#ifdef _OPENMP
#pragma omp critical
#endif
        status = st;
      }
    }
    free(s);
  }
  return status;
}

/*
 * Attention over a union of disjoint key sets from the attention over each
 * set: softmax over the union is the mixture of the per-set softmaxes, each set
 * weighted by its normaliser exp(lse_r).  With M = max_r lse_r and
 * w_r = exp(lse_r - M) (0 when lse_r = -inf):
 *   out = sum_r w_r o_r / sum_r w_r,   lse = M + log(sum_r w_r).
 * parts_o [nparts][rows][D], parts_lse [nparts][rows] (fp64) -> out [rows][D],
 * lse [rows].  All parts -inf: out = 0, lse = -inf.
 */
int tidar_oracle_merge(int nparts, int64_t rows, int D, const double* parts_o, const double* parts_lse,
                       double* out, double* lse) {
  int64_t i;
  int r, d;
  if (nparts <= 0 || rows < 0 || D <= 0) return ORACLE_ERR_ARG;
  for (i = 0; i < rows; ++i) {
    double M = -INFINITY, z = 0.0;
    for (r = 0; r < nparts; ++r) if (parts_lse[(int64_t)r * rows + i] > M) M = parts_lse[(int64_t)r * rows + i];
    for (d = 0; d < D; ++d) out[i * D + d] = 0.0;
    if (M == -INFINITY) { lse[i] = -INFINITY; continue; }
    for (r = 0; r < nparts; ++r) {
      const double l = parts_lse[(int64_t)r * rows + i];
      const double w = l == -INFINITY ? 0.0 : exp(l - M);
      z += w;
      if (w != 0.0)
        for (d = 0; d < D; ++d) out[i * D + d] += w * parts_o[((int64_t)r * rows + i) * D + d];
    }
    for (d = 0; d < D; ++d) out[i * D + d] /= z;
    lse[i] = M + log(z);
  }
  return ORACLE_OK;
}

/*
 * Speculative write of the draft rows' K/V into the cache: the K/V of step rows
 * 0..n-1 (D_1..D_k; the single row when k = 0) go to cache positions
 * P_b .. P_b+n-1 of every KV head.  Byte copies (elem_bytes per element).
 * The carried-over drafts are the second zone of a step ([NDfr] paragraph on
 * the three zones); keeping their entries is what "reuse the settled cache"
 * means once they are accepted.
 */
int tidar_oracle_append(int B, int Hkv, int D, int k, int page_size, int elem_bytes,
                        void* k_pages, void* v_pages, const int32_t* page_table, int max_pages,
                        int num_pages, const int32_t* seq_lens, const void* k_blk,
                        const void* v_blk) {
  const int R = rows_per_seq(k);
  const int n = k > 0 ? k : 1;
  int b, r, g, status = ORACLE_OK;
  for (b = 0; b < B; ++b) {
    for (r = 0; r < n; ++r) {
      for (g = 0; g < Hkv; ++g) {
        int64_t dst = cache_row(page_table, max_pages, num_pages, page_size, Hkv, D, b, g,
                                (int64_t)seq_lens[b] + r);
        int64_t src = (((int64_t)b * R + r) * Hkv + g) * D;
        if (dst < 0) { status = ORACLE_ERR_PAGE; continue; }
        memcpy((char*)k_pages + dst * elem_bytes, (const char*)k_blk + src * elem_bytes,
               (size_t)D * elem_bytes);
        memcpy((char*)v_pages + dst * elem_bytes, (const char*)v_blk + src * elem_bytes,
               (size_t)D * elem_bytes);
      }
    }
  }
  return status;
}

/* softmax of one logit row in fp64: writes p[0..V-1] (may be NULL) and returns
 * nothing else.  Two passes: maximum, then normaliser. */
static void softmax_row(const void* base, int64_t off, int V, int dtype, double* p) {
  double m = -INFINITY, z = 0.0;
  int x;
  for (x = 0; x < V; ++x) { double v = elem(base, off + x, dtype); if (v > m) m = v; }
  for (x = 0; x < V; ++x) { p[x] = exp(elem(base, off + x, dtype) - m); z += p[x]; }
  for (x = 0; x < V; ++x) p[x] /= z;
}

/* argmax with the lowest index winning ties, on the exact stored values */
static int argmax_row(const void* base, int64_t off, int V, int dtype) {
  int x, best = 0;
  double bv = elem(base, off, dtype);
  for (x = 1; x < V; ++x) {
    double v = elem(base, off + x, dtype);
    if (v > bv) { bv = v; best = x; }
  }
  return best;
}

/*
 * Verification and acceptance ("Talk in Autoregression"): the drafts are
 * scored left to right under the strict AR distribution ([NDfr] paragraph on
 * betting on every outcome: strict left-to-right scoring; [MS] §1: a good
 * draft is accepted, a bad one corrected); the output must equal plain AR
 * sampling ([EN] section "TiDAR 在做什麼": mathematically equivalent to pure AR
 * sampling; [NDfr] last paragraph: accepted text is rescored under the strict
 * distribution).  The rejection rule is the speculative-sampling rule of the
 * lineage [MS] names (Leviathan et al., Chen et al.), which keeps the AR
 * distribution exact.
 *
 *   logits [B][n][V]: row i (1-based) is the AR distribution p_i of the token
 *     after d_1..d_i.  drafts [B][k]: d_1..d_k (d_1 is the token sampled at the
 *     end of the previous step and is always kept).
 *   draft_logits [B][k-1][V] (mode 1): row i-1 gives q_i, the distribution d_{i+1}
 *     was drafted from.   uniforms [B][n] in [0,1) (mode 1).
 *   block_guesses [B][k][k] or NULL: slot guesses of mask block j (row j-1).
 *
 * Algorithm (n = max(k,1)):
 *   j = 1; for i = 1..n-1: accept d_{i+1} iff
 *     greedy:    d_{i+1} == argmax l_i (lowest index on ties)
 *     rejection: u[i-1] * q_i(d_{i+1}) < p_i(d_{i+1})
 *   and continue while accepted (j = i+1), stop at the first rejection.
 *   The token t* at row j:
 *     greedy: argmax l_j;
 *     rejection, j < n: residual w = max(0, p_j - q_j) (all zero -> w = p_j);
 *     rejection, j = n: w = p_j (bonus token);
 *     t* = smallest t with u[n-1] * sum(w) < sum_{x<=t} w(x), summed in index order.
 *   Emitted tokens: d_2..d_j, then t* (j tokens), -1 padded to n.
 *   selected_block = j (0 when k = 0, which has no mask blocks).
 *   next_drafts = [t*, g_{j,2}, .., g_{j,k}] (-1 where block_guesses is NULL).
 *
 * margins [B][n] (may be NULL), rejection only: entry i-1 is the relative
 * distance |u q - p| / p of the i-th accept test (i <= j-1 accepted ones and the
 * rejecting one), entry n-1 the distance of u*sum(w) to the nearest boundary of
 * the cumulative sum, divided by sum(w).  Unused entries are +inf.  They let a
 * test exclude decisions that differ only by summation order.
 */
int tidar_oracle_verify(int B, int k, int V, int dtype, int mode, const void* logits,
                        const int32_t* drafts, const void* draft_logits, const float* uniforms,
                        const int32_t* block_guesses, int32_t* accept_count, int32_t* out_tokens,
                        int32_t* next_drafts, int32_t* selected_block, double* margins) {
  const int n = k > 0 ? k : 1;
  double *p, *qd, *w;
  int b;
  if (B < 0 || k < 0 || V <= 0 || (mode != 0 && mode != 1)) return ORACLE_ERR_ARG;
  if (k > 1 && !drafts) return ORACLE_ERR_ARG;
  if (mode == 1 && (!uniforms || (k > 1 && !draft_logits))) return ORACLE_ERR_ARG;
  p = (double*)malloc(sizeof(double) * V);
  qd = (double*)malloc(sizeof(double) * V);
  w = (double*)malloc(sizeof(double) * V);
  if (!p || !qd || !w) { free(p); free(qd); free(w); return ORACLE_ERR_ARG; }

  for (b = 0; b < B; ++b) {
    int i, j = 1, x, t_star = 0, e;
    if (margins) for (i = 0; i < n; ++i) margins[(int64_t)b * n + i] = INFINITY;

    /* accept scan, left to right */
    for (i = 1; i <= n - 1; ++i) {
      int d_next = drafts[(int64_t)b * k + i];   /* d_{i+1} */
      int64_t lrow = ((int64_t)b * n + (i - 1)) * V;
      int accept;
      if (d_next < 0 || d_next >= V) { accept = 0; }
      else if (mode == 0) {
        accept = (d_next == argmax_row(logits, lrow, V, dtype));
      } else {
        double u = (double)uniforms[(int64_t)b * n + (i - 1)];
        int64_t qrow = ((int64_t)b * (k - 1) + (i - 1)) * V;
        softmax_row(logits, lrow, V, dtype, p);
        softmax_row(draft_logits, qrow, V, dtype, qd);
        accept = (u * qd[d_next] < p[d_next]);
        if (margins)
          margins[(int64_t)b * n + (i - 1)] = fabs(u * qd[d_next] - p[d_next]) / p[d_next];
      }
      if (!accept) break;
      j = i + 1;
    }

    /* the token at row j */
    {
      int64_t lrow = ((int64_t)b * n + (j - 1)) * V;
      if (mode == 0) {
        t_star = argmax_row(logits, lrow, V, dtype);
      } else {
        double u = (double)uniforms[(int64_t)b * n + (n - 1)];
        double total = 0.0, c = 0.0, target, prev = 0.0;
        softmax_row(logits, lrow, V, dtype, p);
        if (j < n) {
          int64_t qrow = ((int64_t)b * (k - 1) + (j - 1)) * V;
          softmax_row(draft_logits, qrow, V, dtype, qd);
          for (x = 0; x < V; ++x) { double r = p[x] - qd[x]; w[x] = r > 0.0 ? r : 0.0; total += w[x]; }
          if (!(total > 0.0)) { for (x = 0; x < V; ++x) w[x] = p[x]; total = 0.0; for (x = 0; x < V; ++x) total += w[x]; }
        } else {
          for (x = 0; x < V; ++x) { w[x] = p[x]; total += w[x]; }
        }
        target = u * total;
        t_star = V - 1;
        for (x = 0; x < V; ++x) {
          prev = c;
          c += w[x];
          if (target < c) { t_star = x; break; }
        }
        if (margins) {
          double lo = target - prev, hi = c - target;
          margins[(int64_t)b * n + (n - 1)] = (lo < hi ? lo : hi) / total;
        }
      }
    }

    /* outputs */
    accept_count[b] = j;
    for (e = 0; e < n; ++e) out_tokens[(int64_t)b * n + e] = -1;
    for (e = 0; e < j - 1; ++e) out_tokens[(int64_t)b * n + e] = drafts[(int64_t)b * k + e + 1];
    out_tokens[(int64_t)b * n + j - 1] = t_star;
    if (selected_block) selected_block[b] = k > 0 ? j : 0;
    if (next_drafts && k > 0) {
      next_drafts[(int64_t)b * k] = t_star;
      for (e = 1; e < k; ++e)
        next_drafts[(int64_t)b * k + e] =
            block_guesses ? block_guesses[((int64_t)b * k + (j - 1)) * k + e] : -1;
    }
  }
  free(p); free(qd); free(w);
  return ORACLE_OK;
}

/*
 * The sampling transform of a logit row, applied alike to the AR
 * distribution p and to the draft distribution q.  The pages fix no
 * temperature or truncation (they speak only of sampling from the AR
 * distribution, [EN] section "TiDAR 在做什麼", and of drafting from the mask
 * blocks' marginals, [MS] §2); this is the plainest reading of the usual
 * sampling controls, and the speculative-sampling rule stays exact for any
 * pair (p, q) it produces:
 *   temperature T > 0:   p(x) proportional to exp(l(x) / T);
 *   nucleus top_p:       order the tokens larger logit first, lower index first
 *                        among equal logits; keep token x iff the probability
 *                        of the tokens before it is below top_p (so the kept run
 *                        is the shortest one reaching top_p); renormalise the
 *                        kept tokens (sum in index order).  top_p >= 1 keeps
 *                        every token.
 * Writes p[0..V-1] (fp64).  cut_margin (may be NULL) receives the distance of
 * top_p to the nearest cumulative sum around the cut -- min(top_p - mass before
 * the last kept token, mass through it - top_p) / top_p -- or +inf without
 * truncation: a decision that close to a tie is fixed by summation order only.
 */
typedef struct {
  double v;
  int x;
} oracle_tok;

static int tok_order(const void* a, const void* b) {
  const oracle_tok* p = (const oracle_tok*)a;
  const oracle_tok* q = (const oracle_tok*)b;
  if (p->v > q->v) return -1;
  if (p->v < q->v) return 1;
  return p->x < q->x ? -1 : (p->x > q->x ? 1 : 0);
}

static int dist_row(const void* base, int64_t off, int V, int dtype, double T, double top_p,
                    double* p, double* cut_margin) {
  double m = -INFINITY, z = 0.0;
  int x;
  if (cut_margin) *cut_margin = INFINITY;
  for (x = 0; x < V; ++x) { double v = elem(base, off + x, dtype) / T; if (v > m) m = v; }
  for (x = 0; x < V; ++x) { p[x] = exp(elem(base, off + x, dtype) / T - m); z += p[x]; }
  for (x = 0; x < V; ++x) p[x] /= z;
  if (top_p < 1.0) {
    oracle_tok* t = (oracle_tok*)malloc(sizeof(oracle_tok) * (size_t)V);
    char* keep = (char*)malloc((size_t)V);
    double cum = 0.0, before_last = 0.0, through_last = 0.0, s = 0.0;
    int i;
    if (!t || !keep) { free(t); free(keep); return ORACLE_ERR_ARG; }
    for (x = 0; x < V; ++x) { t[x].v = elem(base, off + x, dtype); t[x].x = x; keep[x] = 0; }
    qsort(t, (size_t)V, sizeof(oracle_tok), tok_order);
    for (i = 0; i < V; ++i) {
      if (cum < top_p) {
        keep[t[i].x] = 1;
        before_last = cum;
        through_last = cum + p[t[i].x];
      }
      cum += p[t[i].x];
    }
    for (x = 0; x < V; ++x) if (keep[x]) s += p[x];
    for (x = 0; x < V; ++x) p[x] = keep[x] ? p[x] / s : 0.0;
    if (cut_margin) {
      double lo = top_p - before_last, hi = through_last - top_p;
      *cut_margin = (lo < hi ? lo : hi) / top_p;
    }
    free(t);
    free(keep);
  }
  return ORACLE_OK;
}

/* The transformed distribution of one logit row (for the pins in tests/). */
int tidar_oracle_dist_row(int V, int dtype, double T, double top_p, const void* row, double* p,
                          double* cut_margin) {
  if (V <= 0 || !(T > 0.0) || !(top_p > 0.0)) return ORACLE_ERR_ARG;
  return dist_row(row, 0, V, dtype, T, top_p, p, cut_margin);
}

/*
 * Verification with the sampling transform: the algorithm of
 * tidar_oracle_verify, step by step, with p_i and q_i taken through
 * dist_row(T, top_p).  Greedy acceptance is unchanged by the transform (the
 * most likely token is always kept and T > 0 keeps the order), so greedy
 * ignores T and top_p.  cut_margins [B] (may be NULL) receives, per sequence,
 * the smallest cut margin of the rows its decisions read (+inf without
 * truncation).
 */
int tidar_oracle_verify_sampled(int B, int k, int V, int dtype, int mode, double T, double top_p,
                                const void* logits, const int32_t* drafts, const void* draft_logits,
                                const float* uniforms, const int32_t* block_guesses,
                                int32_t* accept_count, int32_t* out_tokens, int32_t* next_drafts,
                                int32_t* selected_block, double* margins, double* cut_margins) {
  const int n = k > 0 ? k : 1;
  double *p, *qd, *w;
  int b;
  if (B < 0 || k < 0 || V <= 0 || (mode != 0 && mode != 1) || !(T > 0.0) || !(top_p > 0.0))
    return ORACLE_ERR_ARG;
  if (k > 1 && !drafts) return ORACLE_ERR_ARG;
  if (mode == 1 && (!uniforms || (k > 1 && !draft_logits))) return ORACLE_ERR_ARG;
  p = (double*)malloc(sizeof(double) * V);
  qd = (double*)malloc(sizeof(double) * V);
  w = (double*)malloc(sizeof(double) * V);
  if (!p || !qd || !w) { free(p); free(qd); free(w); return ORACLE_ERR_ARG; }

  for (b = 0; b < B; ++b) {
    int i, j = 1, x, t_star = 0, e;
    double cm = INFINITY, c1;
    if (margins) for (i = 0; i < n; ++i) margins[(int64_t)b * n + i] = INFINITY;

    /* accept scan, left to right */
    for (i = 1; i <= n - 1; ++i) {
      int d_next = drafts[(int64_t)b * k + i];   /* d_{i+1} */
      int64_t lrow = ((int64_t)b * n + (i - 1)) * V;
      int accept;
      if (d_next < 0 || d_next >= V) { accept = 0; }
      else if (mode == 0) {
        accept = (d_next == argmax_row(logits, lrow, V, dtype));
      } else {
        double u = (double)uniforms[(int64_t)b * n + (i - 1)];
        int64_t qrow = ((int64_t)b * (k - 1) + (i - 1)) * V;
        dist_row(logits, lrow, V, dtype, T, top_p, p, &c1);
        if (c1 < cm) cm = c1;
        dist_row(draft_logits, qrow, V, dtype, T, top_p, qd, &c1);
        if (c1 < cm) cm = c1;
        accept = (u * qd[d_next] < p[d_next]);
        if (margins && p[d_next] > 0.0)
          margins[(int64_t)b * n + (i - 1)] = fabs(u * qd[d_next] - p[d_next]) / p[d_next];
      }
      if (!accept) break;
      j = i + 1;
    }

    /* the token at row j */
    {
      int64_t lrow = ((int64_t)b * n + (j - 1)) * V;
      if (mode == 0) {
        t_star = argmax_row(logits, lrow, V, dtype);
      } else {
        double u = (double)uniforms[(int64_t)b * n + (n - 1)];
        double total = 0.0, c = 0.0, target, prev = 0.0;
        dist_row(logits, lrow, V, dtype, T, top_p, p, &c1);
        if (c1 < cm) cm = c1;
        if (j < n) {
          int64_t qrow = ((int64_t)b * (k - 1) + (j - 1)) * V;
          dist_row(draft_logits, qrow, V, dtype, T, top_p, qd, &c1);
          if (c1 < cm) cm = c1;
          for (x = 0; x < V; ++x) { double r = p[x] - qd[x]; w[x] = r > 0.0 ? r : 0.0; total += w[x]; }
          if (!(total > 0.0)) { for (x = 0; x < V; ++x) w[x] = p[x]; total = 0.0; for (x = 0; x < V; ++x) total += w[x]; }
        } else {
          for (x = 0; x < V; ++x) { w[x] = p[x]; total += w[x]; }
        }
        target = u * total;
        t_star = V - 1;
        for (x = 0; x < V; ++x) {
          prev = c;
          c += w[x];
          if (target < c) { t_star = x; break; }
        }
        if (margins) {
          double lo = target - prev, hi = c - target;
          margins[(int64_t)b * n + (n - 1)] = (lo < hi ? lo : hi) / total;
        }
      }
    }
    if (cut_margins) cut_margins[b] = cm;

    /* outputs */
    accept_count[b] = j;
    for (e = 0; e < n; ++e) out_tokens[(int64_t)b * n + e] = -1;
    for (e = 0; e < j - 1; ++e) out_tokens[(int64_t)b * n + e] = drafts[(int64_t)b * k + e + 1];
    out_tokens[(int64_t)b * n + j - 1] = t_star;
    if (selected_block) selected_block[b] = k > 0 ? j : 0;
    if (next_drafts && k > 0) {
      next_drafts[(int64_t)b * k] = t_star;
      for (e = 1; e < k; ++e)
        next_drafts[(int64_t)b * k + e] =
            block_guesses ? block_guesses[((int64_t)b * k + (j - 1)) * k + e] : -1;
    }
  }
  free(p); free(qd); free(w);
  return ORACLE_OK;
}

/*
 * The next step's drafts from the selected mask block ([MS] §2: the mask slots
 * give the diffusion predictions the next drafts come from; [NDfr] paragraph on
 * betting on every outcome: the block matching the accept count is the one
 * waiting).  With j = selected_block[b] (a value outside 1..k reads block 1 and
 * the call returns ORACLE_ERR_COUNT), slot s = 2..k of block j supplies
 * next_drafts[b][s-1]:
 *   greedy (mode 0): the slot row's argmax (lowest index on ties);
 *   sampling (mode 1): the smallest t with u[b][s-1] * 1 < sum_{x<=t} q_s(x),
 *     q_s = dist_row(T, top_p) of the slot row, summed in index order (the
 *     same inverse CDF as t*).
 * next_drafts[b][0] (t*, from verification) is left as it is.
 *   block_logits [B][k][k][V] (block j-1, slot s-1), uniforms [B][k] (mode 1).
 * margins [B][k] (may be NULL): the distance of u to the nearest cumulative
 * sum (mode 1), +inf elsewhere.
 */
int tidar_oracle_sample_drafts(int B, int k, int V, int dtype, int mode, double T, double top_p,
                               const void* block_logits, const int32_t* selected_block,
                               const float* uniforms, int32_t* next_drafts, double* margins) {
  double* q;
  int b, status = ORACLE_OK;
  if (B < 0 || k < 0 || V <= 0 || (mode != 0 && mode != 1) || !(T > 0.0) || !(top_p > 0.0))
    return ORACLE_ERR_ARG;
  if (mode == 1 && !uniforms) return ORACLE_ERR_ARG;
  q = (double*)malloc(sizeof(double) * V);
  if (!q) return ORACLE_ERR_ARG;
  for (b = 0; b < B; ++b) {
    int j = selected_block[b], s;
    if (margins) for (s = 0; s < k; ++s) margins[(int64_t)b * k + s] = INFINITY;
    if (j < 1 || j > k) { j = 1; status = ORACLE_ERR_COUNT; }
    for (s = 2; s <= k; ++s) {
      const int64_t row = (((int64_t)b * k + (j - 1)) * k + (s - 1)) * V;
      int tok;
      if (mode == 0) {
        tok = argmax_row(block_logits, row, V, dtype);
      } else {
        double u = (double)uniforms[(int64_t)b * k + (s - 1)], c = 0.0, prev = 0.0, total = 0.0, c1;
        int x;
        dist_row(block_logits, row, V, dtype, T, top_p, q, &c1);
        for (x = 0; x < V; ++x) total += q[x];
        tok = V - 1;
        for (x = 0; x < V; ++x) {
          prev = c;
          c += q[x];
          if (u * total < c) { tok = x; break; }
        }
        if (margins) {
          double lo = u * total - prev, hi = c - u * total, mm = (lo < hi ? lo : hi) / total;
          margins[(int64_t)b * k + (s - 1)] = mm < c1 ? mm : c1;
        }
      }
      next_drafts[(int64_t)b * k + (s - 1)] = tok;
    }
  }
  free(q);
  return status;
}

/*
 * KV commit / evict ("the settled cache is reused, the rejected entries are
 * evicted", [NDfr] paragraph on the three zones; exact KV cache, [MS] "KV
 * Cache" and [FG] abstract).  Accepted drafts are always a prefix of the draft
 * zone ([NDfr]: "only the first survives, two survive, all survive"), so no row
 * moves.  For each b with c = accept_count[b] in 0..n:
 *   rows P_b+c .. P_b+n-1 of every KV head are set to zero (K and V);
 *   seq_lens[b] = P_b + c;
 *   page-table entries i in [ceil((P_b+c)/ps), ceil((P_b+n)/ps)) -- the pages
 *   that held only rejected draft rows -- are released: their ids are appended
 *   to `released` in (b, i) order and the entries set to -1.
 * `released` holds B*(ceil(n/ps)+1) entries, -1 padded; *num_released counts
 * the ids written.  A sequence with c out of range, or whose draft rows are
 * not mapped to valid pages, is left untouched and the call returns an error.
 */
int tidar_oracle_commit(int B, int Hkv, int D, int k, int page_size, int elem_bytes,
                        void* k_pages, void* v_pages, int32_t* page_table, int max_pages,
                        int num_pages, int32_t* seq_lens, const int32_t* accept_count,
                        int32_t* released, int32_t* num_released) {
  const int n = k > 0 ? k : 1;
  const int cap = B * ((n + page_size - 1) / page_size + 1);
  int b, status = ORACLE_OK, count = 0, e;
  for (e = 0; e < cap; ++e) released[e] = -1;
  for (b = 0; b < B; ++b) {
    int P = seq_lens[b], c = accept_count[b], r, g, ok = 1;
    int64_t i, first, last;
    if (c < 0 || c > n) { status = ORACLE_ERR_COUNT; continue; }
    for (r = 0; r < n && ok; ++r)
      if (cache_row(page_table, max_pages, num_pages, page_size, Hkv, D, b, 0, (int64_t)P + r) < 0)
        ok = 0;
    if (!ok) { status = ORACLE_ERR_PAGE; continue; }
    for (r = c; r < n; ++r) {
      for (g = 0; g < Hkv; ++g) {
        int64_t row = cache_row(page_table, max_pages, num_pages, page_size, Hkv, D, b, g,
                                (int64_t)P + r);
        memset((char*)k_pages + row * elem_bytes, 0, (size_t)D * elem_bytes);
        memset((char*)v_pages + row * elem_bytes, 0, (size_t)D * elem_bytes);
      }
    }
    seq_lens[b] = P + c;
    first = ((int64_t)P + c + page_size - 1) / page_size;
    last = ((int64_t)P + n + page_size - 1) / page_size;
    for (i = first; i < last; ++i) {
      int32_t* ent = &page_table[(int64_t)b * max_pages + i];
      if (*ent >= 0) { released[count++] = *ent; *ent = -1; }
    }
  }
  *num_released = count;
  return status;
}

/*
 * Page reservation for a step's draft rows, from a stack of free pages.
 *
 * The pages evict the rejected entries and reuse the settled cache ([NDfr]
 * paragraph on the three zones); the step's draft rows P_b .. P_b+n-1 need
 * cache pages before they are written ([NDfr], same paragraph: candidates
 * carried from the previous step sit after the settled tokens).  The pages say
 * nothing about where those pages come from.  The plainest reading, taken
 * here: the pages a commit released return to a pool, and the pool is a stack
 * (the last page returned is the first reused).  Flags, not statuses, because
 * several can arise in one call:
 *   1. The `returned` ids (num_returned >= 0 of them; returned may be NULL
 *      when that is 0) are pushed in order: free[count + t] = returned[t].
 *      If num_returned < 0 or count + num_returned > capacity, nothing at all
 *      changes and RESERVE_FLAG_POOL is returned.
 *   2. For each b, with P = seq_lens[b]: if P < 0 or P > max_prefix or
 *      ceil((P+n)/ps) > max_pages, RESERVE_FLAG_LEN and b is skipped.  Rows
 *      P .. P+n-1 lie on entries floor(P/ps) .. ceil((P+n)/ps)-1.  An entry
 *      below ceil(P/ps) also holds prefix rows and must be a page in
 *      [0, num_pages); an entry at or above it is a page in [0, num_pages)
 *      (kept) or -1 (needs a page).  Anything else: RESERVE_FLAG_PAGE and b is
 *      skipped.
 *   3. If the entries that need a page outnumber count, no entry changes and
 *      RESERVE_FLAG_POOL is raised (the push of step 1 stands).
 *   4. Otherwise the needing entries, in (b, i) order, pop the stack one by
 *      one: the t-th takes free[count - 1 - t]; count drops by their number.
 * Popped ids are not checked; the step attention reports an out-of-range one.
 */
#define RESERVE_FLAG_PAGE 1
#define RESERVE_FLAG_LEN 2
#define RESERVE_FLAG_POOL 4

/* Classifies sequence b: returns -1 (and sets *flag) if it is skipped, else the
 * number of its entries that need a page. */
static int reserve_need(int b, int n, int page_size, int max_prefix, const int32_t* page_table,
                        int max_pages, int num_pages, const int32_t* seq_lens, int* flag) {
  const int64_t P = seq_lens[b];
  int64_t i, lo, settled, hi;
  int need = 0;
  if (P < 0 || P > max_prefix || (P + n + page_size - 1) / page_size > max_pages) {
    *flag |= RESERVE_FLAG_LEN;
    return -1;
  }
  lo = P / page_size;
  settled = (P + page_size - 1) / page_size;   /* entries below hold prefix rows */
  hi = (P + n + page_size - 1) / page_size;
  for (i = lo; i < hi; ++i) {
    const int32_t e = page_table[(int64_t)b * max_pages + i];
    if (e >= 0 && e < num_pages) continue;
    if (e == -1 && i >= settled) { ++need; continue; }
    *flag |= RESERVE_FLAG_PAGE;
    return -1;
  }
  return need;
}

int tidar_oracle_reserve(int B, int k, int page_size, int max_prefix, int32_t* page_table,
                         int max_pages, int num_pages, const int32_t* seq_lens,
                         int32_t* free_pages, int32_t* free_count, int capacity,
                         const int32_t* returned, int num_returned) {
  const int n = k > 0 ? k : 1;
  int flag = 0, b, t, total = 0, count = *free_count;
  int64_t i;
  if (num_returned < 0 || (int64_t)count + num_returned > capacity) return RESERVE_FLAG_POOL;
  for (t = 0; t < num_returned; ++t) free_pages[count + t] = returned[t];
  count += num_returned;
  *free_count = count;
  for (b = 0; b < B; ++b) {
    const int need = reserve_need(b, n, page_size, max_prefix, page_table, max_pages, num_pages,
                                  seq_lens, &flag);
    if (need > 0) total += need;
  }
  if (total > count) return flag | RESERVE_FLAG_POOL;
  t = 0;
  for (b = 0; b < B; ++b) {
    int unused = 0;
    const int64_t P = seq_lens[b];
    if (reserve_need(b, n, page_size, max_prefix, page_table, max_pages, num_pages, seq_lens,
                     &unused) <= 0)
      continue;
    for (i = (P + page_size - 1) / page_size; i < (P + n + page_size - 1) / page_size; ++i) {
      int32_t* e = &page_table[(int64_t)b * max_pages + i];
      if (*e == -1) *e = free_pages[count - 1 - t++];
    }
  }
  *free_count = count - total;
  return flag;
}

/*
 * The draft distributions of a step, taken from the previous step's mask
 * blocks.  Each block of k slots drafts the k tokens that follow one possible
 * accept count ([NDfr] paragraph on betting on every outcome: one guess block
 * per future, the matching one is waiting when verification confirms it;
 * [MS] §2: the pre-drafts are sampled from the diffusion predictions of the
 * mask slots).  The selected block j becomes the next step's drafts
 * [t*, g_{j,2}, .., g_{j,k}], so draft d_{i+1} (i >= 1) is slot i+1 of block j
 * and was drawn from that slot's distribution: q_i = softmax(row (j-1, i) of
 * the block logits).  Plainest reading of the slot order: slot s of block j is
 * row (j-1)*k + (s-1) of the [k][k][V] logits, slot 1 being the one t* replaces.
 *
 *   block_logits [B][k][k][V] (dtype), draft_block [B] (the previous step's
 *   selected block, 1..k).  Writes draft_logits [B][k-1][V]: row i-1 = block
 *   logits row (draft_block[b]-1, i), i = 1..k-1.  A draft_block outside 1..k
 *   reads block 1 and raises GATHER_FLAG_BLOCK.  Returns the flags.
 */
#define GATHER_FLAG_BLOCK 1
int tidar_oracle_gather_block_q(int B, int k, int V, int elem_bytes, const void* block_logits,
                                const int32_t* draft_block, void* draft_logits) {
  int b, i, flags = 0;
  if (k < 2) return 0;
  for (b = 0; b < B; ++b) {
    int j = draft_block[b];
    if (j < 1 || j > k) { flags |= GATHER_FLAG_BLOCK; j = 1; }
    for (i = 1; i <= k - 1; ++i) {
      const int64_t src = (((int64_t)b * k + (j - 1)) * k + i) * V;
      const int64_t dst = ((int64_t)b * (k - 1) + (i - 1)) * V;
      memcpy((char*)draft_logits + dst * elem_bytes, (const char*)block_logits + src * elem_bytes,
             (size_t)V * elem_bytes);
    }
  }
  return flags;
}

/*
 * Layer-level pieces around the step attention (for a step with synthetic
 * weights: query/key/value projection, rotary position embedding at the zone
 * positions, output projection).  The pages describe one backbone doing both
 * jobs in one pass ([NDfr] paragraph on the three zones) and a mask placed so
 * that it slides forward as the text grows ([NDfr] masking paragraph); they do
 * not give the position of each row or the position encoding.  Readings taken
 * here (the plainest ones the rest supports):
 *   - draft row r (1..k) sits at position P + r - 1, the cache row it is
 *     appended at;
 *   - mask slot s of block j sits at P + j + s - 1: block j drafts the tokens
 *     that follow d_1..d_j, so slot 1 is where t* lands when j drafts are
 *     accepted and slots 2..k become the next step's drafts d_2..d_k there;
 *   - k = 0: the single row sits at P;
 *   - rotary embedding in the rotate-half form: dims f and f + D/2 of a head
 *     form a pair rotated by the angle pos * base^(-2f/D), f = 0..D/2-1.
 */

/* Positions of the R query rows of a step with committed length P. */
int tidar_oracle_zone_positions(int k, int64_t P, int64_t* pos) {
  int r, j, s;
  if (k < 0) return ORACLE_ERR_ARG;
  if (k == 0) { pos[0] = P; return ORACLE_OK; }
  for (r = 1; r <= k; ++r) pos[r - 1] = P + r - 1;
  for (j = 1; j <= k; ++j)
    for (s = 1; s <= k; ++s) pos[k + (j - 1) * k + (s - 1)] = P + j + s - 1;
  return ORACLE_OK;
}

/* Rotary embedding of x [rows][H][D] (fp32 or bf16) at pos[rows], in fp64:
 *   out[f]       = x[f] cos(a_f) - x[f + D/2] sin(a_f)
 *   out[f + D/2] = x[f] sin(a_f) + x[f + D/2] cos(a_f),   a_f = pos * base^(-2f/D). */
int tidar_oracle_rope(int rows, int H, int D, double base, const int64_t* pos, const void* x,
                      int dtype, double* out) {
  int r, h, f;
  if (rows < 0 || H <= 0 || D <= 0 || (D & 1) || base <= 0.0) return ORACLE_ERR_ARG;
  for (r = 0; r < rows; ++r)
    for (h = 0; h < H; ++h) {
      const int64_t o = ((int64_t)r * H + h) * D;
      for (f = 0; f < D / 2; ++f) {
        const double ang = (double)pos[r] * pow(base, -2.0 * f / D);
        const double c = cos(ang), sn = sin(ang);
        const double a = elem(x, o + f, dtype), b = elem(x, o + f + D / 2, dtype);
        out[o + f] = a * c - b * sn;
        out[o + f + D / 2] = a * sn + b * c;
      }
    }
  return ORACLE_OK;
}

/* y [M][N] = x [M][K] times the transpose of w [N][K] (a linear layer whose
 * weight rows are its outputs), fp64 sums in index order. */
int tidar_oracle_linear(int M, int N, int K, const void* x, int x_dtype, const void* w,
                        int w_dtype, double* y) {
  int64_t mn;
  if (M < 0 || N < 0 || K < 0) return ORACLE_ERR_ARG;
  /* each output is its own index-order sum; the outputs are independent, so
     they are spread over the host's cores (the arithmetic does not change) */
#pragma omp parallel for schedule(static)
  for (mn = 0; mn < (int64_t)M * N; ++mn) {
    const int64_t m = mn / N, n = mn % N;
    int kk;
    double acc = 0.0;
    for (kk = 0; kk < K; ++kk)
      acc += elem(x, m * K + kk, x_dtype) * elem(w, n * K + kk, w_dtype);
    y[m * N + n] = acc;
  }
  return ORACLE_OK;
}
