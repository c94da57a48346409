/*
 * libeagle_tree -- one EAGLE tree-verification step on NVIDIA B200 (sm_100a).
 *
 * The step (as described on three web pages about EAGLE / EAGLE-2 / EAGLE-3 /
 * EAGLE-4):
 *   1. build the EAGLE-2 dynamic draft tree from draft logits: confidence
 *      c(x) = softmax(draft logits)_x, global acceptance V = product of the
 *      confidences on the root path, per-level top-k expansion, rerank to the
 *      best m nodes                       ("EAGLE" notes, section EAGLE-2:
 *      "Well-Calibrated Draft Model", "Expansion of tree", "Reranking Nodes");
 *   2. per-node ancestor bitmask: a tree token attends to the shared prefix,
 *      its ancestors and itself, never to siblings or other branches
 *      ("Технический анализ EAGLE-4", section "Деревья проверки EAGLE-4 и
 *      утилита управления");
 *   3. tree-masked attention of the m tree queries over the prefix KV cache
 *      plus the tree's own keys ("Tree Attention" for verification, "EAGLE"
 *      notes "3.Verify"; mask semantics as in 2; optional sliding window as in
 *      the EAGLE-4 drafter, section "Архитектура EAGLE-4");
 *   4. acceptance: greedy longest path of target argmaxes, or sampling that
 *      accepts a draft token with probability min(1, p_target/p_draft) and
 *      resamples from the normalised max(0, p_target - p_draft) ("EAGLE" notes,
 *      EAGLE-2 "Well-Calibrated Draft Model"; "Что такое EAGLE-3", section 4
 *      steps 3-4).
 * Around it: the whole step as one call (eagle_verify_step); the tree grown
 * one level at a time for a draft model in the loop (eagle_tree_grow_*), with
 * the EAGLE-4 harness's cost-aware sizing (eagle_cost_at,
 * eagle_size_keep_level); EAGLE-1's static tree (eagle_static_tree_build);
 * sampling without replacement (eagle_accept_with_rule); a paged prefix cache
 * (eagle_tree_attention_paged); and the accepted path's keys and values into
 * the cache (eagle_kv_compact, _paged).
 *
 * Conventions shared by every entry point
 *   - All array arguments are DEVICE pointers owned by the caller, unless a
 *     parameter says otherwise.  Arrays are dense, row-major, in the index
 *     order written in brackets.  The library allocates nothing; kernels that
 *     need scratch space take a caller-provided workspace (size from the
 *     matching *_workspace_bytes function, 256-byte aligned).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work; outputs are valid after the
 *     stream is synchronised.  No call synchronises the host.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a non-zero eagle_status and launches nothing.  A
 *     failed launch returns EAGLE_ERR_CUDA (the CUDA error string is available
 *     from eagle_last_cuda_error()).  What the host cannot see (device data
 *     such as a paged cache's page ids, or a wait inside a kernel that gave
 *     up) is reported through a device status word in the workspace (see
 *     eagle_tree_attention); no kernel traps.
 *   - Logits are fp32 (EAGLE_F32) or bf16 (EAGLE_BF16, raw 16-bit patterns).
 *     Rows must hold finite values; at least k values per row must be > -inf
 *     where a top-k is taken.  Attention tensors (q, K, V) are bf16.
 *   - Ties: every top-k and argmax orders by value, then by LOWER token id;
 *     every node ranking orders by log V, then by lower candidate id.
 *
 * Tree layout (one tree per sequence b; n = min(m, P) nodes, P the pool size)
 *   nodes are numbered 1..n, node 0 is the root (the last accepted token, the
 *   last entry of the prefix KV cache).  Node order = ascending candidate id,
 *   so a parent always precedes its children and siblings are in confidence
 *   order.
 *     tokens   [B][n] int32   token of node i+1
 *     parents  [B][n] int32   parent node id of node i+1 (0 = root)
 *     depth    [B][n] int32   1..tree depth
 *     logV     [B][n] float   log of the global acceptance V of node i+1
 *     gid      [B][n] int32   candidate id (level-major, see eagle_tree_build)
 *     draft_row[B][n+1] int32 draft-logit row holding node j's distribution
 *                             (j = 0 is the root -> row 0), -1 if never expanded
 *     row_lse  [B][R] double  log-sum-exp of every draft row
 *     mask     [B][n][2] uint64  bit j%64 of word j/64 set iff node j+1 is node
 *                             i+1 or one of its ancestors (n <= 128)
 *     pos      [B][n] int32   position id: prefix_len[b] - 1 + depth
 */
#ifndef EAGLE_TREE_H
#define EAGLE_TREE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EAGLE_API __attribute__((visibility("default")))
#else
#define EAGLE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  EAGLE_OK = 0,
  EAGLE_ERR_NULL = 1,       /* a required pointer is NULL */
  EAGLE_ERR_SHAPE = 2,      /* a size is non-positive or sizes disagree */
  EAGLE_ERR_DTYPE = 3,      /* unsupported element type */
  EAGLE_ERR_LIMIT = 4,      /* a size exceeds a compiled limit below */
  EAGLE_ERR_WORKSPACE = 5,  /* workspace missing, too small or misaligned */
  EAGLE_ERR_ALIGN = 6,      /* a tensor pointer is not 16-byte aligned */
  EAGLE_ERR_CUDA = 7        /* a CUDA launch or runtime call failed */
} eagle_status;

typedef enum { EAGLE_F32 = 0, EAGLE_BF16 = 1 } eagle_dtype;

#define EAGLE_MAX_NODES 128   /* m (nodes per tree, root excluded) */
#define EAGLE_MAX_TOPK 32     /* k */
#define EAGLE_MAX_DEPTH 16    /* tree depth */
#define EAGLE_MAX_POOL 4096   /* P = k + (depth-1) k^2 candidates per tree */
#define EAGLE_MASK_WORDS 2    /* uint64 words per mask row */

/* Device pointers of one batch of trees (see "Tree layout" above).  gid may be
 * NULL when not wanted; the others are required by eagle_tree_build. */
typedef struct {
  int32_t* tokens;
  int32_t* parents;
  int32_t* depth;
  float* logV;
  int32_t* gid;
  int32_t* draft_row;
  double* row_lse;
} eagle_tree_t;

/* Human-readable name of a status code (static string). */
EAGLE_API const char* eagle_status_string(int status);
/* Text of the last CUDA error seen by this library in this thread ("" if none). */
EAGLE_API const char* eagle_last_cuda_error(void);
/* Library version, major*10000 + minor*100 + patch. */
EAGLE_API int eagle_version(void);

/* ---------------------------------------------------------------- row stats
 * Per logit row: the k largest logits (ties to the lower token id) and the
 * log-sum-exp, i.e. what turns logits into confidences c(x) = exp(l_x - lse)
 * ("EAGLE" notes, EAGLE-2 "Well-Calibrated Draft Model").
 *   logits      [rows][V] (dtype)
 *   topk_token  [rows][k] int32, descending logit (may be NULL)
 *   topk_logit  [rows][k] float  (may be NULL)
 *   lse         [rows]    double (may be NULL)
 * Limits: 1 <= k <= min(V, EAGLE_MAX_TOPK).  Workspace: eagle_row_stats_workspace_bytes. */
EAGLE_API size_t eagle_row_stats_workspace_bytes(long long rows, int V, int dtype, int k);
EAGLE_API eagle_status eagle_row_stats(const void* logits, int dtype, long long rows, int V, int k,
                             int32_t* topk_token, float* topk_logit, double* lse,
                             void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------- tree build
 * EAGLE-2 dynamic tree for B sequences ("EAGLE" notes, EAGLE-2 sections
 * "Expansion of tree" and "Reranking Nodes").
 *   draft_logits [B][R][V] (dtype), R = 1 + (depth-1)*k.  Row 0 is the root's
 *     distribution; the node in frontier slot s of level l (1 <= l < depth)
 *     owns row 1 + (l-1)*k + s, its children are that row's top-k tokens.
 *   Level 1 = the root's top-k children.  At each level the frontier is the
 *   k candidates with the largest log V (= sum of log confidences on the
 *   path), slot = rank.  Candidate id: gid = r at level 1 and
 *   gid = k + (l-2)k^2 + s*k + r at level l >= 2 (s = parent's slot, r = child
 *   rank).  After the last level the n = min(m, P) candidates with the
 *   largest log V over all levels are kept and numbered by ascending gid.
 *   out:      device pointers of the tree arrays (all but gid required)
 *   n_nodes:  HOST pointer, receives n (may be NULL)
 * Limits: depth <= EAGLE_MAX_DEPTH, k <= EAGLE_MAX_TOPK, k <= V,
 *         m <= EAGLE_MAX_NODES, P <= EAGLE_MAX_POOL.
 * Workspace: eagle_tree_build_workspace_bytes. */
EAGLE_API size_t eagle_tree_build_workspace_bytes(int B, int R, int V, int dtype, int k);
EAGLE_API eagle_status eagle_tree_build(const void* draft_logits, int dtype, int B, int R, int V, int depth,
                              int k, int m, const eagle_tree_t* out, int* n_nodes,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------- tree mask
 * Ancestor-or-self bitmask and position ids ("Технический анализ EAGLE-4",
 * "Деревья проверки EAGLE-4 и утилита управления").
 *   parents [B][n], depth [B][n], prefix_len [B] (int32) -> mask [B][n][2]
 *   uint64, pos [B][n] int32 (pos may be NULL; prefix_len may be NULL when pos is).
 * parents must name earlier nodes (0 <= parents[i] <= i); an out-of-range parent
 * ends that node's walk (its mask then holds the ancestors seen so far).
 * Limits: n <= EAGLE_MAX_NODES. */
EAGLE_API eagle_status eagle_tree_mask(const int32_t* parents, const int32_t* depth, const int32_t* prefix_len,
                             int B, int n, uint64_t* mask, int32_t* pos, void* stream);

/* -------------------------------------------------------- tree attention
 * out[b][i][h] = softmax_j(q[b][i][h] . key_j * scale) weighted sum of value_j
 * over the keys node i+1 may see: prefix entries p < prefix_len[b] of KV head
 * g = h / (Hq/Hkv) (with window W > 0: only p >= pos_i - W + 1) and tree
 * entries j with mask bit (i, j) set (with a window: pos_j >= pos_i - W + 1).
 *   q        [B][n][Hq][D]     bf16
 *   k_cache  [B][Hkv][Lmax][D] bf16, v_cache likewise; entries past
 *            prefix_len[b] are ignored but must be finite
 *   prefix_len [B] int32, clamped to [0, Lmax] on the device
 *   k_tree   [B][n][Hkv][D]    bf16 (keys of the tree tokens), v_tree likewise
 *   mask     [B][n][2] uint64  (from eagle_tree_mask)
 *   pos      [B][n] int32      (from eagle_tree_mask; required iff window > 0)
 *   out      [B][n][Hq][D]     bf16
 *   scale    softmax scale; <= 0 selects 1/sqrt(D)
 * Limits: D in {64, 128}, Hq % Hkv == 0, n <= EAGLE_MAX_NODES, all tensor
 * pointers 16-byte aligned.  Workspace: eagle_tree_attention_workspace_bytes.
 * It starts with a 256-byte header whose first int is the device status word,
 * rewritten by every call (0 = ok, 1 = an internal wait gave up, 3 = a paged
 * cache named a page outside its pool for a key in use); the rest holds
 * the normalised partial outputs of key ranges split across CTAs (fp32, about
 * (148 + B*Hkv*ceil(n*Hq/Hkv/128)) * 128 * (D+1) * 4 bytes).  The call launches
 * two kernels; either may start while its predecessor on the stream drains
 * (programmatic dependent launch) and waits for it before reading any input. */
EAGLE_API size_t eagle_tree_attention_workspace_bytes(int B, int n, int Hq, int Hkv, int D, int Lmax, int window);
EAGLE_API eagle_status eagle_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* prefix_len, int Lmax, const void* k_tree,
                                  const void* v_tree, const uint64_t* mask, const int32_t* pos,
                                  int B, int n, int Hq, int Hkv, int D, int window, float scale,
                                  void* out, void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------------- paged prefix cache
 * eagle_tree_attention over a paged prefix cache, for batches whose prefixes
 * differ in length: the cache is a pool of pages instead of one [Lmax] slab
 * per sequence.
 *   k_pages, v_pages [num_pages][Hkv][page_size][D] bf16 (16-byte aligned);
 *   block_table [B][pages_per_seq] int32 device: sequence b's key at position
 *     p sits at offset p % page_size of page block_table[b][p / page_size];
 *     entries past a sequence's length are not read for it (any value).
 *   page_size: 16, 32 or a multiple of 64; num_pages * Hkv * page_size < 2^31.
 *   A sequence holds up to pages_per_seq * page_size keys (prefix_len is
 *   clamped to that); pass that product as Lmax to
 *   eagle_tree_attention_workspace_bytes.
 * Everything else (q, tree K/V, mask, pos, window, scale, out, workspace) as
 * in eagle_tree_attention, with the same result up to the order of
 * floating-point sums (identical without a window).  A page id outside
 * [0, num_pages) for a key below prefix_len reads zeros and sets device
 * status 3 in the workspace header (see eagle_tree_attention).  Host errors:
 * EAGLE_ERR_NULL, EAGLE_ERR_SHAPE (page_size), EAGLE_ERR_LIMIT, EAGLE_ERR_ALIGN,
 * EAGLE_ERR_WORKSPACE. */
EAGLE_API eagle_status eagle_tree_attention_paged(const void* q, const void* k_pages, const void* v_pages,
                                                  int num_pages, int page_size, const int32_t* block_table,
                                                  int pages_per_seq, const int32_t* prefix_len, const void* k_tree,
                                                  const void* v_tree, const uint64_t* mask, const int32_t* pos,
                                                  int B, int n, int Hq, int Hkv, int D, int window, float scale,
                                                  void* out, void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------- accept
 * Walk each tree from the root ("EAGLE" notes, EAGLE-2 "Well-Calibrated Draft
 * Model"; "Что такое EAGLE-3", section 4 steps 3-4; EAGLE-4 write-up, section
 * "Деревья проверки EAGLE-4 и утилита управления").
 *   target_logits [B][n+1][V] (target_dtype): row j = target distribution
 *     after node j (row 0 after the root).
 *   uniforms == NULL -> greedy: t = argmax of the current row (ties to the
 *     lower id); move to the first child (node order) whose token is t, else
 *     stop; bonus = t.
 *   uniforms != NULL -> sampling, uniforms [B][2][n+1] float in [0, 1): row 0
 *     is u_acc indexed by the tested child's node id, row 1 is u_res indexed
 *     by the node where the walk stops.  At node j, p = softmax(target row j),
 *     q = softmax(draft row draft_row[j]).  Children in node order: accept c
 *     iff u_acc[c] < p(x_c)/q(x_c); on acceptance move to c (fresh p, q); on
 *     rejection p <- max(0, p - q) / sum(max(0, p - q)), q unchanged.  With no
 *     child left, stop and draw the bonus from the current p by inverse CDF:
 *     the smallest token i with cumsum(p)_i > u_res[j] * sum(p).
 *     draft_logits [B][R][draft_dtype] with draft_lse [B][R] (double, e.g. the
 *     tree's row_lse) encode q; both are required for sampling, ignored for
 *     greedy.
 *   tokens, parents [B][n], draft_row [B][n+1]: the tree.
 *   accepted_len [B], path [B][depth] (accepted node ids, -1 padded), bonus [B].
 * The uniforms are device data and are not checked on the host.  The walk
 * reads a u_res that is NaN or negative as 0 and one >= 1 as the largest float
 * below 1 (1 - 2^-24), so every sequence gets a bonus token; a u_acc outside
 * [0, 1) is used as given (NaN rejects).
 * Limits: n <= EAGLE_MAX_NODES, depth <= EAGLE_MAX_DEPTH; for sampling
 * V <= 262144 (bf16) or 131072 (fp32).
 * Workspace: eagle_accept_workspace_bytes. */
EAGLE_API size_t eagle_accept_workspace_bytes(int B, int n, int V, int target_dtype);

/* How q changes when a sampled child is rejected (the pages do not say):
 *   EAGLE_SAMPLE_WITH_REPLACEMENT: q is kept (eagle_accept);
 *   EAGLE_SAMPLE_WITHOUT_REPLACEMENT: for siblings drafted without replacement
 *     (distinct tokens, as top-k children always are): after the residual step
 *     the rejected token is removed from q and q renormalised,
 *     q <- q with q(x_c) = 0, divided by its remaining sum.
 *     With one child per node both rules give the same walk.  If nothing is
 *     left in q the walk stops at that node and the bonus is the target argmax. */
enum { EAGLE_SAMPLE_WITH_REPLACEMENT = 0, EAGLE_SAMPLE_WITHOUT_REPLACEMENT = 1 };

/* eagle_accept with the sampling rule chosen (ignored for greedy, uniforms ==
 * NULL); any other rule value returns EAGLE_ERR_SHAPE.  Arguments otherwise as
 * in eagle_accept. */
EAGLE_API eagle_status eagle_accept_with_rule(const void* target_logits, int target_dtype, const void* draft_logits,
                                              int draft_dtype, const double* draft_lse, int R,
                                              const int32_t* tokens, const int32_t* parents,
                                              const int32_t* draft_row, const float* uniforms, int sampling_rule,
                                              int B, int n, int V, int depth, int32_t* accepted_len,
                                              int32_t* path, int32_t* bonus, void* workspace,
                                              size_t workspace_bytes, void* stream);
EAGLE_API eagle_status eagle_accept(const void* target_logits, int target_dtype, const void* draft_logits,
                          int draft_dtype, const double* draft_lse, int R, const int32_t* tokens,
                          const int32_t* parents, const int32_t* draft_row, const float* uniforms,
                          int B, int n, int V, int depth, int32_t* accepted_len, int32_t* path,
                          int32_t* bonus, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------- tree grown one level at a time
 * The build of eagle_tree_build for a draft model that produces each level's
 * distributions only once it knows the frontier ("EAGLE" notes, EAGLE-2
 * "Expansion of tree", "Reranking Nodes").  On one stream:
 *   eagle_tree_grow_begin(root_logits [B][V])      row 0; writes the level-1
 *     frontier: frontier_tokens [B][k] (slot order), frontier_parents [B][k]
 *     (-1: the root);
 *   eagle_tree_grow_level(level_logits [B][k][V], level = 2..depth): row s is
 *     the distribution after frontier slot s of the previous level (draft row
 *     1 + (level-2)k + s of eagle_tree_build); writes the level's k best
 *     candidates, the next frontier (tokens, and each one's parent as a slot
 *     of the previous frontier);
 *   eagle_tree_grow_gains(gains [B] double, device): after begin or a level,
 *     per sequence the sum of V = exp(log V) over that level's k best
 *     candidates, the expected number of tokens they add (the gain a
 *     cost-aware harness weighs against the level's cost; EAGLE-4 write-up,
 *     "Деревья проверки EAGLE-4 и утилита управления");
 *   eagle_tree_grow_finish(levels, m, out): the tree over the first `levels`
 *     levels grown (1 <= levels <= depth; n = min(m, k + (levels-1)k^2)),
 *     equal bit for bit to eagle_tree_build with that depth on the same rows
 *     (same kernels, same fp64 log V, the rows' log-sum-exps summed in the
 *     same order).  out->row_lse is [B][R] with R = 1 + (depth-1)k; rows of
 *     levels not grown are undefined.
 * frontier pointers may be NULL.  state: eagle_tree_grow_state_bytes bytes,
 * 256-byte aligned, kept by the caller from begin to finish (it holds every
 * row's top-k and log-sum-exp and the frontier's log V).  Limits: those of
 * eagle_tree_build. */
EAGLE_API size_t eagle_tree_grow_state_bytes(int B, int V, int dtype, int depth, int k);
EAGLE_API eagle_status eagle_tree_grow_begin(const void* root_logits, int dtype, int B, int V, int depth, int k,
                                             void* state, size_t state_bytes, int32_t* frontier_tokens,
                                             int32_t* frontier_parents, void* stream);
EAGLE_API eagle_status eagle_tree_grow_level(const void* level_logits, int dtype, int B, int V, int depth, int k,
                                             int level, void* state, size_t state_bytes, int32_t* frontier_tokens,
                                             int32_t* frontier_parents, void* stream);
EAGLE_API eagle_status eagle_tree_grow_gains(int dtype, int B, int V, int depth, int k, void* state,
                                             size_t state_bytes, double* gains, void* stream);
EAGLE_API eagle_status eagle_tree_grow_finish(int dtype, int B, int V, int depth, int k, int levels, int m,
                                              void* state, size_t state_bytes, const eagle_tree_t* out,
                                              int* n_nodes, void* stream);
/* Widening or deepening (EAGLE-4 write-up, same section as the sizing below:
 * the harness widens or deepens the tree while gain over marginal cost stays
 * above a threshold, with no fixed top-k):
 *   eagle_tree_grow_level_width: as eagle_tree_grow_level, but the level is
 *     drafted from the first `width` frontier slots only (1 <= width <= k):
 *     level_logits is [B][width][V]; the other slots count as rows of -inf,
 *     whose candidates have V = 0 (token -1) and are never chosen.
 *   eagle_tree_grow_frontier_logv (logv [B][k] double, device): after begin
 *     or a level, each sequence's k best candidates of that level, log V in
 *     rank order (-inf for a candidate of V = 0); the input of
 *     eagle_size_level_width.
 *   eagle_tree_grow_finish_widths (widths HOST [levels]): the tree keeping
 *     the widths[l-1] best candidates of each level l, n = their sum nodes,
 *     numbered by ascending candidate id; requires 1 <= widths[0] <= k and
 *     1 <= widths[l] <= min(k, widths[l-1] k), level l + 1 having been drafted
 *     from widths[l-1] slots.  Errors: EAGLE_ERR_SHAPE for widths outside
 *     those bounds, EAGLE_ERR_LIMIT for n > EAGLE_MAX_NODES. */
EAGLE_API eagle_status eagle_tree_grow_level_width(const void* level_logits, int dtype, int B, int V, int depth,
                                                   int k, int level, int width, void* state, size_t state_bytes,
                                                   int32_t* frontier_tokens, int32_t* frontier_parents,
                                                   void* stream);
EAGLE_API eagle_status eagle_tree_grow_frontier_logv(int dtype, int B, int V, int depth, int k, void* state,
                                                     size_t state_bytes, double* logv, void* stream);
EAGLE_API eagle_status eagle_tree_grow_finish_widths(int dtype, int B, int V, int depth, int k, int levels,
                                                     const int* widths, void* state, size_t state_bytes,
                                                     const eagle_tree_t* out, int* n_nodes, void* stream);

/* ------------------------------------------------- cost-aware tree sizing
 * EAGLE-4 write-up, "Деревья проверки EAGLE-4 и утилита управления": a table
 * of verification latency against batch size, context length and candidates
 * per sequence, measured once on the GPU; at each draft level the gain in
 * cumulative probability over the level's marginal cost against a threshold.
 * Host functions (no device access, no stream):
 *   table: ascending grids B[nB], L[nL], N[nN] (N = candidates verified per
 *     sequence) and latencies us[nB][nL][nN] (any time unit), all finite,
 *     host memory owned by the caller.  Cost between grid points:
 *     multilinear interpolation; outside the grid the end segments are
 *     extended; an axis with one point is constant.
 *   eagle_cost_at: the interpolated cost, NaN for an invalid table.
 *   eagle_size_keep_level: level l (1-based) grows the verified set from
 *     (l-1)k to lk candidates per sequence; ratio = sum(gains[0..nb)) /
 *     (C(B, L, lk) - C(B, L, (l-1)k)), infinite when the cost does not grow;
 *     *keep = ratio >= threshold.  gains: HOST [nb], the level's per-sequence
 *     gains (eagle_tree_grow_gains).  A harness drafts level l + 1 only while
 *     level l is kept, and verifies m = k x (levels kept) candidates.
 *     ratio may be NULL.  Errors: EAGLE_ERR_NULL, EAGLE_ERR_SHAPE (invalid
 *     table or arguments). */
typedef struct {
  int nB, nL, nN;
  const double* B;
  const double* L;
  const double* N;
  const double* us; /* [nB][nL][nN] */
} eagle_cost_table_t;
EAGLE_API double eagle_cost_at(const eagle_cost_table_t* table, double B, double L, double N);
EAGLE_API eagle_status eagle_size_keep_level(const eagle_cost_table_t* table, double B, double L, int k, int level,
                                             const double* gains, int nb, double threshold, int* keep,
                                             double* ratio);
/* eagle_size_level_width: the width of one level when the harness widens or
 * deepens.  logv: HOST [nb][k], each sequence's k best candidates of the
 * level, log V in descending order (eagle_tree_grow_frontier_logv);
 * n_before: candidates per sequence chosen at the earlier levels.  The j-th
 * best of every sequence is taken together, in order: gain = sum over the
 * batch of its V = exp(log V), marginal cost C(B, L, n_before + j) -
 * C(B, L, n_before + j - 1); taken while gain > 0 and gain / cost >=
 * threshold (infinite when the cost does not grow); the first that fails ends
 * the level.  *width = the number taken (0: stop drafting).  ratios (HOST [k]
 * or NULL): each examined candidate's ratio, NaN past the first failure.
 * Errors: EAGLE_ERR_NULL, EAGLE_ERR_SHAPE. */
EAGLE_API eagle_status eagle_size_level_width(const eagle_cost_table_t* table, double B, double L, int n_before,
                                              const double* logv, int k, int nb, double threshold, int* width,
                                              double* ratios);

/* -------------------------------------------------------- static tree
 * EAGLE-1's fixed draft tree ("EAGLE" notes, "1. EAGLE pipeline / Draft
 * Model"): one template for every step; node i's token is the rank-r_i token
 * of its parent's draft row (by logit, ties to the lower token id).
 *   parents [n], ranks [n]: HOST arrays, the template.  parents[i] is the
 *     parent of node i+1: 0 for the root, else a node id <= i (a parent comes
 *     first).  ranks[i] in [0, EAGLE_MAX_TOPK); siblings have distinct ranks.
 *     n <= EAGLE_MAX_NODES.  The template is copied into the launch
 *     parameters: the arrays may be freed when the call returns.
 *   draft_logits [B][R][V] (dtype): row 0 is the root's; every node with a
 *     child owns a row, numbered 1, 2, ... in node order;
 *     R = eagle_static_tree_rows(parents, ranks, n).
 *   out: as for eagle_tree_build, with n nodes per sequence in template order;
 *     gid (optional) = the node's template index i; row_lse [B][R].
 * An invalid template returns EAGLE_ERR_SHAPE (eagle_static_tree_rows: -1),
 * a largest rank >= V EAGLE_ERR_LIMIT.  Two launches: the vocabulary sweep
 * (k = largest rank + 1) and the fill kernel.
 * Workspace: eagle_static_tree_workspace_bytes (0 for an invalid template). */
EAGLE_API int eagle_static_tree_rows(const int32_t* parents, const int32_t* ranks, int n);
EAGLE_API size_t eagle_static_tree_workspace_bytes(int B, int V, int dtype, const int32_t* parents,
                                                   const int32_t* ranks, int n);
EAGLE_API eagle_status eagle_static_tree_build(const void* draft_logits, int dtype, int B, int R, int V,
                                               const int32_t* parents, const int32_t* ranks, int n,
                                               const eagle_tree_t* out, void* workspace, size_t workspace_bytes,
                                               void* stream);

/* ------------------------------------------------- KV-cache compaction
 * After acceptance ("Технический анализ EAGLE-4", section "Деревья проверки
 * EAGLE-4 и утилита управления": the accepted continuation is kept, the
 * rejected KV-cache entries are freed): the keys and values that the
 * verification pass computed for the accepted nodes are appended to each
 * sequence's prefix cache in path order, the i-th accepted node (depth i+1)
 * at position prefix_len[b] + i, which is its position id; rejected nodes are
 * not copied (the bonus token has no key or value yet).
 *   k_tree, v_tree [B][n][Hkv][D] bf16 (the tree's keys and values)
 *   path [B][depth], accepted_len [B] (from eagle_accept; node ids 1..n)
 *   prefix_len [B] (clamped to [0, Lmax])
 *   k_cache, v_cache [B][Hkv][Lmax][D] bf16, updated in place
 *   new_prefix_len [B] int32 (must not be prefix_len itself): prefix_len plus
 *     the entries copied.  The copy ends at the first path entry that is not a
 *     node id in 1..n or whose position would reach Lmax.
 * Limits: n <= EAGLE_MAX_NODES, depth <= EAGLE_MAX_DEPTH, B <= 65535, D % 8 ==
 * 0, tensor pointers 16-byte aligned.  No workspace. */
EAGLE_API eagle_status eagle_kv_compact(const void* k_tree, const void* v_tree, const int32_t* path,
                                        const int32_t* accepted_len, const int32_t* prefix_len, void* k_cache,
                                        void* v_cache, int32_t* new_prefix_len, int B, int n, int Hkv, int D,
                                        int Lmax, int depth, void* stream);
/* The same into a paged cache (layout as for eagle_tree_attention_paged):
 * position p goes to offset p % page_size of page block_table[b][p /
 * page_size]; a sequence holds up to pages_per_seq * page_size keys, and the
 * copy also ends at a position whose page id lies outside [0, num_pages) (a
 * page not allocated yet). */
EAGLE_API eagle_status eagle_kv_compact_paged(const void* k_tree, const void* v_tree, const int32_t* path,
                                              const int32_t* accepted_len, const int32_t* prefix_len, void* k_pages,
                                              void* v_pages, int num_pages, int page_size,
                                              const int32_t* block_table, int pages_per_seq,
                                              int32_t* new_prefix_len, int B, int n, int Hkv, int D, int depth,
                                              void* stream);

/* ---------------------------------------------------------- one whole step
 * One verification step in its order: build (eagle_tree_build), mask and
 * position ids (fused into the build's expansion kernel), tree attention
 * (eagle_tree_attention) and acceptance (eagle_accept), on one stream.  The
 * outputs equal those of the four calls made one after another on the same
 * inputs (the same kernels and the same arithmetic).  The scratch is cleared
 * once at the start and each kernel may start while its predecessor drains
 * (programmatic dependent launch): two memsets, seven kernels, no host
 * synchronisation.
 *
 * Inputs (device pointers unless noted; layouts as in the calls above):
 *   draft_logits [B][R][V] (logits_dtype), R = 1 + (depth-1)*k
 *   q [B][n][Hq][D], k_cache / v_cache [B][Hkv][Lmax][D], k_tree / v_tree
 *   [B][n][Hkv][D] (bf16), prefix_len [B] int32, with n = min(m, pool size)
 *   (the tree size, also written to the HOST int *n_nodes when not NULL)
 *   target_logits [B][n+1][V] (logits_dtype, the target's rows of the tree)
 *   uniforms [B][2][n+1] float, or NULL for greedy acceptance
 *   sampling_rule: EAGLE_SAMPLE_WITH_REPLACEMENT or _WITHOUT_REPLACEMENT (as
 *   in eagle_accept_with_rule; ignored for greedy)
 * Outputs (caller-allocated, sized by n): the tree arrays (tree.gid may be
 *   NULL), mask [B][n][2] uint64, pos [B][n] int32, attn_out [B][n][Hq][D]
 *   bf16, accepted_len [B], path [B][depth], bonus [B] int32.
 * Limits: those of the four calls.  Workspace: eagle_verify_step_workspace_bytes
 * (256-byte aligned).  The attention's device status word (as for
 * eagle_tree_attention) is the int at byte offset
 * eagle_verify_step_attention_status_offset of the workspace after the step. */
typedef struct {
  const void* draft_logits;
  const void* target_logits;
  int logits_dtype;
  int B, V, depth, k, m;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* prefix_len;
  int Lmax;
  const void* k_tree;
  const void* v_tree;
  int Hq, Hkv, D, window;
  float scale;  /* <= 0 selects 1/sqrt(D) */
  const float* uniforms;
  int sampling_rule;  /* EAGLE_SAMPLE_WITH_REPLACEMENT or _WITHOUT_REPLACEMENT (sampled acceptance) */
  /* paged prefix cache (block_table != NULL): k_cache / v_cache are the page
   * pools and Lmax is unused, as in eagle_tree_attention_paged */
  const int32_t* block_table;
  int page_size, pages_per_seq, num_pages;
} eagle_step_in_t;

typedef struct {
  eagle_tree_t tree;
  uint64_t* mask;
  int32_t* pos;
  void* attn_out;
  int32_t* accepted_len;
  int32_t* path;
  int32_t* bonus;
} eagle_step_out_t;

/* Both return 0 for an invalid shape (the step itself then reports why). */
EAGLE_API size_t eagle_verify_step_workspace_bytes(const eagle_step_in_t* in);
EAGLE_API size_t eagle_verify_step_attention_status_offset(const eagle_step_in_t* in);
EAGLE_API eagle_status eagle_verify_step(const eagle_step_in_t* in, const eagle_step_out_t* out, int* n_nodes,
                                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------ diagnostics
 * Not a step of the method: a probe of the attention kernel's failure path.
 * With limit_ns > 0, every attention launch that follows (eagle_tree_attention,
 * _paged and the attention of eagle_verify_step) makes each softmax warp first
 * wait limit_ns on a barrier that nothing completes.  The wait gives up, and
 * the CTA takes the same path as any bounded wait that runs out: it sets its
 * abort flag, the other roles stop, every TMA copy and MMA in flight is drained,
 * TMEM is freed, and the workspace's status word reads 1 (the output is then
 * undefined).  limit_ns = 0 turns the probe off.  Process-wide; calls that race
 * with launches on other threads see either setting.  For tests of error
 * handling: nothing faults, traps or hangs. */
EAGLE_API void eagle_debug_attention_wait_probe(unsigned long long limit_ns);

/* ----------------------------------------------------- tree build, no workspace
 * Not a step of the method (the pages have no counterpart): the same build as
 * eagle_tree_build for callers that cannot allocate device memory when they
 * build a tree -- for example a serving loop whose memory pool is sealed after
 * warm-up, or a plugin interface that hands over only buffers and a stream.
 * Scratch comes from a fixed 2 MiB array inside the library (held on every GPU
 * that loads the library until the process exits); nothing is allocated.
 * Shapes whose eagle_tree_build_workspace_bytes exceeds 2 MiB return
 * EAGLE_ERR_LIMIT and launch nothing.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) and must come before any
 * stream capture on that device; the address is cached for the life of the
 * process, so a process that resets the device (cudaDeviceReset) must restart
 * before calling this again.  All calls share the array: calls whose work
 * overlaps on the GPU race and must be serialised by the caller. */
EAGLE_API eagle_status eagle_tree_build_noalloc(const void* draft_logits, int dtype, int B, int R, int V,
                                                int depth, int k, int m, const eagle_tree_t* out, int* n_nodes,
                                                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EAGLE_TREE_H */
