// EAGLE-2 dynamic tree grown one level at a time ("EAGLE" notes, EAGLE-2
// sections "Expansion of tree" and "Reranking Nodes"), for a draft model that
// produces the next level's distributions only once it knows the frontier.
//
//   begin   the root's draft row: its top-k children form level 1; all of them
//           are the level-1 frontier (slot = rank)
//   level   the k draft rows of the current frontier (row s = frontier slot s):
//           their top-k children form the next level's k^2 candidates,
//           log V = log V(parent) + log c(child); the k best (log V, then lower
//           candidate id) form the next frontier
//   finish  the expansion / rerank kernel of eagle_tree_build on the rows of
//           the levels grown: the m best candidates, numbered by ascending id
//   gains   per sequence, the sum of V = exp(log V) over the last level's k
//           best candidates: the expected number of tokens those candidates
//           add (EAGLE-4 write-up, harness: the gain in cumulative
//           probability that a level brings)
//   widths  (the harness widening or deepening) a level may be drafted from
//           the first w frontier slots only: the caller passes w rows per
//           sequence, the other slots count as rows of -inf (no children);
//           frontier_logv reads the last level's k best log V in rank order,
//           and finish_widths keeps the w_l best candidates of each level.
//
// The state keeps each row's top-k tokens and logits and its log-sum-exp in
// the layout the one-shot build uses, plus the frontier's log V, so the tree
// equals eagle_tree_build on the same rows bit for bit (the same kernels and
// the same fp64 arithmetic for log V).
#include "eagle_internal.h"

namespace eagle {

namespace {

struct GrowLayout {
  size_t row_tok, row_val, row_lse, front_lv, gain, lvl_tok, lvl_val, lvl_lse, row_ws, total;
};

GrowLayout grow_layout(int B, int V, int dtype, int depth, int k) {
  const size_t R = 1 + (size_t)(depth - 1) * k;
  const size_t lvl_rows = (size_t)B * k;  // the most rows one call sweeps
  GrowLayout g;
  size_t o = 0;
  g.row_tok = o;  o = align_up(o + sizeof(int32_t) * B * R * k, 256);
  g.row_val = o;  o = align_up(o + sizeof(float) * B * R * k, 256);
  g.row_lse = o;  o = align_up(o + sizeof(double) * B * R, 256);
  g.front_lv = o; o = align_up(o + sizeof(double) * B * k, 256);
  g.gain = o;     o = align_up(o + sizeof(double) * B, 256);
  g.lvl_tok = o;  o = align_up(o + sizeof(int32_t) * lvl_rows * k, 256);
  g.lvl_val = o;  o = align_up(o + sizeof(float) * lvl_rows * k, 256);
  g.lvl_lse = o;  o = align_up(o + sizeof(double) * lvl_rows, 256);
  // the level sweeps cut rows into chunks as the one-shot build's sweep of all B*R rows does
  g.row_ws = o;   o = align_up(o + row_stats_ws_bytes((long long)lvl_rows, V, dtype_bytes(dtype), k, (long long)B * R), 256);
  g.total = o;
  return g;
}

constexpr int kGrowThreads = 1024;

// One CTA per sequence: file the swept rows of this level into the row arrays,
// then pick the level's k best candidates (the next frontier) and their gain.
//   level 1: rows = {0}, candidates = the root's k children (gid = r)
//   level l: rows = 1 + (l-2)k + s, candidates gid = k + (l-2)k^2 + s k + r
__global__ void __launch_bounds__(kGrowThreads)
tree_grow_kernel(const int32_t* __restrict__ lvl_tok, const float* __restrict__ lvl_val,
                 const double* __restrict__ lvl_lse, int32_t* __restrict__ row_tok, float* __restrict__ row_val,
                 double* __restrict__ row_lse, double* __restrict__ front_lv, double* __restrict__ gain,
                 int32_t* __restrict__ front_tok, int32_t* __restrict__ front_par, int R, int k, int level,
                 int width) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double s_lv[32 * 32];
  __shared__ int s_tok[32 * 32];
  __shared__ uint64_t s_key[32 * 32];
  __shared__ double s_flv[32];
  __shared__ double s_best[32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int nrows = level == 1 ? 1 : k;      // the level's slots
  const int nin = level == 1 ? 1 : width;    // rows swept: the first nin slots; the rest have no children
  const int r0 = level == 1 ? 0 : 1 + (level - 2) * k;
  // 1. this level's rows into the per-sequence row arrays
  for (int e = tid; e < nrows * k; e += kGrowThreads) {
    const int rr = e / k, j = e - rr * k;
    const size_t src = ((size_t)b * nin + rr) * k + j;
    const size_t dst = ((size_t)b * R + r0 + rr) * k + j;
    row_tok[dst] = rr < nin ? lvl_tok[src] : -1;
    row_val[dst] = rr < nin ? lvl_val[src] : -INFINITY;
  }
  for (int rr = tid; rr < nrows; rr += kGrowThreads)
    row_lse[(size_t)b * R + r0 + rr] = rr < nin ? lvl_lse[(size_t)b * nin + rr] : -INFINITY;
  // 2. the level's candidates: log V = log V(parent) + (logit - lse), as the one-shot build forms it
  for (int s = tid; s < k; s += kGrowThreads) s_flv[s] = level == 1 ? 0.0 : front_lv[(size_t)b * k + s];
  __syncthreads();
  const int cnt = nrows * k;
  const int gid0 = level == 1 ? 0 : k + (level - 2) * k * k;
  for (int c = tid; c < cnt; c += kGrowThreads) {
    const int s = c / k;
    const size_t src = ((size_t)b * nin + s) * k + (c - s * k);
    const int tok = s < nin ? lvl_tok[src] : -1;
    const double lp = tok >= 0 ? (double)lvl_val[src] - lvl_lse[(size_t)b * nin + s] : -INFINITY;
    const double lv = level == 1 ? lp : s_flv[s] + lp;
    s_lv[c] = lv;
    s_tok[c] = tok;
    s_key[c] = cand_key(lv, gid0 + c);
  }
  __syncthreads();
  // 3. rank = number of larger keys; the k best become the next frontier
  for (int c = tid; c < cnt; c += kGrowThreads) {
    const uint64_t mine = s_key[c];
    int rank = 0;
    for (int o = 0; o < cnt; ++o) rank += s_key[o] > mine ? 1 : 0;
    if (rank < k) {
      s_best[rank] = s_lv[c];
      if (front_tok) front_tok[(size_t)b * k + rank] = s_tok[c];
      if (front_par) front_par[(size_t)b * k + rank] = level == 1 ? -1 : c / k;
    }
  }
  __syncthreads();
  // s_flv (the previous frontier) is read above; the new one replaces it only now
  for (int s = tid; s < k; s += kGrowThreads) front_lv[(size_t)b * k + s] = s_best[s];
  if (tid == 0) {
    double g = 0.0;  // in rank order
    for (int s = 0; s < k; ++s) g += exp(s_best[s]);
    gain[b] = g;
  }
}

eagle_status grow_check(int dtype, int B, int V, int depth, int k, void* state, size_t state_bytes) {
  if (dtype != EAGLE_F32 && dtype != EAGLE_BF16) return EAGLE_ERR_DTYPE;
  if (B <= 0 || V <= 0 || depth <= 0 || k <= 0) return EAGLE_ERR_SHAPE;
  if (depth > EAGLE_MAX_DEPTH || k > EAGLE_MAX_TOPK || k > V) return EAGLE_ERR_LIMIT;
  if ((long long)k + (long long)(depth - 1) * k * k > EAGLE_MAX_POOL) return EAGLE_ERR_LIMIT;
  if (!state || state_bytes < grow_layout(B, V, dtype, depth, k).total || ((uintptr_t)state & 255u) != 0)
    return EAGLE_ERR_WORKSPACE;
  return EAGLE_OK;
}

// Sweep the level's rows (1 at the root, else `width` per sequence) and file
// them (and pick the frontier).
cudaError_t grow_step(const void* logits, int dtype, int B, int V, int depth, int k, int level, int width,
                      void* state, int32_t* ftok, int32_t* fpar, cudaStream_t s) {
  const GrowLayout g = grow_layout(B, V, dtype, depth, k);
  char* st = static_cast<char*>(state);
  const int nrows = level == 1 ? 1 : width;
  RowOut ro;
  ro.tok = reinterpret_cast<int32_t*>(st + g.lvl_tok);
  ro.val = reinterpret_cast<float*>(st + g.lvl_val);
  ro.lse = reinterpret_cast<double*>(st + g.lvl_lse);
  const int R = 1 + (depth - 1) * k;
  cudaError_t e = launch_row_stats(logits, dtype, (long long)B * nrows, V, k, true, ro, st + g.row_ws, s, true, false,
                                   (long long)B * R);
  if (e != cudaSuccess) return e;
  return launch_kernel(tree_grow_kernel, dim3(B), dim3(kGrowThreads), 0, s, true, ro.tok, ro.val,
                       (const double*)ro.lse, reinterpret_cast<int32_t*>(st + g.row_tok),
                       reinterpret_cast<float*>(st + g.row_val), reinterpret_cast<double*>(st + g.row_lse),
                       reinterpret_cast<double*>(st + g.front_lv), reinterpret_cast<double*>(st + g.gain), ftok,
                       fpar, R, k, level, width);
}

eagle_status cuda_st(cudaError_t e) { return report_cuda(e); }

}  // namespace

}  // namespace eagle

using namespace eagle;

extern "C" {

size_t eagle_tree_grow_state_bytes(int B, int V, int dtype, int depth, int k) {
  if (B <= 0 || V <= 0 || depth <= 0 || k <= 0 || (dtype != EAGLE_F32 && dtype != EAGLE_BF16)) return 0;
  return grow_layout(B, V, dtype, depth, k).total;
}

EAGLE_API eagle_status eagle_tree_grow_begin(const void* root_logits, int dtype, int B, int V, int depth, int k,
                                             void* state, size_t state_bytes, int32_t* frontier_tokens,
                                             int32_t* frontier_parents, void* stream) {
  if (!root_logits) return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  return cuda_st(grow_step(root_logits, dtype, B, V, depth, k, 1, 1, state, frontier_tokens, frontier_parents,
                           static_cast<cudaStream_t>(stream)));
}

EAGLE_API eagle_status eagle_tree_grow_level(const void* level_logits, int dtype, int B, int V, int depth, int k,
                                             int level, void* state, size_t state_bytes, int32_t* frontier_tokens,
                                             int32_t* frontier_parents, void* stream) {
  if (!level_logits) return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  if (level < 2 || level > depth) return EAGLE_ERR_SHAPE;
  return cuda_st(grow_step(level_logits, dtype, B, V, depth, k, level, k, state, frontier_tokens, frontier_parents,
                           static_cast<cudaStream_t>(stream)));
}

EAGLE_API eagle_status eagle_tree_grow_level_width(const void* level_logits, int dtype, int B, int V, int depth,
                                                   int k, int level, int width, void* state, size_t state_bytes,
                                                   int32_t* frontier_tokens, int32_t* frontier_parents,
                                                   void* stream) {
  if (!level_logits) return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  if (level < 2 || level > depth || width < 1 || width > k) return EAGLE_ERR_SHAPE;
  return cuda_st(grow_step(level_logits, dtype, B, V, depth, k, level, width, state, frontier_tokens,
                           frontier_parents, static_cast<cudaStream_t>(stream)));
}

EAGLE_API eagle_status eagle_tree_grow_frontier_logv(int dtype, int B, int V, int depth, int k, void* state,
                                                     size_t state_bytes, double* logv, void* stream) {
  if (!logv) return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  const GrowLayout g = grow_layout(B, V, dtype, depth, k);
  return cuda_st(cudaMemcpyAsync(logv, static_cast<char*>(state) + g.front_lv, sizeof(double) * B * k,
                                 cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
}

EAGLE_API eagle_status eagle_tree_grow_gains(int dtype, int B, int V, int depth, int k, void* state,
                                             size_t state_bytes, double* gains, void* stream) {
  if (!gains) return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  const GrowLayout g = grow_layout(B, V, dtype, depth, k);
  return cuda_st(cudaMemcpyAsync(gains, static_cast<char*>(state) + g.gain, sizeof(double) * B,
                                 cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
}

EAGLE_API eagle_status eagle_tree_grow_finish(int dtype, int B, int V, int depth, int k, int levels, int m,
                                              void* state, size_t state_bytes, const eagle_tree_t* out,
                                              int* n_nodes, void* stream) {
  if (!out || !out->tokens || !out->parents || !out->depth || !out->logV || !out->draft_row || !out->row_lse)
    return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  if (m <= 0 || levels < 1 || levels > depth) return EAGLE_ERR_SHAPE;
  if (m > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  const long long P = (long long)k + (long long)(levels - 1) * k * k;
  const int n = (int)(m < P ? m : P);
  if (n_nodes) *n_nodes = n;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const GrowLayout g = grow_layout(B, V, dtype, depth, k);
  char* stp = static_cast<char*>(state);
  const int R = 1 + (depth - 1) * k;
  // the expansion reads each row's log-sum-exp from the tree's row_lse
  cudaError_t e = cudaMemcpyAsync(out->row_lse, stp + g.row_lse, sizeof(double) * B * R, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_st(e);
  return cuda_st(launch_tree_expand(reinterpret_cast<const int32_t*>(stp + g.row_tok),
                                    reinterpret_cast<const float*>(stp + g.row_val), B, R, levels, k, n, *out,
                                    nullptr, false, s));
}

EAGLE_API eagle_status eagle_tree_grow_finish_widths(int dtype, int B, int V, int depth, int k, int levels,
                                                     const int* widths, void* state, size_t state_bytes,
                                                     const eagle_tree_t* out, int* n_nodes, void* stream) {
  if (!widths || !out || !out->tokens || !out->parents || !out->depth || !out->logV || !out->draft_row ||
      !out->row_lse)
    return EAGLE_ERR_NULL;
  const eagle_status st = grow_check(dtype, B, V, depth, k, state, state_bytes);
  if (st != EAGLE_OK) return st;
  if (levels < 1 || levels > depth) return EAGLE_ERR_SHAPE;
  int n = 0;
  for (int l = 0; l < levels; ++l) {
    // level 1 has k candidates; a deeper level's come from the w_{l-1} nodes chosen above it
    const int avail = l == 0 ? k : widths[l - 1] * k;
    if (widths[l] < 1 || widths[l] > k || widths[l] > avail) return EAGLE_ERR_SHAPE;
    n += widths[l];
  }
  if (n > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  if (n_nodes) *n_nodes = n;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const GrowLayout g = grow_layout(B, V, dtype, depth, k);
  char* stp = static_cast<char*>(state);
  const int R = 1 + (depth - 1) * k;
  cudaError_t e = cudaMemcpyAsync(out->row_lse, stp + g.row_lse, sizeof(double) * B * R, cudaMemcpyDeviceToDevice, s);
  if (e != cudaSuccess) return cuda_st(e);
  return cuda_st(launch_tree_expand(reinterpret_cast<const int32_t*>(stp + g.row_tok),
                                    reinterpret_cast<const float*>(stp + g.row_val), B, R, levels, k, n, *out,
                                    nullptr, false, s, widths));
}

}  // extern "C"
