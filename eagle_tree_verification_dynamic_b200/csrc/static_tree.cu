// EAGLE-1 static draft tree ("EAGLE" notes, "1. EAGLE pipeline / Draft Model"):
// one fixed template, the same at every step, whose node i takes the rank-r_i
// token of its parent's draft row (tokens ordered by logit, ties to the lower
// id).  Rows belong to the nodes that have children, in node order.
//
// The template is checked on the host and travels by value in the kernel's
// parameters (about 700 bytes), so the only memory a step reads is the draft
// rows: the vocabulary sweep (row_stats.cu) takes each row's top-k (k = the
// largest rank + 1) and log-sum-exp, then one small CTA per sequence reads its
// nodes' tokens out of that and forms log V level by level.
#include "eagle_internal.h"

namespace eagle {

namespace {

struct StaticPlan {
  uint8_t parent[EAGLE_MAX_NODES];   // 0 = root, else the parent's node id (< own id)
  uint8_t rank[EAGLE_MAX_NODES];     // sibling rank: index into the parent row's top-k
  uint8_t depth[EAGLE_MAX_NODES];
  int16_t row[EAGLE_MAX_NODES + 1];  // draft row of node j (j = 0: the root), -1 without children
  int n, R, k, max_depth;
};

constexpr int kStaticThreads = EAGLE_MAX_NODES;

// Checks the template and derives depths and rows; false if it is invalid.
bool make_plan(const int32_t* parents, const int32_t* ranks, int n, StaticPlan* p) {
  if (!parents || !ranks || n <= 0 || n > EAGLE_MAX_NODES) return false;
  bool has_child[EAGLE_MAX_NODES + 1] = {};
  uint32_t used[EAGLE_MAX_NODES + 1] = {};  // sibling ranks taken under each parent
  int k = 0, max_depth = 0;
  for (int i = 0; i < n; ++i) {
    const int par = parents[i], r = ranks[i];
    if (par < 0 || par > i) return false;  // a parent precedes its child (node ids are 1-based)
    if (r < 0 || r >= EAGLE_MAX_TOPK) return false;
    if (used[par] & (1u << r)) return false;  // two siblings with one rank would share a token
    used[par] |= 1u << r;
    has_child[par] = true;
    p->parent[i] = (uint8_t)par;
    p->rank[i] = (uint8_t)r;
    const int d = par == 0 ? 1 : p->depth[par - 1] + 1;
    p->depth[i] = (uint8_t)d;
    if (d > max_depth) max_depth = d;
    if (r + 1 > k) k = r + 1;
  }
  int R = 0;
  for (int j = 0; j <= n; ++j) p->row[j] = has_child[j] || j == 0 ? (int16_t)R++ : (int16_t)-1;
  p->n = n;
  p->R = R;
  p->k = k;
  p->max_depth = max_depth;
  return true;
}

__global__ void __launch_bounds__(kStaticThreads)
static_tree_kernel(const int32_t* __restrict__ row_tok, const float* __restrict__ row_val,
                   const double* __restrict__ row_lse, const __grid_constant__ StaticPlan plan, eagle_tree_t out) {
  griddep_wait();  // the rows' top-k come from the sweep before
  griddep_launch_dependents();
  __shared__ double lv[EAGLE_MAX_NODES];
  const int b = blockIdx.x, i = threadIdx.x;
  const int n = plan.n, R = plan.R, k = plan.k;
  int tok = -1, par = 0;
  double lp = 0.0;
  if (i < n) {
    par = plan.parent[i];
    const int row = plan.row[par];
    const size_t e = ((size_t)b * R + row) * k + plan.rank[i];
    tok = row_tok[e];
    lp = tok >= 0 ? (double)row_val[e] - row_lse[(size_t)b * R + row] : -INFINITY;
  }
  // log V = log V(parent) + log-confidence, one level per pass (a parent is one level up)
  for (int d = 1; d <= plan.max_depth; ++d) {
    if (i < n && plan.depth[i] == d) lv[i] = par == 0 ? lp : lv[par - 1] + lp;
    __syncthreads();
  }
  if (i < n) {
    const size_t o = (size_t)b * n + i;
    out.tokens[o] = tok;
    out.parents[o] = par;
    out.depth[o] = plan.depth[i];
    out.logV[o] = (float)lv[i];
    if (out.gid) out.gid[o] = i;
  }
  for (int j = i; j <= n; j += kStaticThreads) out.draft_row[(size_t)b * (n + 1) + j] = plan.row[j];
}

struct StaticWs {
  size_t tok, val, total;
};

StaticWs static_ws(int B, int R, int V, int dtype, int k) {
  StaticWs w;
  const size_t rows = (size_t)B * R;
  size_t o = align_up(row_stats_ws_bytes((long long)rows, V, dtype_bytes(dtype), k), 256);
  w.tok = o;
  o = align_up(o + sizeof(int32_t) * rows * k, 256);
  w.val = o;
  o = align_up(o + sizeof(float) * rows * k, 256);
  w.total = o;
  return w;
}

}  // namespace

}  // namespace eagle

using namespace eagle;

extern "C" {

EAGLE_API int eagle_static_tree_rows(const int32_t* parents, const int32_t* ranks, int n) {
  StaticPlan p;
  return make_plan(parents, ranks, n, &p) ? p.R : -1;
}

EAGLE_API size_t eagle_static_tree_workspace_bytes(int B, int V, int dtype, const int32_t* parents,
                                                   const int32_t* ranks, int n) {
  StaticPlan p;
  if (B <= 0 || V <= 0 || (dtype != EAGLE_F32 && dtype != EAGLE_BF16) || !make_plan(parents, ranks, n, &p)) return 0;
  return static_ws(B, p.R, V, dtype, p.k).total;
}

EAGLE_API eagle_status eagle_static_tree_build(const void* draft_logits, int dtype, int B, int R, int V,
                                               const int32_t* parents, const int32_t* ranks, int n,
                                               const eagle_tree_t* out, void* workspace, size_t workspace_bytes,
                                               void* stream) {
  if (!draft_logits || !parents || !ranks || !out || !out->tokens || !out->parents || !out->depth || !out->logV ||
      !out->draft_row || !out->row_lse)
    return EAGLE_ERR_NULL;
  if (dtype != EAGLE_F32 && dtype != EAGLE_BF16) return EAGLE_ERR_DTYPE;
  if (B <= 0 || V <= 0 || B > 65535) return EAGLE_ERR_SHAPE;
  if (n <= 0 || n > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  StaticPlan plan;
  if (!make_plan(parents, ranks, n, &plan)) return EAGLE_ERR_SHAPE;
  if (R != plan.R) return EAGLE_ERR_SHAPE;
  if (plan.k > V) return EAGLE_ERR_LIMIT;
  if ((long long)B * R > 0x7fffffffLL) return EAGLE_ERR_SHAPE;
  const StaticWs w = static_ws(B, R, V, dtype, plan.k);
  if (!workspace || workspace_bytes < w.total || ((uintptr_t)workspace & 255u) != 0) return EAGLE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  RowOut ro;
  ro.tok = reinterpret_cast<int32_t*>(ws + w.tok);
  ro.val = reinterpret_cast<float*>(ws + w.val);
  ro.lse = out->row_lse;  // [B][R], the tree's own row_lse
  cudaError_t e = launch_row_stats(draft_logits, dtype, (long long)B * R, V, plan.k, true, ro, ws, s);
  if (e != cudaSuccess) return report_cuda(e);
  return report_cuda(launch_kernel(static_tree_kernel, dim3(B), dim3(kStaticThreads), 0, s, true,
                                   (const int32_t*)ro.tok, (const float*)ro.val, (const double*)ro.lse, plan, *out));
}

}  // extern "C"
