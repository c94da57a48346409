// C-ABI entry points of libeagle_tree: argument validation on the host, then
// kernel launches on the caller's stream.  Nothing here allocates memory or
// synchronises the host.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <map>

#include "eagle_internal.h"

using namespace eagle;

namespace eagle {
cudaError_t ensure_smem_limit(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(kernel, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

int device_sm_count() {
  constexpr int kMaxDev = 64;
  static int cached[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();  // clear the error a GPU-less host leaves behind
    return 148;
  }
  if (cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  cached[dev] = n;  // a racing writer stores the same value
  return n;
}
}  // namespace eagle

namespace {

thread_local char g_cuda_err[256] = "";
eagle_status cuda_status(cudaError_t e);

}  // namespace

eagle_status eagle::report_cuda(cudaError_t e) { return cuda_status(e); }

namespace {

eagle_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return EAGLE_OK;
  snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return EAGLE_ERR_CUDA;
}

bool valid_dtype(int d) { return d == EAGLE_F32 || d == EAGLE_BF16; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

eagle_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return EAGLE_OK;
  if (ws == nullptr || have < need || ((uintptr_t)ws & 255u) != 0) return EAGLE_ERR_WORKSPACE;
  return EAGLE_OK;
}

}  // namespace

extern "C" {

const char* eagle_status_string(int status) {
  switch (status) {
    case EAGLE_OK: return "ok";
    case EAGLE_ERR_NULL: return "null pointer";
    case EAGLE_ERR_SHAPE: return "invalid shape";
    case EAGLE_ERR_DTYPE: return "unsupported dtype";
    case EAGLE_ERR_LIMIT: return "size exceeds a library limit";
    case EAGLE_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case EAGLE_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case EAGLE_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* eagle_last_cuda_error(void) { return g_cuda_err; }

int eagle_version(void) { return 200; }  // 0.2.0: eagle_step_in_t gained the sampling rule and paged-cache fields

// ------------------------------------------------------------------ row stats
size_t eagle_row_stats_workspace_bytes(long long rows, int V, int dtype, int k) {
  if (rows <= 0 || V <= 0 || !valid_dtype(dtype) || k < 1) return 0;
  return row_stats_ws_bytes(rows, V, dtype_bytes(dtype), k);
}

eagle_status eagle_row_stats(const void* logits, int dtype, long long rows, int V, int k, int32_t* topk_token,
                             float* topk_logit, double* lse, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!logits) return EAGLE_ERR_NULL;
  if (!valid_dtype(dtype)) return EAGLE_ERR_DTYPE;
  if (rows <= 0 || V <= 0 || k < 1 || rows > 0x7fffffffLL) return EAGLE_ERR_SHAPE;
  if (k > EAGLE_MAX_TOPK || k > V) return EAGLE_ERR_LIMIT;
  eagle_status st = check_ws(workspace, workspace_bytes, row_stats_ws_bytes(rows, V, dtype_bytes(dtype), k));
  if (st != EAGLE_OK) return st;
  RowOut out;
  out.tok = topk_token;
  out.val = topk_logit;
  out.lse = lse;
  return cuda_status(launch_row_stats(logits, dtype, rows, V, k, lse != nullptr, out, workspace,
                                      static_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------------------------- tree build
size_t eagle_tree_build_workspace_bytes(int B, int R, int V, int dtype, int k) {
  if (B <= 0 || R <= 0 || V <= 0 || !valid_dtype(dtype) || k < 1) return 0;
  return tree_build_ws_bytes(B, R, V, dtype_bytes(dtype), k);
}

eagle_status eagle_tree_build(const void* draft_logits, int dtype, int B, int R, int V, int depth, int k,
                              int m, const eagle_tree_t* out, int* n_nodes, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!draft_logits || !out) return EAGLE_ERR_NULL;
  if (!out->tokens || !out->parents || !out->depth || !out->logV || !out->draft_row || !out->row_lse)
    return EAGLE_ERR_NULL;
  if (!valid_dtype(dtype)) return EAGLE_ERR_DTYPE;
  if (B <= 0 || V <= 0 || depth <= 0 || k <= 0 || m <= 0) return EAGLE_ERR_SHAPE;
  if (depth > EAGLE_MAX_DEPTH || k > EAGLE_MAX_TOPK || k > V || m > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  const long long P = (long long)k + (long long)(depth - 1) * k * k;
  if (P > EAGLE_MAX_POOL) return EAGLE_ERR_LIMIT;
  if (R != 1 + (depth - 1) * k) return EAGLE_ERR_SHAPE;
  eagle_status st = check_ws(workspace, workspace_bytes, tree_build_ws_bytes(B, R, V, dtype_bytes(dtype), k));
  if (st != EAGLE_OK) return st;
  const int n = (int)(m < P ? m : P);
  if (n_nodes) *n_nodes = n;
  return cuda_status(launch_tree_build(draft_logits, dtype, B, R, V, depth, k, n, *out, workspace,
                                       static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ tree mask
eagle_status eagle_tree_mask(const int32_t* parents, const int32_t* depth, const int32_t* prefix_len, int B,
                             int n, uint64_t* mask, int32_t* pos, void* stream) {
  if (!parents || !mask) return EAGLE_ERR_NULL;
  if (pos && (!depth || !prefix_len)) return EAGLE_ERR_NULL;
  if (B <= 0 || n <= 0) return EAGLE_ERR_SHAPE;
  if (n > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  return cuda_status(launch_tree_mask(parents, depth, prefix_len, B, n, mask, pos,
                                      static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------- tree attention
size_t eagle_tree_attention_workspace_bytes(int B, int n, int Hq, int Hkv, int D, int Lmax, int window) {
  if (B <= 0 || n <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax < 0) return 0;
  return attention_ws_bytes(B, n, Hq, Hkv, D, Lmax, window);
}

eagle_status eagle_tree_attention(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* prefix_len, int Lmax, const void* k_tree, const void* v_tree,
                                  const uint64_t* mask, const int32_t* pos, int B, int n, int Hq, int Hkv, int D,
                                  int window, float scale, void* out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (!q || !k_tree || !v_tree || !mask || !prefix_len || !out) return EAGLE_ERR_NULL;
  if (Lmax > 0 && (!k_cache || !v_cache)) return EAGLE_ERR_NULL;
  if (window > 0 && !pos) return EAGLE_ERR_NULL;
  if (B <= 0 || n <= 0 || Hq <= 0 || Hkv <= 0 || Lmax < 0 || window < 0) return EAGLE_ERR_SHAPE;
  if (Hq % Hkv != 0) return EAGLE_ERR_SHAPE;
  if (D != 64 && D != 128) return EAGLE_ERR_LIMIT;
  if (n > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  if (!aligned16(q) || !aligned16(k_tree) || !aligned16(v_tree) || !aligned16(out) ||
      (Lmax > 0 && (!aligned16(k_cache) || !aligned16(v_cache))))
    return EAGLE_ERR_ALIGN;
  eagle_status st = check_ws(workspace, workspace_bytes, attention_ws_bytes(B, n, Hq, Hkv, D, Lmax, window));
  if (st != EAGLE_OK) return st;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)D);
  return cuda_status(launch_tree_attention(q, k_cache, v_cache, prefix_len, Lmax, k_tree, v_tree, mask, pos, B, n,
                                           Hq, Hkv, D, window, scale, out, workspace,
                                           static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// A paged prefix cache's description: page_size 16, 32 or a multiple of 64;
// every row index of the pools and every capacity fits in an int.
eagle_status check_paged(const int32_t* block_table, int page_size, int pages_per_seq, int num_pages, int Hkv) {
  if (!block_table) return EAGLE_ERR_NULL;
  if (page_size <= 0 || pages_per_seq <= 0 || num_pages <= 0 || Hkv <= 0) return EAGLE_ERR_SHAPE;
  if (!(page_size == 16 || page_size == 32 || page_size % 64 == 0)) return EAGLE_ERR_SHAPE;
  if ((long long)num_pages * Hkv * page_size > 0x7fffffffLL) return EAGLE_ERR_LIMIT;
  if ((long long)pages_per_seq * page_size > (1LL << 30)) return EAGLE_ERR_LIMIT;
  return EAGLE_OK;
}

}  // namespace

extern "C" {

eagle_status eagle_tree_attention_paged(const void* q, const void* k_pages, const void* v_pages, int num_pages,
                                        int page_size, const int32_t* block_table, int pages_per_seq,
                                        const int32_t* prefix_len, const void* k_tree, const void* v_tree,
                                        const uint64_t* mask, const int32_t* pos, int B, int n, int Hq, int Hkv,
                                        int D, int window, float scale, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (!q || !k_pages || !v_pages || !k_tree || !v_tree || !mask || !prefix_len || !out) return EAGLE_ERR_NULL;
  if (window > 0 && !pos) return EAGLE_ERR_NULL;
  eagle_status st = check_paged(block_table, page_size, pages_per_seq, num_pages, Hkv);
  if (st != EAGLE_OK) return st;
  if (B <= 0 || n <= 0 || Hq <= 0 || window < 0 || Hq % Hkv != 0) return EAGLE_ERR_SHAPE;
  if (D != 64 && D != 128) return EAGLE_ERR_LIMIT;
  if (n > EAGLE_MAX_NODES) return EAGLE_ERR_LIMIT;
  if (!aligned16(q) || !aligned16(k_tree) || !aligned16(v_tree) || !aligned16(out) || !aligned16(k_pages) ||
      !aligned16(v_pages))
    return EAGLE_ERR_ALIGN;
  const int cap = pages_per_seq * page_size;
  st = check_ws(workspace, workspace_bytes, attention_ws_bytes(B, n, Hq, Hkv, D, cap, window));
  if (st != EAGLE_OK) return st;
  if (!(scale > 0.f)) scale = 1.0f / sqrtf((float)D);
  const PagedKV pg = {block_table, page_size, pages_per_seq, num_pages};
  return cuda_status(launch_tree_attention(q, k_pages, v_pages, prefix_len, cap, k_tree, v_tree, mask, pos, B, n,
                                           Hq, Hkv, D, window, scale, out, workspace,
                                           static_cast<cudaStream_t>(stream), &pg));
}

eagle_status eagle_kv_compact_paged(const void* k_tree, const void* v_tree, const int32_t* path,
                                    const int32_t* accepted_len, const int32_t* prefix_len, void* k_pages,
                                    void* v_pages, int num_pages, int page_size, const int32_t* block_table,
                                    int pages_per_seq, int32_t* new_prefix_len, int B, int n, int Hkv, int D,
                                    int depth, void* stream) {
  if (!k_tree || !v_tree || !path || !accepted_len || !prefix_len || !k_pages || !v_pages || !new_prefix_len)
    return EAGLE_ERR_NULL;
  eagle_status st = check_paged(block_table, page_size, pages_per_seq, num_pages, Hkv);
  if (st != EAGLE_OK) return st;
  if (B <= 0 || n <= 0 || D <= 0 || depth <= 0) return EAGLE_ERR_SHAPE;
  if (D % 8 != 0 || new_prefix_len == prefix_len) return EAGLE_ERR_SHAPE;
  if (n > EAGLE_MAX_NODES || depth > EAGLE_MAX_DEPTH || B > 65535) return EAGLE_ERR_LIMIT;
  if (!aligned16(k_tree) || !aligned16(v_tree) || !aligned16(k_pages) || !aligned16(v_pages)) return EAGLE_ERR_ALIGN;
  const PagedKV pg = {block_table, page_size, pages_per_seq, num_pages};
  return cuda_status(launch_kv_compact(k_tree, v_tree, path, accepted_len, prefix_len, k_pages, v_pages,
                                       new_prefix_len, B, n, Hkv, D, pages_per_seq * page_size, depth,
                                       static_cast<cudaStream_t>(stream), &pg));
}

// --------------------------------------------------------------------- accept
size_t eagle_accept_workspace_bytes(int B, int n, int V, int target_dtype) {
  if (B <= 0 || n <= 0 || V <= 0 || !valid_dtype(target_dtype)) return 0;
  return accept_ws_bytes(B, n, V, target_dtype);
}

eagle_status eagle_accept(const void* target_logits, int target_dtype, const void* draft_logits, int draft_dtype,
                          const double* draft_lse, int R, const int32_t* tokens, const int32_t* parents,
                          const int32_t* draft_row, const float* uniforms, int B, int n, int V, int depth,
                          int32_t* accepted_len, int32_t* path, int32_t* bonus, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return eagle_accept_with_rule(target_logits, target_dtype, draft_logits, draft_dtype, draft_lse, R, tokens, parents,
                                draft_row, uniforms, EAGLE_SAMPLE_WITH_REPLACEMENT, B, n, V, depth, accepted_len,
                                path, bonus, workspace, workspace_bytes, stream);
}

eagle_status eagle_accept_with_rule(const void* target_logits, int target_dtype, const void* draft_logits,
                                    int draft_dtype, const double* draft_lse, int R, const int32_t* tokens,
                                    const int32_t* parents, const int32_t* draft_row, const float* uniforms,
                                    int sampling_rule, int B, int n, int V, int depth, int32_t* accepted_len,
                                    int32_t* path, int32_t* bonus, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (sampling_rule != EAGLE_SAMPLE_WITH_REPLACEMENT && sampling_rule != EAGLE_SAMPLE_WITHOUT_REPLACEMENT)
    return EAGLE_ERR_SHAPE;
  if (!target_logits || !tokens || !parents || !draft_row || !accepted_len || !path || !bonus)
    return EAGLE_ERR_NULL;
  if (!valid_dtype(target_dtype)) return EAGLE_ERR_DTYPE;
  const bool stoch = uniforms != nullptr;
  if (stoch) {
    if (!draft_logits || !draft_lse) return EAGLE_ERR_NULL;
    if (!valid_dtype(draft_dtype)) return EAGLE_ERR_DTYPE;
    if (draft_dtype != target_dtype) return EAGLE_ERR_DTYPE;
    if (R <= 0) return EAGLE_ERR_SHAPE;
    if (V > accept_max_vocab(target_dtype)) return EAGLE_ERR_LIMIT;
  }
  if (B <= 0 || n <= 0 || V <= 0 || depth <= 0) return EAGLE_ERR_SHAPE;
  if (n > EAGLE_MAX_NODES || depth > EAGLE_MAX_DEPTH) return EAGLE_ERR_LIMIT;
  if ((long long)B * (n + 1) > 0x7fffffffLL) return EAGLE_ERR_SHAPE;
  eagle_status st = check_ws(workspace, workspace_bytes, accept_ws_bytes(B, n, V, target_dtype));
  if (st != EAGLE_OK) return st;
  return cuda_status(launch_accept(target_logits, target_dtype, draft_logits, draft_dtype, draft_lse, R, tokens,
                                   parents, draft_row, uniforms, B, n, V, depth, accepted_len, path, bonus,
                                   workspace, static_cast<cudaStream_t>(stream), true, false,
                                   sampling_rule == EAGLE_SAMPLE_WITHOUT_REPLACEMENT));
}

// ------------------------------------------------------ KV-cache compaction
eagle_status eagle_kv_compact(const void* k_tree, const void* v_tree, const int32_t* path,
                              const int32_t* accepted_len, const int32_t* prefix_len, void* k_cache, void* v_cache,
                              int32_t* new_prefix_len, int B, int n, int Hkv, int D, int Lmax, int depth,
                              void* stream) {
  if (!k_tree || !v_tree || !path || !accepted_len || !prefix_len || !k_cache || !v_cache || !new_prefix_len)
    return EAGLE_ERR_NULL;
  if (B <= 0 || n <= 0 || Hkv <= 0 || D <= 0 || Lmax <= 0 || depth <= 0) return EAGLE_ERR_SHAPE;
  if (D % 8 != 0 || new_prefix_len == prefix_len) return EAGLE_ERR_SHAPE;
  if (n > EAGLE_MAX_NODES || depth > EAGLE_MAX_DEPTH || B > 65535) return EAGLE_ERR_LIMIT;
  if (!aligned16(k_tree) || !aligned16(v_tree) || !aligned16(k_cache) || !aligned16(v_cache)) return EAGLE_ERR_ALIGN;
  return cuda_status(launch_kv_compact(k_tree, v_tree, path, accepted_len, prefix_len, k_cache, v_cache,
                                       new_prefix_len, B, n, Hkv, D, Lmax, depth, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ whole step
}  // extern "C"

namespace {

struct StepLayout {
  int R, n;
  size_t build_off, attn_off, acc_off, total;
};

// Shapes of the step; false for sizes that no call accepts (the step reports which).
bool step_layout(const eagle_step_in_t* in, StepLayout* L) {
  if (!in || in->B <= 0 || in->V <= 0 || in->depth <= 0 || in->k <= 0 || in->m <= 0 || !valid_dtype(in->logits_dtype))
    return false;
  if (in->depth > EAGLE_MAX_DEPTH || in->k > EAGLE_MAX_TOPK || in->m > EAGLE_MAX_NODES) return false;
  const long long P = (long long)in->k + (long long)(in->depth - 1) * in->k * in->k;
  if (P > EAGLE_MAX_POOL) return false;
  if (in->Hq <= 0 || in->Hkv <= 0 || in->D <= 0 || in->Lmax < 0 || in->window < 0) return false;
  if (in->block_table && (in->page_size <= 0 || in->pages_per_seq <= 0 ||
                          (long long)in->pages_per_seq * in->page_size > (1LL << 30)))
    return false;
  // a paged cache holds up to pages_per_seq * page_size keys per sequence
  const int cap = in->block_table ? in->pages_per_seq * in->page_size : in->Lmax;
  L->R = 1 + (in->depth - 1) * in->k;
  L->n = (int)(in->m < P ? in->m : P);
  const int eb = dtype_bytes(in->logits_dtype);
  L->build_off = 0;
  L->attn_off = align_up(tree_build_ws_bytes(in->B, L->R, in->V, eb, in->k), 256);
  L->acc_off = align_up(L->attn_off + attention_ws_bytes(in->B, L->n, in->Hq, in->Hkv, in->D, cap, in->window), 256);
  L->total = align_up(L->acc_off + accept_ws_bytes(in->B, L->n, in->V, in->logits_dtype), 256);
  return true;
}

}  // namespace

extern "C" {

size_t eagle_verify_step_workspace_bytes(const eagle_step_in_t* in) {
  StepLayout L;
  return step_layout(in, &L) ? L.total : 0;
}

size_t eagle_verify_step_attention_status_offset(const eagle_step_in_t* in) {
  StepLayout L;
  return step_layout(in, &L) ? L.attn_off : 0;
}

eagle_status eagle_verify_step(const eagle_step_in_t* in, const eagle_step_out_t* out, int* n_nodes,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!in || !out) return EAGLE_ERR_NULL;
  // --- the checks of the four calls, before anything is launched
  const eagle_tree_t& t = out->tree;
  if (!in->draft_logits || !in->target_logits || !in->q || !in->k_tree || !in->v_tree || !in->prefix_len)
    return EAGLE_ERR_NULL;
  if (!t.tokens || !t.parents || !t.depth || !t.logV || !t.draft_row || !t.row_lse) return EAGLE_ERR_NULL;
  if (!out->mask || !out->pos || !out->attn_out || !out->accepted_len || !out->path || !out->bonus)
    return EAGLE_ERR_NULL;
  const bool paged = in->block_table != nullptr;
  if ((paged || in->Lmax > 0) && (!in->k_cache || !in->v_cache)) return EAGLE_ERR_NULL;
  if (paged) {
    const eagle_status ps = check_paged(in->block_table, in->page_size, in->pages_per_seq, in->num_pages, in->Hkv);
    if (ps != EAGLE_OK) return ps;
  }
  if (!valid_dtype(in->logits_dtype)) return EAGLE_ERR_DTYPE;
  if (in->B <= 0 || in->V <= 0 || in->depth <= 0 || in->k <= 0 || in->m <= 0) return EAGLE_ERR_SHAPE;
  if (in->Hq <= 0 || in->Hkv <= 0 || in->Lmax < 0 || in->window < 0 || in->Hq % in->Hkv != 0) return EAGLE_ERR_SHAPE;
  if (in->depth > EAGLE_MAX_DEPTH || in->k > EAGLE_MAX_TOPK || in->k > in->V || in->m > EAGLE_MAX_NODES)
    return EAGLE_ERR_LIMIT;
  if (in->D != 64 && in->D != 128) return EAGLE_ERR_LIMIT;
  StepLayout L;
  if (!step_layout(in, &L)) return EAGLE_ERR_LIMIT;
  if ((long long)in->B * (L.n + 1) > 0x7fffffffLL) return EAGLE_ERR_SHAPE;
  if (in->uniforms && in->V > accept_max_vocab(in->logits_dtype)) return EAGLE_ERR_LIMIT;
  if (in->sampling_rule != EAGLE_SAMPLE_WITH_REPLACEMENT && in->sampling_rule != EAGLE_SAMPLE_WITHOUT_REPLACEMENT)
    return EAGLE_ERR_SHAPE;
  if (!aligned16(in->q) || !aligned16(in->k_tree) || !aligned16(in->v_tree) || !aligned16(out->attn_out) ||
      ((paged || in->Lmax > 0) && (!aligned16(in->k_cache) || !aligned16(in->v_cache))))
    return EAGLE_ERR_ALIGN;
  eagle_status st = check_ws(workspace, workspace_bytes, L.total);
  if (st != EAGLE_OK) return st;
  if (n_nodes) *n_nodes = L.n;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  const int eb = dtype_bytes(in->logits_dtype);
  const int n = L.n;
  // --- clear both row sweeps' tickets up front; every kernel then chains to
  // its predecessor with programmatic dependent launch
  size_t off = 0, bytes = 0;
  row_stats_tickets_span((long long)in->B * L.R, in->V, eb, in->k, &off, &bytes);
  cudaError_t e = cudaMemsetAsync(ws + L.build_off + off, 0, bytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  row_stats_tickets_span((long long)in->B * (n + 1), in->V, eb, 1, &off, &bytes);
  e = cudaMemsetAsync(ws + L.acc_off + off, 0, bytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  // --- build, with the mask and position ids written by the expansion
  const MaskOut mo = {in->prefix_len, out->mask, out->pos};
  e = launch_tree_build(in->draft_logits, in->logits_dtype, in->B, L.R, in->V, in->depth, in->k, n, t,
                        ws + L.build_off, s, &mo, false, true);
  if (e != cudaSuccess) return cuda_status(e);
  // --- tree attention
  const float scale = in->scale > 0.f ? in->scale : 1.0f / sqrtf((float)in->D);
  const PagedKV pg = {in->block_table, in->page_size, in->pages_per_seq, in->num_pages};
  e = launch_tree_attention(in->q, in->k_cache, in->v_cache, in->prefix_len, in->Lmax, in->k_tree, in->v_tree,
                            out->mask, out->pos, in->B, n, in->Hq, in->Hkv, in->D, in->window, scale, out->attn_out,
                            ws + L.attn_off, s, paged ? &pg : nullptr, /*early=*/true);
  if (e != cudaSuccess) return cuda_status(e);
  // --- acceptance (the draft rows' log-sum-exps are the tree's row_lse)
  e = launch_accept(in->target_logits, in->logits_dtype, in->draft_logits, in->logits_dtype, t.row_lse, L.R,
                    t.tokens, t.parents, t.draft_row, in->uniforms, in->B, n, in->V, in->depth, out->accepted_len,
                    out->path, out->bonus, ws + L.acc_off, s, false, true,
                    in->sampling_rule == EAGLE_SAMPLE_WITHOUT_REPLACEMENT);
  return cuda_status(e);
}

}  // extern "C"
