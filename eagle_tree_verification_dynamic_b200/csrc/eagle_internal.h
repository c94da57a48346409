// Host-side declarations shared by the translation units of libeagle_tree.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "eagle_tree.h"
#include "eagle_common.cuh"

namespace eagle {

// Streaming multiprocessors of the current device (cudaDevAttrMultiProcessorCount,
// read once per device); 148, a B200's count, when no device can be queried
// (host-only sizing on a machine without a GPU).  Grids and workspaces that
// scale with the SM count use it, so a workspace sized on one device is
// checked against the same count when the call launches.
int device_sm_count();

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with an optional programmatic-dependent-launch attribute (the kernel
// may start while its predecessor drains; it waits in griddep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), so
// later launches (including ones under stream capture) only launch.
cudaError_t ensure_smem_limit(const void* kernel, size_t bytes);
inline int dtype_bytes(int dtype) { return dtype == EAGLE_F32 ? 4 : 2; }

// ---- row statistics (row_stats.cu)
struct ChunkPlan {
  int chunk_elems;
  int n_chunks;
};
// Final per-row outputs of the vocabulary sweep (any pointer may be null).
struct RowOut {
  int32_t* tok;  // [rows][k] top-k token ids, descending logit (-1 if the row has fewer)
  float* val;    // [rows][k] their logits
  double* lse;   // [rows] log-sum-exp
};
ChunkPlan plan_chunks(long long rows, int V, int elem_bytes);
// plan_rows > 0: cut rows into chunks as a sweep of plan_rows rows would (the
// chunking fixes the order of the log-sum-exp's fp64 partial sums).
size_t row_stats_ws_bytes(long long rows, int V, int elem_bytes, int k, long long plan_rows = 0);
// zero_tickets: clear the per-row tickets first (else the caller already has);
// pdl: chain the kernel to its predecessor with programmatic dependent launch.
cudaError_t launch_row_stats(const void* x, int dtype, long long rows, int V, int k, bool lse, const RowOut& out,
                             void* ws, cudaStream_t s, bool zero_tickets = true, bool pdl = false,
                             long long plan_rows = 0);
// CUDA error -> status, recording the error text for eagle_last_cuda_error.
eagle_status report_cuda(cudaError_t e);
// Byte range of the per-row tickets inside the row-sweep workspace.
void row_stats_tickets_span(long long rows, int V, int elem_bytes, int k, size_t* off, size_t* bytes);

// ---- tree build (tree_build.cu)
size_t tree_build_smem_bytes(int R, int k, int P);
size_t tree_build_ws_bytes(int B, int R, int V, int elem_bytes, int k);
// Optional fused tree mask: with mask != nullptr the expansion kernel also
// writes each node's ancestor-or-self bitmask and position id (what
// eagle_tree_mask computes).
struct MaskOut {
  const int32_t* prefix_len;  // [B] (required with pos)
  uint64_t* mask;             // [B][n][2]
  int32_t* pos;               // [B][n] (may be null)
};
cudaError_t launch_tree_build(const void* draft_logits, int dtype, int B, int R, int V, int depth, int k, int n,
                              const eagle_tree_t& out, void* ws, cudaStream_t s, const MaskOut* mo = nullptr,
                              bool zero_tickets = true, bool pdl = false);

// The expansion / rerank alone, from each row's top-k tokens and logits
// [B][R][k] and out.row_lse [B][R] (the build's second kernel).
// widths (host, depth entries, or null): keep the widths[l-1] best candidates
// of each level l instead of the n best over all levels (n = their sum).
cudaError_t launch_tree_expand(const int32_t* row_tok, const float* row_val, int B, int R, int depth, int k, int n,
                               const eagle_tree_t& out, const MaskOut* mo, bool pdl, cudaStream_t s,
                               const int* widths = nullptr);

// ---- tree mask (tree_mask.cu)
cudaError_t launch_tree_mask(const int32_t* parents, const int32_t* depth, const int32_t* prefix_len,
                             int B, int n, uint64_t* mask, int32_t* pos, cudaStream_t s);

// ---- attention (attention.cu: workspace plan; attention_tc.cu: kernels)
constexpr int kAttnRowsPerUnit = 128;  // query rows per unit (one MMA M)
constexpr int kAttnKeysPerTile = 64;
// Workspace of eagle_tree_attention, byte offsets from its (256-aligned) base.
struct AttnWorkspace {
  size_t status_off;      // int: the device status word (written by every launch)
  size_t cta_status_off;  // int [C]: per-CTA status of the main kernel
  size_t part_lse_off;    // float [C + U][128]: log-sum-exp of each partial
  size_t part_o_off;      // float [C + U][128][D]: normalised partial outputs
  size_t bytes;
};
int attention_row_groups(int n, int Hq, int Hkv);
// The wait probe's limit for the next attention launches (0: off); see
// eagle_debug_attention_wait_probe.
unsigned long long attention_wait_probe_ns();
int attention_ctas(int B, int n, int Hq, int Hkv, int Lmax, int window);  // C
AttnWorkspace attention_ws_layout(int B, int n, int Hq, int Hkv, int D, int Lmax, int window);
inline size_t attention_ws_bytes(int B, int n, int Hq, int Hkv, int D, int Lmax, int window) {
  return attention_ws_layout(B, n, Hq, Hkv, D, Lmax, window).bytes;
}
// A paged prefix cache: pools [num_pages][Hkv][page_size][D], block_table
// [B][pages_per_seq] page ids; page_size is 16, 32 or a multiple of 64.
struct PagedKV {
  const int32_t* block_table;
  int page_size, pages_per_seq, num_pages;
};
// pg == nullptr: dense caches [B][Hkv][Lmax][D]; else kc / vc are the pools
// and a sequence holds up to pages_per_seq * page_size keys (Lmax unused).
// early: every input except mask and pos was complete before the previous
// kernel on the stream started, so the K/V stream begins before that kernel
// ends (only the fused step, whose previous kernel is the expansion, sets it).
cudaError_t launch_tree_attention(const void* q, const void* kc, const void* vc, const int32_t* plen,
                                  int Lmax, const void* kt, const void* vt, const uint64_t* mask,
                                  const int32_t* pos, int B, int n, int Hq, int Hkv, int D, int window,
                                  float scale, void* out, void* ws, cudaStream_t s, const PagedKV* pg = nullptr,
                                  bool early = false);

// ---- KV-cache compaction after acceptance (kv_compact.cu)
cudaError_t launch_kv_compact(const void* k_tree, const void* v_tree, const int32_t* path, const int32_t* accepted_len,
                              const int32_t* prefix_len, void* k_cache, void* v_cache, int32_t* new_len, int B, int n,
                              int Hkv, int D, int Lmax, int depth, cudaStream_t s, const PagedKV* pg = nullptr);

// ---- accept (accept.cu)
size_t accept_ws_bytes(int B, int n, int V, int dtype);
int accept_max_vocab(int dtype);  // largest V the sampled walk supports
cudaError_t launch_accept(const void* tgt, int tdtype, const void* dft, int ddtype, const double* dlse,
                          int R, const int32_t* tokens, const int32_t* parents, const int32_t* draft_row,
                          const float* uniforms, int B, int n, int V, int depth, int32_t* accepted_len,
                          int32_t* path, int32_t* bonus, void* ws, cudaStream_t s, bool zero_tickets = true,
                          bool pdl = false, bool without_replacement = false);

}  // namespace eagle
