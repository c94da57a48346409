// EAGLE-2 dynamic draft tree ("EAGLE" notes, EAGLE-2 sections "Expansion of
// tree" and "Reranking Nodes").  One CTA per sequence:
//   0. (before it, in parallel over all rows) the vocabulary sweep gives each
//      draft row's log-sum-exp and top-k;
//   1. lp = logit - lse turns the top-k logits into log-confidences;
//   2. level 1 = the root's k children; for each level, every candidate counts
//      the larger (log V desc, candidate id asc) keys of its level: that count
//      is its rank, which places it in the level's sorted list, and the first
//      k ranks form the frontier (slot = rank, which names the draft row of
//      the node); their k children each enter the next level with
//      log V = log V(parent) + lp (log of the product of confidences);
//   3. rerank: a candidate's rank among all P is its rank in its own level
//      plus, for every other level, the number of larger keys there (an 8-way
//      search in that level's sorted list); the n with rank < n are kept;
//   4. a prefix count renumbers the kept candidates 1..n by ascending id and
//      the tree arrays are written.
// log V is carried in fp64 so that the rounding of one path sum can only
// reorder candidates whose values agree to ~1e-15 relative.
#include "eagle_internal.h"

namespace eagle {

constexpr int kBuildThreads = 256;  // the largest expansion block

struct BuildSmem {
  double* row_lp;    // [R*k] log-confidence of each row's top-k children
  double* cand_lv;   // [P]   log V
  uint64_t* keys;    // [P]   ranking key of candidate g
  uint64_t* sorted;  // [P]   each level's keys in rank order, at the level's id range
  int* row_tok;      // [R*k]
  int* cand_tok;     // [P]
  int* cand_par;     // [P]   parent candidate id, -1 = root
  int* cand_row;     // [P]   draft row of an expanded candidate, -1 otherwise
  int* node_of;      // [P]   kept flag, then 1-based node id (0 = dropped)
  int* frontier;     // [32]
  int* warp_cnt;     // [NT / 32]
  int* node_par;     // [EAGLE_MAX_NODES] parent node id of node i+1 (mask fusion)
  int* node_dep;     // [EAGLE_MAX_NODES]
};


// Per-level widths of the cost-aware harness (on = 0: keep the best n overall).
struct LevelWidths {
  int w[EAGLE_MAX_DEPTH];
  int on;
};

// The number of keys of the descending list S[0, size) above x: an 8-way
// search (seven independent probes narrow the range eightfold per round,
// then at most eight keys are counted), so a list of 100 keys takes three
// rounds of shared-memory loads instead of a binary search's seven.
__device__ __forceinline__ int count_greater(const uint64_t* S, int size, uint64_t x) {
  int lo = 0, n = size;  // the count lies in [lo, lo + n]
  while (n > 8) {
    const int step = (n + 7) >> 3;
    int c = 0;  // S descends: the probes above x form a prefix
#pragma unroll
    for (int j = 1; j < 8; ++j) {
      const int q = step * j;
      if (q <= n && S[lo + q - 1] > x) ++c;
    }
    const int hi = (c < 7 && step * (c + 1) <= n) ? lo + step * (c + 1) - 1 : lo + n;
    lo += step * c;
    n = hi - lo;
  }
  int c = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < n && S[lo + j] > x) ++c;
  return lo + c;
}

// row_tok / row_val: each draft row's top-k tokens and logits (descending),
// row_lse: each row's log-sum-exp (also the tree's row_lse output).
template <int NT>
__global__ void __launch_bounds__(NT)
tree_expand_kernel(const int32_t* __restrict__ row_tok_g, const float* __restrict__ row_val_g, int R, int depth,
                   int k, int n, eagle_tree_t out, MaskOut mo, LevelWidths lw) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kk = k * k;
  const int P = k + (depth - 1) * kk;

  griddep_wait();  // the row statistics come from the previous kernel
  griddep_launch_dependents();
  BuildSmem sm;
  {
    unsigned char* p = smem_raw;
    sm.row_lp = reinterpret_cast<double*>(p);    p += sizeof(double) * R * k;
    sm.cand_lv = reinterpret_cast<double*>(p);   p += sizeof(double) * P;
    sm.keys = reinterpret_cast<uint64_t*>(p);    p += sizeof(uint64_t) * P;
    sm.sorted = reinterpret_cast<uint64_t*>(p);  p += sizeof(uint64_t) * P;
    sm.row_tok = reinterpret_cast<int*>(p);      p += sizeof(int) * R * k;
    sm.cand_tok = reinterpret_cast<int*>(p);     p += sizeof(int) * P;
    sm.cand_par = reinterpret_cast<int*>(p);     p += sizeof(int) * P;
    sm.cand_row = reinterpret_cast<int*>(p);     p += sizeof(int) * P;
    sm.node_of = reinterpret_cast<int*>(p);      p += sizeof(int) * P;
    sm.frontier = reinterpret_cast<int*>(p);     p += sizeof(int) * 32;
    sm.warp_cnt = reinterpret_cast<int*>(p);     p += sizeof(int) * (NT / 32);
    sm.node_par = reinterpret_cast<int*>(p);     p += sizeof(int) * EAGLE_MAX_NODES;
    sm.node_dep = reinterpret_cast<int*>(p);
  }

  // 1. each row's children and their log-confidence lp = logit - lse (fp64)
  for (int e = tid; e < R * k; e += NT) {
    const size_t g = (size_t)b * R * k + e;
    const int tok = row_tok_g[g];
    sm.row_tok[e] = tok;
    sm.row_lp[e] = tok >= 0 ? (double)row_val_g[g] - out.row_lse[(size_t)b * R + e / k] : -INFINITY;
  }
  __syncthreads();
  for (int c = tid; c < P; c += NT) {
    sm.cand_row[c] = -1;
    if (c < k) {  // level 1: the root's children
      sm.cand_lv[c] = sm.row_lp[c];
      sm.cand_tok[c] = sm.row_tok[c];
      sm.cand_par[c] = -1;
      sm.keys[c] = cand_key(sm.row_lp[c], c);
    }
  }
  __syncthreads();

  // 2. level by level: a candidate's rank = how many keys of its level are
  //    larger; it files the key into the level's sorted list, and the first k
  //    ranks form the frontier whose children make the next level
  for (int level = 1; level <= depth; ++level) {
    const int lo = level == 1 ? 0 : k + (level - 2) * kk;
    const int cnt = level == 1 ? k : kk;
    // tpc adjacent lanes share a candidate's count (a power of two, so a
    // group never straddles a warp); every lane runs the same iterations
    int tpc = 1;
    while (tpc < 8 && tpc * 2 * cnt <= NT) tpc *= 2;
    const int sub = tid & (tpc - 1);
    for (int base = 0; base < cnt * tpc; base += NT) {
      const int c = (base + tid) / tpc;
      const uint64_t mine = c < cnt ? sm.keys[lo + c] : ~0ull;
      // this lane's share [o0, o1) of the level, eight independent loads a step
      const int o0 = sub * cnt / tpc, o1 = (sub + 1) * cnt / tpc;
      const uint64_t* kp = sm.keys + lo;
      int rank = 0, o = o0;
      for (; o + 8 <= o1; o += 8) {
        uint64_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = kp[o + u];
#pragma unroll
        for (int u = 0; u < 8; ++u) rank += v[u] > mine ? 1 : 0;
      }
      for (; o < o1; ++o) rank += kp[o] > mine ? 1 : 0;
      for (int m = 1; m < tpc; m <<= 1) rank += __shfl_xor_sync(kFull, rank, m);
      if (c < cnt && sub == 0) {
        sm.sorted[lo + rank] = mine;
        if (level < depth && rank < k) {
          sm.frontier[rank] = lo + c;
          sm.cand_row[lo + c] = 1 + (level - 1) * k + rank;
        }
      }
    }
    __syncthreads();
    if (level == depth) break;
    const int lo2 = k + (level - 1) * kk;
    for (int idx = tid; idx < kk; idx += NT) {
      const int s = idx / k, r = idx - s * k;
      const int parent = sm.frontier[s];
      const int row = 1 + (level - 1) * k + s;
      const int g = lo2 + idx;
      const double lv = sm.cand_lv[parent] + sm.row_lp[row * k + r];
      sm.cand_lv[g] = lv;
      sm.cand_tok[g] = sm.row_tok[row * k + r];
      sm.cand_par[g] = parent;
      sm.keys[g] = cand_key(lv, g);
    }
    __syncthreads();
  }

  // 3. rerank: rank among all P = rank in its own level + the larger keys of
  //    every other level (an 8-way search of that level's descending list);
  //    with per-level widths, the level's rank against its width.  Threads
  //    take the levels' sorted lists in order, so the lanes of a warp search
  //    for neighbouring keys (the same or adjacent words) and a warp of ranks
  //    past n leaves at once.
  for (int e = tid; e < P; e += NT) {
    const uint64_t x = sm.sorted[e];
    const int g = key_gid(x);
    const int own = e < k ? 1 : 2 + (e - k) / kk;
    int rank = e - (own == 1 ? 0 : k + (own - 2) * kk);
    if (lw.on) {
      sm.node_of[g] = rank < lw.w[own - 1] ? 1 : 0;
      continue;
    }
    for (int level = 1; level <= depth && rank < n; ++level) {
      if (level == own) continue;
      const int lo = level == 1 ? 0 : k + (level - 2) * kk;
      rank += count_greater(sm.sorted + lo, level == 1 ? k : kk, x);
    }
    sm.node_of[g] = rank < n ? 1 : 0;
  }
  __syncthreads();

  // 4. renumber kept candidates by ascending id (block scan over contiguous ranges)
  const int per = (P + NT - 1) / NT;
  const int g0 = min(P, tid * per), g1 = min(P, g0 + per);
  int local = 0;
  for (int g = g0; g < g1; ++g) local += sm.node_of[g];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.warp_cnt[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += sm.warp_cnt[w];
  int next = base + incl - local;
  for (int g = g0; g < g1; ++g)
    if (sm.node_of[g]) sm.node_of[g] = ++next;
  __syncthreads();

  for (int g = tid; g < P; g += NT) {
    const int node = sm.node_of[g];
    if (!node) continue;
    const size_t o = (size_t)b * n + (node - 1);
    const int par = sm.cand_par[g];
    out.tokens[o] = sm.cand_tok[g];
    out.parents[o] = par < 0 ? 0 : sm.node_of[par];
    out.depth[o] = g < k ? 1 : 2 + (g - k) / kk;
    out.logV[o] = (float)sm.cand_lv[g];
    if (out.gid) out.gid[o] = g;
    out.draft_row[(size_t)b * (n + 1) + node] = sm.cand_row[g];
    sm.node_par[node - 1] = par < 0 ? 0 : sm.node_of[par];
    sm.node_dep[node - 1] = g < k ? 1 : 2 + (g - k) / kk;
  }
  if (tid == 0) out.draft_row[(size_t)b * (n + 1)] = 0;
  if (mo.mask == nullptr) return;
  // 5. (fused mask) node i+1 sees itself and its ancestors: walk the parent chain
  __syncthreads();
  for (int i = tid; i < n; i += NT) {
    uint64_t w0 = 0, w1 = 0;
    int node = i + 1;
    for (int step = 0; step < n && node >= 1; ++step) {
      const int j = node - 1;
      if (j < 64) w0 |= 1ull << j; else w1 |= 1ull << (j - 64);
      node = sm.node_par[j];
    }
    const size_t o = (size_t)b * n + i;
    mo.mask[o * 2] = w0;
    mo.mask[o * 2 + 1] = w1;
    if (mo.pos) mo.pos[o] = mo.prefix_len[b] - 1 + sm.node_dep[i];
  }
}

// Block size of the expansion: 128 threads for pools up to 128 candidates,
// else 256 (the work is in per-level loops; block barriers cost less with
// fewer warps).
static int build_threads(int P) { return P <= 128 ? 128 : kBuildThreads; }

size_t tree_build_smem_bytes(int R, int k, int P) {
  const int nt = build_threads(P);
  return sizeof(double) * ((size_t)R * k + P) + 2 * sizeof(uint64_t) * P +
         sizeof(int) * ((size_t)R * k + 4 * (size_t)P + 32 + nt / 32 + 2 * EAGLE_MAX_NODES);
}

// workspace: [chunk stats][chunk keys][row tokens B*R*k int32][row logits B*R*k float]
size_t tree_build_ws_bytes(int B, int R, int V, int elem_bytes, int k) {
  const size_t rows = (size_t)B * R;
  return row_stats_ws_bytes((long long)rows, V, elem_bytes, k) + align_up(rows * k * sizeof(int32_t), 256) +
         align_up(rows * k * sizeof(float), 256);
}

cudaError_t launch_tree_expand(const int32_t* row_tok, const float* row_val, int B, int R, int depth, int k, int n,
                               const eagle_tree_t& out, const MaskOut* mo_in, bool pdl, cudaStream_t s,
                               const int* widths) {
  const int P = k + (depth - 1) * k * k;
  const size_t smem = tree_build_smem_bytes(R, k, P);
  const MaskOut mo = mo_in ? *mo_in : MaskOut{nullptr, nullptr, nullptr};
  LevelWidths lw = {};
  lw.on = widths != nullptr;
  for (int l = 0; widths && l < depth; ++l) lw.w[l] = widths[l];
  auto go = [&](auto kernel, int nt) -> cudaError_t {
    cudaError_t e2 = ensure_smem_limit((const void*)kernel, smem);
    if (e2 != cudaSuccess) return e2;
    return launch_kernel(kernel, dim3(B), dim3(nt), smem, s, pdl, row_tok, row_val, R, depth, k, n, out, mo, lw);
  };
  if (build_threads(P) == 128) return go(tree_expand_kernel<128>, 128);
  return go(tree_expand_kernel<kBuildThreads>, kBuildThreads);
}

cudaError_t launch_tree_build(const void* draft_logits, int dtype, int B, int R, int V, int depth, int k, int n,
                              const eagle_tree_t& out, void* ws, cudaStream_t s, const MaskOut* mo_in,
                              bool zero_tickets, bool pdl) {
  const long long rows = (long long)B * R;
  const int eb = dtype_bytes(dtype);
  char* tail = static_cast<char*>(ws) + row_stats_ws_bytes(rows, V, eb, k);
  RowOut ro;
  ro.tok = reinterpret_cast<int32_t*>(tail);
  ro.val = reinterpret_cast<float*>(tail + align_up((size_t)rows * k * sizeof(int32_t), 256));
  ro.lse = out.row_lse;
  cudaError_t e = launch_row_stats(draft_logits, dtype, rows, V, k, true, ro, ws, s, zero_tickets, pdl);
  if (e != cudaSuccess) return e;
  return launch_tree_expand(ro.tok, ro.val, B, R, depth, k, n, out, mo_in, pdl, s);
}

}  // namespace eagle
