// EAGLE-2 dynamic draft tree ("EAGLE" notes, EAGLE-2 sections "Expansion of
// tree" and "Reranking Nodes").  One CTA per sequence:
//   1. merge the chunk statistics of the sequence's R draft rows into each
//      row's log-sum-exp and top-k (token, log-confidence lp = logit - lse);
//   2. level 1 = the root's k children; for each level up to depth-1, rank the
//      level's candidates by (log V desc, candidate id asc), the first k form
//      the frontier (slot = rank, which names the draft row of the node), and
//      their k children each enter the next level with
//      log V = log V(parent) + lp (log of the product of confidences);
//   3. a block-wide bitonic sort over all P candidates keeps the best n;
//   4. a prefix count renumbers the kept candidates 1..n by ascending id and
//      the tree arrays are written.
// log V is carried in fp64 so that the rounding of one path sum can only
// reorder candidates whose values agree to ~1e-15 relative.
#include <climits>

#include "eagle_internal.h"

namespace eagle {

constexpr int kBuildThreads = 256;

struct BuildSmem {
  double* row_lp;  // [R*k]
  double* cand_lv; // [P]
  double* sort_lv; // [Ppow]
  int* row_tok;    // [R*k]
  int* cand_tok;   // [P]
  int* cand_par;   // [P]   parent candidate id, -1 = root
  int* cand_row;   // [P]   draft row of an expanded candidate, -1 otherwise
  int* node_of;    // [P]   kept flag, then 1-based node id (0 = dropped)
  int* sort_gid;   // [Ppow]
  int* frontier;   // [32]
  int* scan;       // [kBuildThreads + 1]
};

__host__ __device__ inline int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

__device__ __forceinline__ bool cand_better(double la, int ga, double lb, int gb) {
  return la > lb || (la == lb && ga < gb);
}

__global__ void __launch_bounds__(kBuildThreads)
tree_expand_kernel(const ChunkStat* __restrict__ stats, const uint64_t* __restrict__ keys,
                   int n_chunks, int R, int depth, int k, int n, eagle_tree_t out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = kBuildThreads / 32;
  const int kk = k * k;
  const int P = k + (depth - 1) * kk;
  const int Ppow = next_pow2(P);

  BuildSmem sm;
  {
    unsigned char* p = smem_raw;
    sm.row_lp = reinterpret_cast<double*>(p);  p += sizeof(double) * R * k;
    sm.cand_lv = reinterpret_cast<double*>(p); p += sizeof(double) * P;
    sm.sort_lv = reinterpret_cast<double*>(p); p += sizeof(double) * Ppow;
    sm.row_tok = reinterpret_cast<int*>(p);    p += sizeof(int) * R * k;
    sm.cand_tok = reinterpret_cast<int*>(p);   p += sizeof(int) * P;
    sm.cand_par = reinterpret_cast<int*>(p);   p += sizeof(int) * P;
    sm.cand_row = reinterpret_cast<int*>(p);   p += sizeof(int) * P;
    sm.node_of = reinterpret_cast<int*>(p);    p += sizeof(int) * P;
    sm.sort_gid = reinterpret_cast<int*>(p);   p += sizeof(int) * Ppow;
    sm.frontier = reinterpret_cast<int*>(p);   p += sizeof(int) * 32;
    sm.scan = reinterpret_cast<int*>(p);
  }

  // 1. per-row log-sum-exp and top-k
  for (int r = warp; r < R; r += nwarps) {
    const size_t row = (size_t)b * R + r;
    double lse = 0.0;
    uint64_t key = 0;
    warp_finalize_row(stats + row * n_chunks, keys + row * n_chunks * k, n_chunks, k, true, &lse, &key);
    if (lane < k) {
      sm.row_tok[r * k + lane] = key ? key_index(key) : -1;
      sm.row_lp[r * k + lane] = key ? (double)key_value(key) - lse : -INFINITY;
    }
    if (lane == 0) out.row_lse[row] = lse;
  }
  __syncthreads();

  // 2. level by level
  for (int c = tid; c < k; c += kBuildThreads) {
    sm.cand_lv[c] = sm.row_lp[c];
    sm.cand_tok[c] = sm.row_tok[c];
    sm.cand_par[c] = -1;
    sm.cand_row[c] = -1;
  }
  __syncthreads();
  for (int level = 1; level < depth; ++level) {
    const int lo = level == 1 ? 0 : k + (level - 2) * kk;
    const int cnt = level == 1 ? k : kk;
    for (int c = lo + tid; c < lo + cnt; c += kBuildThreads) {
      const double lv = sm.cand_lv[c];
      int rank = 0;
      for (int o = lo; o < lo + cnt; ++o) rank += cand_better(sm.cand_lv[o], o, lv, c) ? 1 : 0;
      if (rank < k) {
        sm.frontier[rank] = c;
        sm.cand_row[c] = 1 + (level - 1) * k + rank;
      }
    }
    __syncthreads();
    const int lo2 = k + (level - 1) * kk;
    for (int idx = tid; idx < kk; idx += kBuildThreads) {
      const int s = idx / k, r = idx - s * k;
      const int parent = sm.frontier[s];
      const int row = 1 + (level - 1) * k + s;
      const int g = lo2 + idx;
      sm.cand_lv[g] = sm.cand_lv[parent] + sm.row_lp[row * k + r];
      sm.cand_tok[g] = sm.row_tok[row * k + r];
      sm.cand_par[g] = parent;
      sm.cand_row[g] = -1;
    }
    __syncthreads();
  }

  // 3. rerank: bitonic sort of all candidates, best first
  for (int i = tid; i < Ppow; i += kBuildThreads) {
    sm.sort_lv[i] = i < P ? sm.cand_lv[i] : -INFINITY;
    sm.sort_gid[i] = i < P ? i : INT_MAX;
  }
  for (int i = tid; i < P; i += kBuildThreads) sm.node_of[i] = 0;
  __syncthreads();
  for (int size = 2; size <= Ppow; size <<= 1) {
    for (int j = size >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < Ppow; i += kBuildThreads) {
        const int o = i ^ j;
        if (o > i) {
          const bool desc = (i & size) == 0;
          const bool i_better = cand_better(sm.sort_lv[i], sm.sort_gid[i], sm.sort_lv[o], sm.sort_gid[o]);
          if (desc != i_better) {
            const double tl = sm.sort_lv[i]; sm.sort_lv[i] = sm.sort_lv[o]; sm.sort_lv[o] = tl;
            const int tg = sm.sort_gid[i]; sm.sort_gid[i] = sm.sort_gid[o]; sm.sort_gid[o] = tg;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n; i += kBuildThreads) sm.node_of[sm.sort_gid[i]] = 1;
  __syncthreads();

  // 4. renumber kept candidates by ascending id
  const int per = (P + kBuildThreads - 1) / kBuildThreads;
  const int g0 = min(P, tid * per), g1 = min(P, g0 + per);
  int local = 0;
  for (int g = g0; g < g1; ++g) local += sm.node_of[g];
  sm.scan[tid] = local;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int t = 0; t < kBuildThreads; ++t) { const int v = sm.scan[t]; sm.scan[t] = acc; acc += v; }
  }
  __syncthreads();
  int next = sm.scan[tid];
  for (int g = g0; g < g1; ++g)
    if (sm.node_of[g]) sm.node_of[g] = ++next;
  __syncthreads();

  for (int g = tid; g < P; g += kBuildThreads) {
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
  }
  if (tid == 0) out.draft_row[(size_t)b * (n + 1)] = 0;
}

size_t tree_build_smem_bytes(int R, int k, int P) {
  const int Ppow = next_pow2(P);
  return sizeof(double) * ((size_t)R * k + P + Ppow) +
         sizeof(int) * ((size_t)R * k + 4 * (size_t)P + Ppow + 32 + kBuildThreads + 1);
}

cudaError_t launch_tree_expand(const ChunkStat* stats, const uint64_t* keys, int n_chunks, int B, int R,
                               int depth, int k, int n, const eagle_tree_t& out, cudaStream_t s) {
  const int P = k + (depth - 1) * k * k;
  const size_t smem = tree_build_smem_bytes(R, k, P);
  cudaError_t e = ensure_smem_limit((const void*)tree_expand_kernel, smem);
  if (e != cudaSuccess) return e;
  tree_expand_kernel<<<B, kBuildThreads, smem, s>>>(stats, keys, n_chunks, R, depth, k, n, out);
  return cudaGetLastError();
}

}  // namespace eagle
