// Tree attention mask ("Технический анализ EAGLE-4", section "Деревья проверки
// EAGLE-4 и утилита управления"): a tree token sees the shared prefix, its
// ancestors and itself.  One thread per node walks the parent chain (at most
// n steps) and writes the node's two mask words and its position id.
#include "eagle_internal.h"

namespace eagle {

__global__ void tree_mask_kernel(const int32_t* __restrict__ parents, const int32_t* __restrict__ depth,
                                 const int32_t* __restrict__ prefix_len, int B, int n,
                                 uint64_t* __restrict__ mask, int32_t* __restrict__ pos) {
  griddep_wait();
  griddep_launch_dependents();
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * n) return;
  const int b = (int)(t / n), i = (int)(t - (long long)b * n);
  const int32_t* par = parents + (size_t)b * n;
  uint64_t w0 = 0, w1 = 0;
  int node = i + 1;
  for (int step = 0; step < n && node >= 1 && node <= i + 1; ++step) {
    const int j = node - 1;
    if (j < 64) w0 |= 1ull << j; else w1 |= 1ull << (j - 64);
    const int p = par[j];
    if (p >= node) break;  // parents must precede children
    node = p;
  }
  mask[(size_t)t * 2 + 0] = w0;
  mask[(size_t)t * 2 + 1] = w1;
  if (pos) pos[t] = prefix_len[b] - 1 + depth[t];
}

cudaError_t launch_tree_mask(const int32_t* parents, const int32_t* depth, const int32_t* prefix_len,
                             int B, int n, uint64_t* mask, int32_t* pos, cudaStream_t s) {
  const long long total = (long long)B * n;
  const int threads = 128;
  const long long blocks = (total + threads - 1) / threads;
  tree_mask_kernel<<<(unsigned)blocks, threads, 0, s>>>(parents, depth, prefix_len, B, n, mask, pos);
  return cudaGetLastError();
}

}  // namespace eagle
