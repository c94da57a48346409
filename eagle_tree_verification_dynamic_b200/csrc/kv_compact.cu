// KV-cache compaction after acceptance (EAGLE-4 write-up, "Технический анализ
// EAGLE-4", section "Деревья проверки EAGLE-4 и утилита управления": after
// verification the accepted continuation is kept and the rejected KV-cache
// entries are freed before the next round).
//
// The verification pass produced keys and values for every tree node; the
// accepted path's entries are appended to the sequence's prefix cache in path
// order (the i-th accepted node, depth i + 1, goes to position prefix_len + i,
// its position id), the rejected ones are simply not copied.  One CTA per
// (sequence, accepted slot) copies that node's rows of all KV heads with
// 16-byte vectors.  The copy ends at the first path entry that is not a node
// id of the tree or whose position would reach Lmax; the new prefix length
// counts the entries copied.  A paged cache (pools [num_pages][Hkv][page_size]
// [D]) takes position pos at offset pos % page_size of page
// block_table[b][pos / page_size]; the copy also ends at a position whose page
// id lies outside the pool (a page the caller has not allocated yet).
#include "eagle_internal.h"

namespace eagle {

constexpr int kCompactThreads = 128;

__global__ void __launch_bounds__(kCompactThreads)
kv_compact_kernel(const uint4* __restrict__ k_tree, const uint4* __restrict__ v_tree, const int32_t* __restrict__ path,
                  const int32_t* __restrict__ accepted_len, const int32_t* __restrict__ prefix_len,
                  uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, int32_t* __restrict__ new_len, int n,
                  int Hkv, int vec_per_row, int Lmax, int depth, PagedKV pg) {
  griddep_wait();  // the path comes from the acceptance kernel
  griddep_launch_dependents();
  const int b = blockIdx.x, i = blockIdx.y;
  const int L = min(max(prefix_len[b], 0), Lmax);
  const int a = min(max(accepted_len[b], 0), depth);
  const int32_t* pb = path + (size_t)b * depth;
  const int32_t* bt = pg.block_table ? pg.block_table + (size_t)b * pg.pages_per_seq : nullptr;
  // the page of position pos (-1: none), paged caches only
  auto page_of = [&](int pos) {
    const int e = pos / pg.page_size;
    const int id = e < pg.pages_per_seq ? bt[e] : -1;
    return id >= 0 && id < pg.num_pages ? id : -1;
  };
  int cnt = 0;  // entries that will be copied: the valid prefix of the path
  while (cnt < a && L + cnt < Lmax && pb[cnt] >= 1 && pb[cnt] <= n && (!bt || page_of(L + cnt) >= 0)) ++cnt;
  if (i == 0 && threadIdx.x == 0) new_len[b] = L + cnt;
  if (i >= cnt) return;
  const int node = pb[i];
  const size_t src_row = ((size_t)b * n + (node - 1)) * Hkv;  // [B][n][Hkv] rows
  // destination row of head 0 and the stride between heads, in rows of D
  size_t dst_row, head_stride;
  if (bt) {
    const int pos = L + i;
    dst_row = (size_t)page_of(pos) * Hkv * pg.page_size + pos % pg.page_size;  // [num_pages][Hkv][page_size]
    head_stride = pg.page_size;
  } else {
    dst_row = (size_t)b * Hkv * Lmax + (L + i);  // [B][Hkv][Lmax]
    head_stride = Lmax;
  }
  for (int e = threadIdx.x; e < Hkv * vec_per_row; e += kCompactThreads) {
    const int h = e / vec_per_row, c = e - h * vec_per_row;
    const size_t s = (src_row + h) * vec_per_row + c;
    const size_t d = (dst_row + (size_t)h * head_stride) * vec_per_row + c;
    k_cache[d] = k_tree[s];
    v_cache[d] = v_tree[s];
  }
}

cudaError_t launch_kv_compact(const void* k_tree, const void* v_tree, const int32_t* path, const int32_t* accepted_len,
                              const int32_t* prefix_len, void* k_cache, void* v_cache, int32_t* new_len, int B, int n,
                              int Hkv, int D, int Lmax, int depth, cudaStream_t s, const PagedKV* pg) {
  const int vec_per_row = D * 2 / 16;  // bf16 rows of D values, D % 8 == 0
  PagedKV none = {nullptr, 1, 0, 0};
  const PagedKV pk = pg && pg->block_table ? *pg : none;
  if (pk.block_table) Lmax = pk.pages_per_seq * pk.page_size;
  return launch_kernel(kv_compact_kernel, dim3(B, depth), dim3(kCompactThreads), 0, s, false,
                       static_cast<const uint4*>(k_tree), static_cast<const uint4*>(v_tree), path, accepted_len,
                       prefix_len, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), new_len, n, Hkv,
                       vec_per_row, Lmax, depth, pk);
}

}  // namespace eagle
