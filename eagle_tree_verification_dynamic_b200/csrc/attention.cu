// Host plan of the tree attention ("Tree Attention" verification of the EAGLE
// notes, "3.Verify"): how many key splits, and how many keys each, so that
// about two CTAs per SM are busy; the kernel itself is attention_tc.cu.
#include "eagle_internal.h"

namespace eagle {

AttnPlan plan_attention(int B, int n, int Hq, int Hkv, int Lmax, int window) {
  AttnPlan p;
  p.span = window > 0 ? (Lmax < window ? Lmax : window) : Lmax;
  if (p.span < 1) p.span = 1;
  // two CTAs per SM: aim for ~2 x 148 CTAs over (row groups x heads x splits);
  // the splits of one head (plus its tree-key split) form one cluster of <= 16
  const int heads = B * Hkv * attention_row_groups(n, Hq, Hkv);
  int splits = (2 * kNumSMs + heads - 1) / heads;
  const int max_splits = (p.span + 63) / 64;
  if (splits > max_splits) splits = max_splits;
  if (splits > 15) splits = 15;
  if (splits < 1) splits = 1;
  int chunk = (p.span + splits - 1) / splits;
  chunk = (chunk + 63) / 64 * 64;
  p.chunk = chunk;
  p.n_splits = (p.span + chunk - 1) / chunk;
  return p;
}

// workspace: a 256-byte header holding the kernel's device status word
size_t attention_ws_bytes(int, int, int, int, int, int, int) { return 256; }

cudaError_t launch_tree_attention(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                                  const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                                  int n, int Hq, int Hkv, int D, int window, float scale, void* out, void* ws,
                                  cudaStream_t s) {
  const AttnPlan p = plan_attention(B, n, Hq, Hkv, Lmax, window);
  int* err = reinterpret_cast<int*>(ws);
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  return launch_attention_tc(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, D, window, scale, p, out,
                             err, s);
}

}  // namespace eagle
