// Host plan of the tree attention ("Tree Attention" verification of the EAGLE
// notes, "3.Verify"): how many CTAs share the tile list, and the workspace that
// holds the partials of units cut by CTA range boundaries.  The kernels are in
// attention_tc.cu.
#include <atomic>

#include "eagle_internal.h"

namespace eagle {

namespace {
std::atomic<unsigned long long> g_probe_ns{0};
}  // namespace

unsigned long long attention_wait_probe_ns() { return g_probe_ns.load(std::memory_order_relaxed); }

int attention_row_groups(int n, int Hq, int Hkv) {
  const int rows = n * (Hq / Hkv);
  return (rows + kAttnRowsPerUnit - 1) / kAttnRowsPerUnit;
}

int attention_ctas(int B, int n, int Hq, int Hkv, int Lmax, int window) {
  const long long span = window > 0 ? (Lmax < window ? Lmax : window) : Lmax;
  const long long tiles_max = (span + kAttnKeysPerTile - 1) / kAttnKeysPerTile + (n + kAttnKeysPerTile - 1) / kAttnKeysPerTile;
  const long long T_max = (long long)B * Hkv * attention_row_groups(n, Hq, Hkv) * tiles_max;
  const int sms = device_sm_count();
  return (int)(T_max < sms ? T_max : sms);
}

AttnWorkspace attention_ws_layout(int B, int n, int Hq, int Hkv, int D, int Lmax, int window) {
  AttnWorkspace w;
  const int C = attention_ctas(B, n, Hq, Hkv, Lmax, window);
  const size_t U = (size_t)B * Hkv * attention_row_groups(n, Hq, Hkv);
  const size_t slots = (size_t)C + U;
  w.status_off = 0;
  w.cta_status_off = 256;
  w.part_lse_off = align_up(w.cta_status_off + sizeof(int) * (size_t)C, 256);
  w.part_o_off = align_up(w.part_lse_off + sizeof(float) * slots * kAttnRowsPerUnit, 256);
  w.bytes = align_up(w.part_o_off + sizeof(float) * slots * kAttnRowsPerUnit * (size_t)D, 256);
  return w;
}

}  // namespace eagle

extern "C" EAGLE_API void eagle_debug_attention_wait_probe(unsigned long long limit_ns) {
  eagle::g_probe_ns.store(limit_ns, std::memory_order_relaxed);
}
