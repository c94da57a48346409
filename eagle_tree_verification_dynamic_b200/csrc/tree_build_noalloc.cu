// eagle_tree_build without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they build a
// tree: a serving loop whose memory pool is sealed after warm-up, a plugin or
// custom-op interface that hands a kernel only its input/output buffers and a
// stream, or a foreign-language caller with no device allocator at hand.  For
// them this entry point draws its scratch space from a fixed array that lives
// in the library itself, so nothing is allocated per call.
//
// The array is a file-scope __device__ object: every GPU on which the library
// is loaded holds kNoAllocScratchBytes for it until the process exits.  Host
// code cannot pass the array's name to a kernel (on the host it names a
// stand-in, not device memory), so on the first call on each device, with that
// device current, its device address is looked up with cudaGetSymbolAddress
// and cached.  That first call on a device should therefore be made before any
// stream capture begins.  The cached address lives as long as the process's
// context on that device: after cudaDeviceReset (or anything else that tears
// the primary context down) the library's module is loaded again elsewhere and
// the cached address is stale, so a process that resets a device must be
// restarted before it calls this entry point again.  Calls share the one
// array: two calls whose work overlaps on the GPU (different streams, or
// different host threads) race on it and must be serialised by the caller.
// What must start at zero is cleared on the caller's stream at every call: the
// per-row tickets of the vocabulary sweep are reset with cudaMemsetAsync
// before its kernel runs; every other scratch byte is written before it is
// read.
#include <mutex>

#include "eagle_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 2u << 20;  // 2 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_build_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" EAGLE_API eagle_status eagle_tree_build_noalloc(const void* draft_logits, int dtype, int B, int R, int V,
                                                           int depth, int k, int m, const eagle_tree_t* out,
                                                           int* n_nodes, void* stream) {
  const size_t need = eagle_tree_build_workspace_bytes(B, R, V, dtype, k);
  if (need > kNoAllocScratchBytes) return EAGLE_ERR_LIMIT;  // shape too large for the fixed scratch
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EAGLE_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_build_scratch);
      if (e != cudaSuccess || p == nullptr) return EAGLE_ERR_CUDA;
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return eagle_tree_build(draft_logits, dtype, B, R, V, depth, k, m, out, n_nodes, scratch, kNoAllocScratchBytes,
                          stream);
}
