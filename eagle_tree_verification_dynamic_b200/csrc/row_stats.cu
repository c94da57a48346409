// Vocabulary sweep over logit rows: the top-k tokens of each row by raw logit
// (ties to the lower token id) and the row's log-sum-exp.  The top-k of the
// draft rows gives the candidate children of a tree node and the log-sum-exp
// turns logits into draft confidences c(x) = exp(l_x) / sum_i exp(l_i)
// ("EAGLE" notes, EAGLE-2 "Well-Calibrated Draft Model"); on target rows the
// same sweep (k = 1) gives the argmax for greedy acceptance and the normaliser
// of p_target for sampling.
//
// One CTA owns one (row, chunk).  Threads stream 16-byte vectors (coalesced,
// L1 no-allocate) and keep, per lane, the M best (value, id) pairs in
// registers plus a base-2 scaled fp64 partial of sum exp(logit).  A warp
// builds its exact top-k from the lanes' lists with bitonic sort/merge rounds
// (a lane is rescanned from memory only if all M of its entries made the
// cut); warps merge pairwise through shared memory.  The CTA that finishes a
// row's last chunk (an atomic ticket; nobody waits) merges the row's chunks
// and writes the final per-row outputs.
#include "eagle_internal.h"

namespace eagle {

constexpr int kStatThreads = 256;
constexpr int kStatWarps = kStatThreads / 32;
constexpr int kUnroll = 8;

// The M largest (value, id) pairs seen by a lane, sorted descending.  Elements
// arrive in increasing id and only a strictly larger value moves ahead, so
// among equal values the lower id stays first.
template <int M>
struct LaneTop {
  float s[M];
  int id[M];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int p = 0; p < M; ++p) { s[p] = -INFINITY; id[p] = -1; }
  }
  __device__ __forceinline__ void push(float v, int idx) {
    if (!(v > s[M - 1])) return;
#pragma unroll
    for (int p = 0; p < M; ++p) {
      if (v > s[p]) {
        const float tv = s[p]; s[p] = v; v = tv;
        const int ti = id[p]; id[p] = idx; idx = ti;
      }
    }
  }
  __device__ __forceinline__ uint64_t key(int p) const { return id[p] >= 0 ? make_key(s[p], id[p]) : 0ull; }
};

// Largest key strictly below `last` among this lane's elements of the chunk
// (same element assignment as the main sweep; -inf and NaN never qualify).
template <typename T, bool VEC>
__device__ uint64_t lane_next_below(const T* __restrict__ rp, int c0, int c1, uint64_t last) {
  uint64_t best = 0;
  if (VEC) {
    constexpr int N = Elem<T>::kPerVec;
    const uint4* vp = reinterpret_cast<const uint4*>(rp + c0);
    const int nvec = (c1 - c0) / N;
    for (int vi = threadIdx.x; vi < nvec; vi += kStatThreads) {
      float f[N];
      Elem<T>::unpack(__ldg(vp + vi), f);
#pragma unroll
      for (int i = 0; i < N; ++i) {
        if (!(f[i] > -INFINITY)) continue;
        const uint64_t key = make_key(f[i], c0 + vi * N + i);
        if (key < last && key > best) best = key;
      }
    }
  } else {
    for (int i = c0 + threadIdx.x; i < c1; i += kStatThreads) {
      const float v = Elem<T>::load(rp + i);
      if (!(v > -INFINITY)) continue;
      const uint64_t key = make_key(v, i);
      if (key < last && key > best) best = key;
    }
  }
  return best;
}

template <typename T, bool LSE, bool VEC, int M>
__global__ void __launch_bounds__(kStatThreads)
row_stats_kernel(const T* __restrict__ x, int V, int chunk_elems, int k, ChunkStat* __restrict__ stats,
                 uint64_t* __restrict__ keys, int* __restrict__ tickets, RowOut out) {
  griddep_wait();  // the logits (and this workspace) may belong to the previous kernel
  const long long row = blockIdx.x;
  const int chunk = blockIdx.y, n_chunks = gridDim.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* rp = x + (size_t)row * (size_t)V;
  const int c0 = chunk * chunk_elems;
  const int c1 = min(V, c0 + chunk_elems);

  LaneTop<M> top;
  top.init();
  float e_ref = -INFINITY;
  double acc = 0.0;

  auto process = [&](const float* f, int n, int idx0) {
    float vmax = f[0];
#pragma unroll
    for (int i = 1; i < Elem<T>::kPerVec; ++i)
      if (i < n) vmax = fmaxf(vmax, f[i]);
    if (vmax > top.s[M - 1]) {
#pragma unroll
      for (int i = 0; i < Elem<T>::kPerVec; ++i)
        if (i < n) top.push(f[i], idx0 + i);
    }
    if (LSE) {
      if (vmax * kLog2eHi > e_ref) {  // a new reference exponent (rare)
        const float e_new = ceilf(vmax * kLog2eHi);
        acc = rescale_pow2(acc, e_ref, e_new);
        e_ref = e_new;
      }
      if (e_ref > -INFINITY) {  // until a finite logit arrives every term is exp(-inf) = 0
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < Elem<T>::kPerVec; ++i)
          if (i < n) part += exp2_scaled(f[i], e_ref);
        acc += (double)part;
      }
    }
  };

  if (VEC) {
    constexpr int N = Elem<T>::kPerVec;
    const uint4* vp = reinterpret_cast<const uint4*>(rp + c0);
    const int nvec = (c1 - c0) / N;
    for (int base = tid; base < nvec; base += kStatThreads * kUnroll) {
      uint4 buf[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int vi = base + u * kStatThreads;
        if (vi < nvec) buf[u] = ld_stream(vp + vi);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int vi = base + u * kStatThreads;
        if (vi < nvec) {
          float f[N];
          Elem<T>::unpack(buf[u], f);
          process(f, N, c0 + vi * N);
        }
      }
    }
  } else {
    for (int i = c0 + tid; i < c1; i += kStatThreads) {
      float f[Elem<T>::kPerVec];
      f[0] = Elem<T>::load(rp + i);
      process(f, 1, i);
    }
  }

  griddep_launch_dependents();  // every CTA that reaches here has done its streaming
  __shared__ uint64_t s_keys[kStatWarps][32];
  __shared__ float s_e[kStatWarps];
  __shared__ double s_s[kStatWarps];
  __shared__ int s_last;

  // ---- warp top-k: lane bests first, then the next entries of the lanes whose
  // previous entry made the cut
  uint64_t list;
  if (k == 1) {
    list = warp_max_u64(top.key(0));
  } else {
    list = warp_sort_desc(top.key(0));
    uint64_t thr = __shfl_sync(kFull, list, k - 1);
    bool need = top.key(0) != 0 && top.key(0) >= thr;
    int r = 1;
    for (; r < M; ++r) {
      const uint64_t cand = need ? top.key(r) : 0ull;
      if (!__any_sync(kFull, cand != 0)) { need = false; break; }
      list = warp_merge_desc(list, warp_sort_desc(cand));
      thr = __shfl_sync(kFull, list, k - 1);
      need = cand != 0 && cand >= thr;
    }
    // all M entries of some lane made the cut: pull its further elements (rare)
    uint64_t last = (r == M && need) ? top.key(M - 1) : 0ull;
    need = last != 0;
    while (__any_sync(kFull, need)) {
      uint64_t nxt = 0;
      if (need) nxt = lane_next_below<T, VEC>(rp, c0, c1, last);
      list = warp_merge_desc(list, warp_sort_desc(nxt));
      thr = __shfl_sync(kFull, list, k - 1);
      need = nxt != 0 && nxt >= thr;
      last = nxt;
    }
  }
  if (lane < k) s_keys[warp][lane] = list;

  // ---- warp partial sums
  if (LSE) {
    const float e = warp_max_f(e_ref);
    double sacc = acc > 0.0 ? rescale_pow2(acc, e_ref, e) : 0.0;
    sacc = warp_sum_d(sacc);
    if (lane == 0) { s_e[warp] = e; s_s[warp] = sacc; }
  }
  __syncthreads();

  // merge the warps' lists pairwise: 3 rounds for 8 warps
  for (int step = 1; step < kStatWarps; step <<= 1) {
    if ((warp & (2 * step - 1)) == 0 && warp + step < kStatWarps) {
      const uint64_t m = warp_merge_desc(lane < k ? s_keys[warp][lane] : 0ull,
                                         lane < k ? s_keys[warp + step][lane] : 0ull);
      if (lane < k) s_keys[warp][lane] = m;
    }
    __syncthreads();
  }

  const size_t slot = (size_t)row * n_chunks + chunk;
  if (warp == 0) {
    if (lane < k) keys[slot * k + lane] = s_keys[0][lane];
    if (LSE && lane == 0) {
      LseAccum a;
      a.init();
      for (int w = 0; w < kStatWarps; ++w) a.add(s_e[w], s_s[w]);
      ChunkStat cs;
      cs.e_ref = a.e;
      cs.pad = 0;
      cs.acc = a.s;
      stats[slot] = cs;
    }
  }

  // ---- the CTA that completes the row merges all of its chunks
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(tickets + row, 1) == n_chunks - 1;
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  const ChunkStat* st = stats + (size_t)row * n_chunks;
  const uint64_t* kk = keys + (size_t)row * n_chunks * k;
  double lse = 0.0;
  if (LSE) {
    LseAccum a;
    a.init();
    for (int c = lane; c < n_chunks; c += 32) {
      const float e2 = __ldcg(&st[c].e_ref);
      const double s2 = __ldcg(&st[c].acc);
      a.add(e2, s2);
    }
    const float e = warp_max_f(a.e);
    double s = a.s > 0.0 ? rescale_pow2(a.s, a.e, e) : 0.0;
    s = warp_sum_d(s);
    lse = s > 0.0 ? kLn2 * ((double)e + log2(s)) : -INFINITY;
  }
  uint64_t merged = 0ull;
  for (int c = 0; c < n_chunks; c += 8) {  // 8 chunk lists in flight, then merged
    uint64_t kv[8];
#pragma unroll
    for (int t = 0; t < 8; ++t)
      kv[t] = (lane < k && c + t < n_chunks) ? __ldcg(reinterpret_cast<const unsigned long long*>(kk) + (c + t) * k + lane) : 0ull;
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (c + t < n_chunks) merged = warp_merge_desc(merged, kv[t]);
  }
  if (lane < k) {
    if (out.tok) out.tok[row * k + lane] = merged ? key_index(merged) : -1;
    if (out.val) out.val[row * k + lane] = merged ? key_value(merged) : -INFINITY;
  }
  if (LSE && out.lse && lane == 0) out.lse[row] = lse;
}

// ------------------------------------------------------------------- host
ChunkPlan plan_chunks(long long rows, int V, int elem_bytes) {
  const int per_vec = 16 / elem_bytes;
  const long long target = 4LL * device_sm_count();
  long long want = rows > 0 ? (target + rows - 1) / rows : 1;
  const long long max_chunks = V / 4096 > 1 ? V / 4096 : 1;
  if (want < 1) want = 1;
  if (want > max_chunks) want = max_chunks;
  ChunkPlan p;
  int ce = (int)((V + want - 1) / want);
  ce = (ce + per_vec - 1) / per_vec * per_vec;
  p.chunk_elems = ce;
  p.n_chunks = (V + ce - 1) / ce;
  return p;
}

// workspace: [chunk stats rows*nc][chunk keys rows*nc*k][row tickets rows]
size_t row_stats_ws_bytes(long long rows, int V, int elem_bytes, int k, long long plan_rows) {
  const ChunkPlan p = plan_chunks(plan_rows > 0 ? plan_rows : rows, V, elem_bytes);
  const size_t n = (size_t)rows * p.n_chunks;
  return align_up(n * sizeof(ChunkStat), 256) + align_up(n * k * sizeof(uint64_t), 256) +
         align_up((size_t)rows * sizeof(int), 256);
}

template <typename T, bool LSE, int M>
static cudaError_t launch_typed(const void* x, long long rows, int V, int k, const ChunkPlan& p, bool vec,
                                ChunkStat* stats, uint64_t* keys, int* tickets, const RowOut& out, cudaStream_t s,
                                bool pdl) {
  const dim3 grid((unsigned)rows, (unsigned)p.n_chunks);
  const T* xp = static_cast<const T*>(x);
  if (vec)
    return launch_kernel(row_stats_kernel<T, LSE, true, M>, grid, dim3(kStatThreads), 0, s, pdl, xp, V,
                         p.chunk_elems, k, stats, keys, tickets, out);
  return launch_kernel(row_stats_kernel<T, LSE, false, M>, grid, dim3(kStatThreads), 0, s, pdl, xp, V,
                       p.chunk_elems, k, stats, keys, tickets, out);
}

template <typename T>
static cudaError_t launch_t(const void* x, long long rows, int V, int k, bool lse, const ChunkPlan& p, bool vec,
                            ChunkStat* stats, uint64_t* keys, int* tickets, const RowOut& out, cudaStream_t s,
                            bool pdl) {
  if (k == 1) {
    if (lse) return launch_typed<T, true, 1>(x, rows, V, k, p, vec, stats, keys, tickets, out, s, pdl);
    return launch_typed<T, false, 1>(x, rows, V, k, p, vec, stats, keys, tickets, out, s, pdl);
  }
  if (lse) return launch_typed<T, true, 4>(x, rows, V, k, p, vec, stats, keys, tickets, out, s, pdl);
  return launch_typed<T, false, 4>(x, rows, V, k, p, vec, stats, keys, tickets, out, s, pdl);
}

void row_stats_tickets_span(long long rows, int V, int elem_bytes, int k, size_t* off, size_t* bytes) {
  const ChunkPlan p = plan_chunks(rows, V, elem_bytes);
  const size_t n = (size_t)rows * p.n_chunks;
  *off = align_up(n * sizeof(ChunkStat), 256) + align_up(n * k * sizeof(uint64_t), 256);
  *bytes = (size_t)rows * sizeof(int);
}

cudaError_t launch_row_stats(const void* x, int dtype, long long rows, int V, int k, bool lse, const RowOut& out,
                             void* ws, cudaStream_t s, bool zero_tickets, bool pdl, long long plan_rows) {
  const int eb = dtype_bytes(dtype);
  const ChunkPlan p = plan_chunks(plan_rows > 0 ? plan_rows : rows, V, eb);
  const size_t n = (size_t)rows * p.n_chunks;
  char* base = static_cast<char*>(ws);
  ChunkStat* stats = reinterpret_cast<ChunkStat*>(base);
  uint64_t* keys = reinterpret_cast<uint64_t*>(base + align_up(n * sizeof(ChunkStat), 256));
  int* tickets = reinterpret_cast<int*>(base + align_up(n * sizeof(ChunkStat), 256) +
                                        align_up(n * k * sizeof(uint64_t), 256));
  if (zero_tickets) {
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)rows * sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  const bool vec = ((uintptr_t)x % 16 == 0) && (((size_t)V * eb) % 16 == 0);
  if (dtype == EAGLE_F32) return launch_t<float>(x, rows, V, k, lse, p, vec, stats, keys, tickets, out, s, pdl);
  return launch_t<__nv_bfloat16>(x, rows, V, k, lse, p, vec, stats, keys, tickets, out, s, pdl);
}

}  // namespace eagle
