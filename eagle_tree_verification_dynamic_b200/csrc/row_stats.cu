// Vocabulary sweep over logit rows: per chunk of a row, the top-k tokens by raw
// logit (ties to the lower token id) and a base-2 scaled partial of
// sum exp(logit).  The top-k of the draft rows gives the candidate children of
// a tree node and the log-sum-exp turns logits into draft confidences
// c(x) = exp(l_x) / sum_i exp(l_i) ("EAGLE" notes, EAGLE-2 "Well-Calibrated
// Draft Model"); on target rows the same sweep (k = 1) gives the argmax for
// greedy acceptance and the normaliser of p_target for sampling.
//
// One CTA owns one (row, chunk).  Threads stream 16-byte vectors (coalesced,
// L1 no-allocate) and keep, per lane, the two best (value, id) pairs plus a
// running partial sum; a warp then builds its exact top-k from the lanes'
// best keys with a bitonic sort, pulling a lane's further elements only when
// that lane already contributed twice.  Warps merge in shared memory.
#include "eagle_internal.h"

namespace eagle {

constexpr int kStatThreads = 256;
constexpr int kStatWarps = kStatThreads / 32;
constexpr int kUnroll = 8;

struct LaneTop2 {
  float s1, s2;
  int i1, i2;
  __device__ __forceinline__ void init() { s1 = s2 = -INFINITY; i1 = i2 = -1; }
  // Elements arrive in increasing id; a later equal value never displaces an
  // earlier one, so among equals the lower id stays ahead.
  __device__ __forceinline__ void push(float v, int idx) {
    if (v > s2) {
      if (v > s1) { s2 = s1; i2 = i1; s1 = v; i1 = idx; }
      else        { s2 = v; i2 = idx; }
    }
  }
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

template <typename T, bool LSE, bool VEC>
__global__ void __launch_bounds__(kStatThreads)
row_chunk_stats_kernel(const T* __restrict__ x, int V, int chunk_elems, int k,
                       ChunkStat* __restrict__ stats, uint64_t* __restrict__ keys) {
  const long long row = blockIdx.x;
  const int chunk = blockIdx.y, n_chunks = gridDim.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const T* rp = x + (size_t)row * (size_t)V;
  const int c0 = chunk * chunk_elems;
  const int c1 = min(V, c0 + chunk_elems);

  LaneTop2 top;
  top.init();
  float e_ref = -INFINITY;
  double acc = 0.0;

  auto process = [&](const float* f, int n, int idx0) {
    float vmax = f[0];
#pragma unroll
    for (int i = 1; i < Elem<T>::kPerVec; ++i)
      if (i < n) vmax = fmaxf(vmax, f[i]);
    if (vmax > top.s2) {
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

  __shared__ uint64_t s_keys[kStatWarps][32];
  __shared__ float s_e[kStatWarps];
  __shared__ double s_s[kStatWarps];

  // ---- warp top-k
  const uint64_t k1 = top.i1 >= 0 ? make_key(top.s1, top.i1) : 0ull;
  uint64_t list;
  if (k == 1) {
    list = warp_max_u64(k1);
  } else {
    list = warp_sort_desc(k1);
    uint64_t thr = __shfl_sync(kFull, list, k - 1);
    uint64_t last = top.i2 >= 0 ? make_key(top.s2, top.i2) : 0ull;
    bool need = last != 0 && last >= thr;
    while (__any_sync(kFull, need)) {
      list = warp_merge_desc(list, warp_sort_desc(need ? last : 0ull));
      thr = __shfl_sync(kFull, list, k - 1);
      uint64_t nxt = 0;
      if (need && last >= thr) nxt = lane_next_below<T, VEC>(rp, c0, c1, last);
      need = nxt != 0 && nxt >= thr;
      last = nxt;
    }
  }
  if (lane < k) s_keys[warp][lane] = list;

  // ---- warp partial sums
  if (LSE) {
    const float e = warp_max_f(e_ref);
    double s = acc > 0.0 ? rescale_pow2(acc, e_ref, e) : 0.0;
    s = warp_sum_d(s);
    if (lane == 0) { s_e[warp] = e; s_s[warp] = s; }
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
  if (warp == 0) {
    const uint64_t merged = lane < k ? s_keys[0][lane] : 0ull;
    const size_t slot = (size_t)row * n_chunks + chunk;
    if (lane < k) keys[slot * k + lane] = merged;
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
}

__global__ void row_stats_finalize_kernel(const ChunkStat* __restrict__ stats,
                                          const uint64_t* __restrict__ keys, long long rows,
                                          int n_chunks, int k, int32_t* __restrict__ topk_token,
                                          float* __restrict__ topk_logit, double* __restrict__ lse) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  double l = 0.0;
  uint64_t key = 0;
  warp_finalize_row(stats + row * n_chunks, keys + row * n_chunks * k, n_chunks, k, lse != nullptr,
                    &l, &key);
  if (lane < k) {
    if (topk_token) topk_token[row * k + lane] = key ? key_index(key) : -1;
    if (topk_logit) topk_logit[row * k + lane] = key ? key_value(key) : -INFINITY;
  }
  if (lse && lane == 0) lse[row] = l;
}

// ------------------------------------------------------------------- host
ChunkPlan plan_chunks(long long rows, int V, int elem_bytes) {
  const int per_vec = 16 / elem_bytes;
  const long long target = 4LL * kNumSMs;
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

size_t row_stats_ws_bytes(long long rows, int V, int elem_bytes, int k) {
  const ChunkPlan p = plan_chunks(rows, V, elem_bytes);
  const size_t n = (size_t)rows * p.n_chunks;
  return align_up(n * sizeof(ChunkStat), 256) + align_up(n * k * sizeof(uint64_t), 256);
}

void row_stats_ws_layout(void* ws, long long rows, int V, int elem_bytes, int k, ChunkStat** stats,
                         uint64_t** keys) {
  const ChunkPlan p = plan_chunks(rows, V, elem_bytes);
  const size_t n = (size_t)rows * p.n_chunks;
  char* base = static_cast<char*>(ws);
  *stats = reinterpret_cast<ChunkStat*>(base);
  *keys = reinterpret_cast<uint64_t*>(base + align_up(n * sizeof(ChunkStat), 256));
}

template <typename T, bool LSE>
static cudaError_t launch_typed(const void* x, long long rows, int V, int k, const ChunkPlan& p,
                                bool vec, ChunkStat* stats, uint64_t* keys, cudaStream_t s) {
  dim3 grid((unsigned)rows, (unsigned)p.n_chunks);
  const T* xp = static_cast<const T*>(x);
  if (vec)
    row_chunk_stats_kernel<T, LSE, true><<<grid, kStatThreads, 0, s>>>(xp, V, p.chunk_elems, k, stats, keys);
  else
    row_chunk_stats_kernel<T, LSE, false><<<grid, kStatThreads, 0, s>>>(xp, V, p.chunk_elems, k, stats, keys);
  return cudaGetLastError();
}

cudaError_t launch_row_chunk_stats(const void* x, int dtype, long long rows, int V, int k, bool lse,
                                   ChunkStat* stats, uint64_t* keys, cudaStream_t s) {
  const int eb = dtype_bytes(dtype);
  const ChunkPlan p = plan_chunks(rows, V, eb);
  const bool vec = ((uintptr_t)x % 16 == 0) && (((size_t)V * eb) % 16 == 0);
  if (dtype == EAGLE_F32)
    return lse ? launch_typed<float, true>(x, rows, V, k, p, vec, stats, keys, s)
               : launch_typed<float, false>(x, rows, V, k, p, vec, stats, keys, s);
  return lse ? launch_typed<__nv_bfloat16, true>(x, rows, V, k, p, vec, stats, keys, s)
             : launch_typed<__nv_bfloat16, false>(x, rows, V, k, p, vec, stats, keys, s);
}

cudaError_t launch_row_stats_finalize(const ChunkStat* stats, const uint64_t* keys, long long rows,
                                      int n_chunks, int k, int32_t* topk_token, float* topk_logit,
                                      double* lse, cudaStream_t s) {
  const int warps = 8;
  const long long blocks = (rows + warps - 1) / warps;
  row_stats_finalize_kernel<<<(unsigned)blocks, warps * 32, 0, s>>>(stats, keys, rows, n_chunks, k,
                                                                    topk_token, topk_logit, lse);
  return cudaGetLastError();
}

}  // namespace eagle
