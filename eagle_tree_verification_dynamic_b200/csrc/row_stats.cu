// Vocabulary sweep over logit rows: the top-k tokens of each row by raw logit
// (ties to the lower token id) and the row's log-sum-exp.  The top-k of the
// draft rows gives the candidate children of a tree node and the log-sum-exp
// turns logits into draft confidences c(x) = exp(l_x) / sum_i exp(l_i)
// ("EAGLE" notes, EAGLE-2 "Well-Calibrated Draft Model"); on target rows the
// same sweep (k = 1) gives the argmax for greedy acceptance and the normaliser
// of p_target for sampling.
//
// Rows whose bytes are 16-byte aligned (the usual case) go through
// row_sweep_kernel: every row is cut into fixed 4 KB chunks, all chunks of all
// rows form one list, and each warp of a persistent grid (up to three CTAs of
// eight warps per SM) takes a contiguous range of it and streams it through
// its own two-stage shared-memory ring (untiled bulk copies, no multicast).
// Per chunk a base-2 scaled fp64 partial of sum exp(logit), reduced over the
// warp in a fixed order, goes to the chunk's slot (so a row's log-sum-exp does
// not depend on the grid).  The top-k of the warp's row segment: for k = 1
// the warp keeps its best (value, id) key; for k > 1 it buffers the keys
// above a threshold and selects by rank, which raises the threshold, so
// almost every chunk is dismissed by one compare of its maximum.  At a segment's end the warp writes its list into the
// segment's last chunk slot and takes the row's ticket; the warp that
// completes a row (nobody waits) merges the row's slots and writes the
// per-row outputs.  Rows that are few and short or long use row_cta_kernel
// (one row per CTA, no cross-SM merge).  Argmax sweeps over many aligned rows
// use row_argmax_kernel, unaligned rows row_stats_kernel: one CTA per (row,
// chunk), 16-byte loads when the rows allow them (scalar otherwise), the same
// ticket merge.
#include <cooperative_groups.h>

#include "eagle_internal.h"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace eagle {

constexpr int kStatThreads = 256;
constexpr int kStatWarps = kStatThreads / 32;
constexpr int kUnroll = 8;

// The M largest (value, id) pairs seen by a lane, sorted by (value desc, id
// asc).  Elements arrive in increasing id, so a new element goes behind any
// equal value; an element it displaces is carried down and goes ahead of an
// equal value with a higher id (it arrived earlier), which keeps the list in
// key order.
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
      if (v > s[p] || (v == s[p] && idx < id[p])) {
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

// ------------------------------------------------- wide argmax (k = 1) sweep
// The per-(row, chunk) layout of row_stats_kernel for argmax sweeps over many
// 16-byte aligned rows, with the streaming loop built for throughput: each
// thread keeps its next four vectors in flight while it works on the current
// four, and every decision off the common path is taken by the whole warp at
// once: a vector is looked at again only when some lane's maximum reaches
// the warp's best value so far, and the warp's log-sum-exp terms share one
// reference exponent (the ceiling of that best value times log2(e)), so no
// lane diverges for a new maximum of its own.
constexpr int kArgPf = 4;  // vectors a thread keeps in flight

template <typename T>
__global__ void __launch_bounds__(kStatThreads, 4)
row_argmax_kernel(const T* __restrict__ x, int V, int chunk_elems, ChunkStat* __restrict__ stats,
                  uint64_t* __restrict__ keys, int* __restrict__ tickets, RowOut out) {
  using namespace sm100;
  constexpr int N = Elem<T>::kPerVec;
  griddep_wait();  // the logits (and this workspace) may belong to the previous kernel
  const long long row = blockIdx.x;
  const int chunk = blockIdx.y, n_chunks = gridDim.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = chunk * chunk_elems;
  const int c1 = min(V, c0 + chunk_elems);
  const uint4* vp = reinterpret_cast<const uint4*>(x + (size_t)row * (size_t)V + c0);
  const int nvec = (c1 - c0) / N;

  uint4 cur[kArgPf], nxt[kArgPf];
  int base = tid;
#pragma unroll
  for (int u = 0; u < kArgPf; ++u) {
    const int vi = base + u * kStatThreads;
    cur[u] = vi < nvec ? ld_stream(vp + vi) : Elem<T>::neg_inf_vec();
  }
  uint64_t best = 0ull;     // the warp's best key (the same in every lane)
  float tv = -INFINITY;     // its value
  float wmax;               // the warp's largest value so far
  float e_ref;              // the warp's reference exponent
  {
    float lm = -INFINITY;
#pragma unroll
    for (int u = 0; u < kArgPf; ++u) lm = fmaxf(lm, Elem<T>::vec_max(cur[u]));
    wmax = warp_max_f(lm);
    e_ref = wmax > -INFINITY ? ceilf(wmax * kLog2eHi) : -INFINITY;
  }
  double acc = 0.0;
  const float2 hi2 = make_float2(kLog2eHi, kLog2eHi), lo2 = make_float2(kLog2eLo, kLog2eLo);
  // the loop test is the warp's (its first lane's): the warp votes inside,
  // so no lane may leave early; a lane past the end holds -inf vectors
  for (; base - lane < nvec; base += kStatThreads * kArgPf) {
    const int nb = base + kStatThreads * kArgPf;
#pragma unroll
    for (int u = 0; u < kArgPf; ++u) {
      const int vi = nb + u * kStatThreads;
      nxt[u] = vi < nvec ? ld_stream(vp + vi) : Elem<T>::neg_inf_vec();
    }
#pragma unroll
    for (int u = 0; u < kArgPf; ++u) {
      const float vmax = Elem<T>::vec_max(cur[u]);
      float f[N];
      Elem<T>::unpack(cur[u], f);
      if (__any_sync(kFull, vmax >= tv)) {  // rare once the warp holds a large value
        uint64_t kl = 0ull;
        if (vmax >= tv) {
          const int idx0 = c0 + (base + u * kStatThreads) * N;
#pragma unroll
          for (int q = 0; q < N; ++q)
            if (f[q] > -INFINITY) kl = umax64(kl, make_key(f[q], idx0 + q));
        }
        best = umax64(best, warp_max_u64(kl));
        if (best) {
          tv = key_value(best);
          wmax = fmaxf(wmax, tv);
          const float e_new = ceilf(wmax * kLog2eHi);
          if (e_new > e_ref) {
            acc = rescale_pow2(acc, e_ref, e_new);
            e_ref = e_new;
          }
        }
      }
      if (e_ref > -INFINITY) {  // until a finite logit arrives every term is exp(-inf) = 0
        const float2 ne = make_float2(-e_ref, -e_ref);
        float2 part = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < N; q += 2) {
          const float2 xq = make_float2(f[q], f[q + 1]);
          const float2 z = ffma2(xq, lo2, ffma2(xq, hi2, ne));
          part = fadd2(part, make_float2(ex2_ftz(z.x), ex2_ftz(z.y)));
        }
        acc += (double)(part.x + part.y);
      }
    }
#pragma unroll
    for (int u = 0; u < kArgPf; ++u) cur[u] = nxt[u];
  }

  griddep_launch_dependents();  // every CTA that reaches here has done its streaming
  __shared__ uint64_t s_best[kStatWarps];
  __shared__ float s_e[kStatWarps];
  __shared__ double s_s[kStatWarps];
  __shared__ int s_last;
  {
    const double sacc = warp_sum_d(acc);  // e_ref is the same in every lane
    if (lane == 0) {
      s_best[warp] = best;
      s_e[warp] = sacc > 0.0 ? e_ref : -INFINITY;
      s_s[warp] = sacc;
    }
  }
  __syncthreads();
  const size_t slot = (size_t)row * n_chunks + chunk;
  if (tid == 0) {
    uint64_t m = 0ull;
    LseAccum a;
    a.init();
    for (int w = 0; w < kStatWarps; ++w) {  // a fixed order
      m = umax64(m, s_best[w]);
      a.add(s_e[w], s_s[w]);
    }
    keys[slot] = m;
    ChunkStat cs;
    cs.e_ref = a.e;
    cs.pad = 0;
    cs.acc = a.s;
    stats[slot] = cs;
    __threadfence();
    s_last = atomicAdd(tickets + row, 1) == n_chunks - 1;
  }
  __syncthreads();
  // ---- the CTA that completes the row merges all of its chunks
  if (!s_last || warp != 0) return;
  __threadfence();
  const ChunkStat* st = stats + (size_t)row * n_chunks;
  const unsigned long long* kk = reinterpret_cast<const unsigned long long*>(keys) + (size_t)row * n_chunks;
  LseAccum a;
  a.init();
  uint64_t m = 0ull;
  for (int c = lane; c < n_chunks; c += 32) {
    a.add(__ldcg(&st[c].e_ref), __ldcg(&st[c].acc));
    m = umax64(m, __ldcg(kk + c));
  }
  const float e = warp_max_f(a.e);
  double sum = a.s > 0.0 ? rescale_pow2(a.s, a.e, e) : 0.0;
  sum = warp_sum_d(sum);
  m = warp_max_u64(m);
  if (lane == 0) {
    if (out.tok) out.tok[row] = m ? key_index(m) : -1;
    if (out.val) out.val[row] = m ? key_value(m) : -INFINITY;
    if (out.lse) out.lse[row] = sum > 0.0 ? kLn2 * ((double)e + log2(sum)) : -INFINITY;
  }
}

// ------------------------------------------------------ chunked TMA sweep
constexpr int kSwWarps = 8;                 // warps per CTA, each streaming its own chunks
constexpr int kSwThreads = kSwWarps * 32;
constexpr int kSwChunkBytes = 4096;         // one chunk = one warp step: 8 16-byte vectors per lane
constexpr int kSwVecPerLane = kSwChunkBytes / 16 / 32;
constexpr int kSwStages = 2;                // each warp's private ring
constexpr int kSwCtasPerSm = 3;
constexpr int kSwCap = 64;                  // candidate keys a warp buffers before it selects

static_assert(kSwCap >= 32 + EAGLE_MAX_TOPK, "after a select one more round of 32 offers must fit");

struct SwShared {
  uint64_t full[kSwWarps][kSwStages];
  uint64_t cand[kSwWarps][kSwCap];
  int abort;
};
constexpr size_t kSwSmemBytes = (size_t)kSwWarps * kSwStages * kSwChunkBytes + sizeof(SwShared);

struct SweepArgs {
  const unsigned char* x;  // row r starts at x + r * row_bytes (16-byte aligned)
  long long nchunks;       // rows * ncpr
  int V, k, ncpr, chunk_elems, row_bytes;
  ChunkStat* stats;  // [rows * ncpr]: log-sum-exp partial of every chunk
  uint64_t* keys;    // [rows * ncpr][k]: a segment's top-k sits in its last chunk's slot, zeros elsewhere
  int* tickets;      // [rows]
  int* status;       // set to 1 when a wait gave up (the outputs are then undefined)
  RowOut out;
};

// The k-th largest of the lanes' values (ties broken by lane), in every lane.
__device__ __forceinline__ float warp_kth_largest(float v, int k) {
  const int lane = threadIdx.x & 31;
  const uint32_t mine = order_bits(v);
  int rank = 0;
#pragma unroll
  for (int d = 1; d < 32; ++d) {
    const int src = (lane + d) & 31;
    const uint32_t o = __shfl_sync(kFull, mine, src);
    rank += (o > mine || (o == mine && src < lane)) ? 1 : 0;
  }
  const unsigned m = __ballot_sync(kFull, rank == k - 1);  // ranks are a permutation of 0..31
  return __shfl_sync(kFull, v, __ffs(m) - 1);
}

// A warp's candidate keys in shared memory.  Invariant: every key offered
// that is above tau is in buf[0, cnt).  select() sorts the buffer by rank
// (the number of larger keys; keys are unique), keeps the best k and, once it
// holds k, raises tau to the k-th.  cnt and tau are warp-uniform.
struct CandBuf {
  uint64_t* buf;
  int cnt;
  uint64_t tau;

  __device__ __forceinline__ void select(int k) {
    constexpr int R = kSwCap / 32;
    const int lane = threadIdx.x & 31;
    __syncwarp();
    uint64_t mine[R];
    int rank[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = lane + 32 * r;
      mine[r] = i < cnt ? buf[i] : 0ull;
      rank[r] = 0;
    }
    for (int j = 0; j < cnt; ++j) {
      const uint64_t o = buf[j];  // the same word in every lane: a broadcast
#pragma unroll
      for (int r = 0; r < R; ++r) rank[r] += o > mine[r] ? 1 : 0;
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (lane + 32 * r < cnt && rank[r] < k) buf[rank[r]] = mine[r];
    __syncwarp();
    if (cnt >= k) {
      cnt = k;
      tau = buf[k - 1];
    }
  }
  // Whole warp; each lane offers one key (0: none).
  __device__ __forceinline__ void offer(uint64_t key, int k) {
    const int lane = threadIdx.x & 31;
    const bool has = key > tau;
    const unsigned m = __ballot_sync(kFull, has);
    if (m == 0u) return;
    if (has) buf[cnt + __popc(m & ((1u << lane) - 1u))] = key;
    cnt += __popc(m);
    if (cnt > kSwCap - 32) select(k);
  }
};

// Element t of a small register array without dynamic indexing (which would
// put the array in local memory).
template <int N>
__device__ __forceinline__ uint64_t pick(const uint64_t (&v)[N], int t) {
  uint64_t r = v[0];
#pragma unroll
  for (int i = 1; i < N; ++i) r = t == i ? v[i] : r;
  return r;
}

// One 4 KB chunk in shared memory (nvec 16-byte vectors; its first element
// has index idx_base in the row), whole warp: returns the chunk's log-sum-exp
// partial (the same in every lane) and folds the chunk into the running top-k
// of the warp's row segment (k = 1: best / best_v, the same in every lane;
// k > 1: cb, with fresh set while the segment has no threshold yet).  Every
// decision that leaves the common path is taken by the whole warp at once
// (the chunk maximum against the segment's best or threshold), so the warp
// never diverges over the vectors that cannot enter the top-k.
template <typename T, bool K1>
__device__ __forceinline__ ChunkStat sweep_chunk(const uint4* sp, int nvec, int idx_base, int k, uint64_t& best,
                                                 float& best_v, CandBuf& cb, bool& fresh) {
  using namespace sm100;
  constexpr int N = Elem<T>::kPerVec;
  const int lane = threadIdx.x & 31;
  // pass 1: the lane's vectors into registers (past the chunk's end: -inf),
  // their maxima, the lane maximum and the chunk maximum
  uint4 raw[kSwVecPerLane];
  float vmx[kSwVecPerLane];
  float lane_max = -INFINITY;
#pragma unroll
  for (int i = 0; i < kSwVecPerLane; ++i) {
    const int v = lane + 32 * i;
    raw[i] = v < nvec ? sp[v] : Elem<T>::neg_inf_vec();
    vmx[i] = Elem<T>::vec_max(raw[i]);
    lane_max = fmaxf(lane_max, vmx[i]);
  }
  const float chunk_max = warp_max_f(lane_max);
  if constexpr (K1) {
    if (chunk_max >= best_v) {  // rare once the segment holds a large value
      uint64_t kl = 0ull;
      if (lane_max >= best_v) {
#pragma unroll
        for (int i = 0; i < kSwVecPerLane; ++i) {
          if (vmx[i] >= best_v) {
            float f[N];
            Elem<T>::unpack(raw[i], f);
#pragma unroll
            for (int q = 0; q < N; ++q)
              if (f[q] > -INFINITY) kl = umax64(kl, make_key(f[q], idx_base + (lane + 32 * i) * N + q));
          }
        }
      }
      best = umax64(best, warp_max_u64(kl));
      best_v = best ? key_value(best) : -INFINITY;
    }
  }
  // pass 2: sum of 2^(x log2(e) - e_ref) with one reference exponent for the
  // chunk, e_ref = ceil(chunk maximum * log2(e)) (every term <= 1; the
  // product x log2(e) formed with log2(e) as a head/tail pair), each vector's
  // terms in fp32, fp64 across vectors and lanes
  const float e_ref = chunk_max > -INFINITY ? ceilf(chunk_max * kLog2eHi) : -INFINITY;
  double acc = 0.0;
  if (e_ref > -INFINITY) {  // else every term is exp(-inf) = 0
    const float2 hi2 = make_float2(kLog2eHi, kLog2eHi), lo2 = make_float2(kLog2eLo, kLog2eLo);
    const float2 ne = make_float2(-e_ref, -e_ref);
#pragma unroll
    for (int i = 0; i < kSwVecPerLane; ++i) {
      float f[N];
      Elem<T>::unpack(raw[i], f);
      float2 part = make_float2(0.f, 0.f);
#pragma unroll
      for (int q = 0; q < N; q += 2) {
        const float2 xq = make_float2(f[q], f[q + 1]);
        const float2 z = ffma2(xq, lo2, ffma2(xq, hi2, ne));
        part = fadd2(part, make_float2(ex2_ftz(z.x), ex2_ftz(z.y)));
      }
      acc += (double)(part.x + part.y);
    }
  }
  // this chunk's log-sum-exp partial: a fixed lane order
  ChunkStat cs;
  cs.e_ref = e_ref;
  cs.pad = 0;
  cs.acc = warp_sum_d(acc);
  if constexpr (!K1) {
    if (fresh) {
      // k lanes hold an element at or above the k-th largest lane maximum
      const float t0 = warp_kth_largest(lane_max, k);
      cb.tau = t0 > -INFINITY ? ((uint64_t)order_bits(t0) << 32) - 1ull : 0ull;
      fresh = false;
    }
    const float tv = cb.tau ? key_value(cb.tau) : -INFINITY;
    if (chunk_max >= tv) {
      // offer this lane's elements above tau, one per lane and round, from
      // the vectors whose maximum reaches tau's value
      uint32_t fl = 0u;
#pragma unroll
      for (int i = 0; i < kSwVecPerLane; ++i)
        if (lane + 32 * i < nvec && vmx[i] >= tv) fl |= 1u << i;
      int cq = 0;  // next element of the lowest flagged vector
      for (;;) {
        uint64_t key = 0ull;
        while (fl != 0u) {
          const int i = __ffs(fl) - 1;
          const int v = lane + 32 * i;
          float f[N];
          Elem<T>::unpack(sp[v], f);
          int nq = N;
#pragma unroll
          for (int q = 0; q < N; ++q) {
            if (key == 0ull && q >= cq && f[q] > -INFINITY) {
              const uint64_t x = make_key(f[q], idx_base + v * N + q);
              if (x > cb.tau) {
                key = x;
                nq = q + 1;
              }
            }
          }
          if (key != 0ull && nq < N) {
            cq = nq;
            break;
          }
          fl &= fl - 1u;
          cq = 0;
          if (key != 0ull) break;
        }
        if (!__any_sync(kFull, key != 0ull)) break;
        cb.offer(key, k);
      }
      // raise the threshold to the k-th key now, so that later chunks of
      // the segment flag fewer vectors
      if (cb.cnt > k) cb.select(k);
    }
  }
  return cs;
}

// Every warp works alone: its contiguous range of the chunk list streams
// through a private two-stage ring (lane 0 issues the bulk copies) and each
// chunk's log-sum-exp partial is a warp reduction written by lane 0.  The
// running top-k of the warp's row segment: with k = 1 the warp keeps its best
// key, looked at again only when a chunk's maximum reaches it; with k > 1 the
// warp buffers candidate keys above a threshold (from the first chunk, the
// k-th largest lane maximum: k elements reach it) and selects by rank after
// every chunk that offered keys, which raises the threshold to the k-th key; a
// vector whose maximum is below the threshold is never looked at again.  At the end of a
// row segment the warp writes its list and takes the row's ticket; the warp
// that completes a row merges it.  No block barrier.
template <typename T, bool K1>
__global__ void __launch_bounds__(kSwThreads, kSwCtasPerSm) row_sweep_kernel(SweepArgs a) {
  using namespace sm100;
  constexpr int N = Elem<T>::kPerVec;
  constexpr int S = kSwStages;
  extern __shared__ __align__(1024) unsigned char sw_smem[];
  SwShared& sh = *reinterpret_cast<SwShared*>(sw_smem + (size_t)kSwWarps * S * kSwChunkBytes);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = K1 ? 1 : a.k;
  const long long W = (long long)gridDim.x * kSwWarps;
  const long long gw = (long long)blockIdx.x * kSwWarps + warp;
  const long long g0 = gw * a.nchunks / W, g1 = (gw + 1) * a.nchunks / W;
  const int nj = (int)(g1 - g0);
  const uint32_t ring = smem_u32(sw_smem + (size_t)warp * S * kSwChunkBytes);
  const unsigned char* ringp = sw_smem + (size_t)warp * S * kSwChunkBytes;
  volatile int* abort = &sh.abort;
  if (threadIdx.x == 0) sh.abort = 0;
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(smem_u32(&sh.full[warp][i]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the logits (and this workspace) may belong to the previous kernel

  // chunk j of this warp: row and chunk-of-row, advanced without divisions
  long long row = g0 / a.ncpr;
  int c = (int)(g0 - row * a.ncpr);
  int issued = 0;
  long long irow = row;
  int ic = c;
  auto issue_next = [&]() {  // lane 0
    const int off = ic * kSwChunkBytes;
    const int bytes = min(kSwChunkBytes, a.row_bytes - off);
    const int st = issued % S;
    const uint32_t fb = smem_u32(&sh.full[warp][st]);
    mbar_arrive_expect_tx(fb, (uint32_t)bytes);
    bulk_load(ring + st * kSwChunkBytes, a.x + (size_t)irow * a.row_bytes + off, (uint32_t)bytes, fb);
    ++issued;
    if (++ic == a.ncpr) { ic = 0; ++irow; }
  };
  if (lane == 0)
    while (issued < nj && issued < S) issue_next();

  uint64_t best = 0ull;      // k = 1: the warp's best key of the segment
  float best_v = -INFINITY;  // and its value
  CandBuf cb;                // k > 1: the warp's candidates of the segment
  cb.buf = sh.cand[warp];
  cb.cnt = 0;
  cb.tau = 0ull;
  bool fresh = true;  // k > 1: the segment has no threshold yet
  long long seg_row = row;
  int seg_c0 = c;

  // end of the segment [seg_c0, c_last] of row seg_row: its top-k into the
  // last chunk's slot (zeros into the others), then the row's ticket
  auto finish_segment = [&](int c_last) {
    const size_t slot0 = (size_t)seg_row * a.ncpr;
    if constexpr (K1) {
      if (lane == 0) a.keys[slot0 + c_last] = best;
      for (int e = lane; e < c_last - seg_c0; e += 32) a.keys[slot0 + seg_c0 + e] = 0ull;
    } else {
      cb.select(k);
      if (lane < k) a.keys[(slot0 + c_last) * k + lane] = lane < cb.cnt ? cb.buf[lane] : 0ull;
      for (int e = lane; e < (c_last - seg_c0) * k; e += 32) a.keys[(slot0 + seg_c0) * k + e] = 0ull;
    }
    __threadfence();
    __syncwarp();
    int last_one = 0;
    if (lane == 0) {
      const int nseg = c_last - seg_c0 + 1;
      last_one = atomicAdd(a.tickets + seg_row, nseg) + nseg == a.ncpr;
    }
    if (!__shfl_sync(kFull, last_one, 0)) return;
    // ---- this warp completed the row: merge its slots.  The chunk partials,
    // the segment lists' k-th keys and the first 256 slot keys are requested
    // together (one round of L2 reads for most rows).
    __threadfence();
    const ChunkStat* st = a.stats + slot0;
    const unsigned long long* kq = reinterpret_cast<const unsigned long long*>(a.keys + slot0 * k);
    const int total = a.ncpr * k;
    uint64_t kv[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int i = lane + 32 * t;
      kv[t] = i < total ? __ldcg(kq + i) : 0ull;
    }
    // k > 1: two lower bounds of the row's k-th key, so that only keys at or
    // above the larger one are merged: the best segment list's k-th key
    // (tk), and the k-th largest of the first two keys of the first 64
    // segment lists (f2: k distinct elements reach it)
    uint64_t tk = 0ull, f2[4];
    if constexpr (!K1) {
      uint64_t v[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = lane + 32 * t;
        v[t] = i < a.ncpr ? __ldcg(kq + (size_t)i * k + (k - 1)) : 0ull;
        const int i2 = (lane >> 1) + 16 * t;
        f2[t] = i2 < a.ncpr ? __ldcg(kq + (size_t)i2 * k + (lane & 1)) : 0ull;
      }
      for (int i0 = 128 + lane; i0 < a.ncpr; i0 += 32) tk = umax64(tk, __ldcg(kq + (size_t)i0 * k + (k - 1)));
#pragma unroll
      for (int t = 0; t < 4; ++t) tk = umax64(tk, v[t]);
    }
    LseAccum la;
    la.init();
    for (int c0 = 0; c0 < a.ncpr; c0 += 64) {  // lane l adds chunks l, l + 32, ... in order
      const int i0 = c0 + lane, i1 = c0 + 32 + lane;
      float e0 = -INFINITY, e1 = -INFINITY;
      double s0 = 0.0, s1 = 0.0;
      if (i0 < a.ncpr) {
        e0 = __ldcg(&st[i0].e_ref);
        s0 = __ldcg(&st[i0].acc);
      }
      if (i1 < a.ncpr) {
        e1 = __ldcg(&st[i1].e_ref);
        s1 = __ldcg(&st[i1].acc);
      }
      la.add(e0, s0);
      la.add(e1, s1);
    }
    const float e = warp_max_f(la.e);
    double sum = la.s > 0.0 ? rescale_pow2(la.s, la.e, e) : 0.0;
    sum = warp_sum_d(sum);
    const double lse = sum > 0.0 ? kLn2 * ((double)e + log2(sum)) : -INFINITY;
    if constexpr (K1) {
      uint64_t m = 0ull;
#pragma unroll
      for (int t = 0; t < 8; ++t) m = umax64(m, kv[t]);
      for (int i0 = 256 + lane; i0 < total; i0 += 32) m = umax64(m, __ldcg(kq + i0));
      m = warp_max_u64(m);
      if (lane == 0) {
        if (a.out.tok) a.out.tok[seg_row] = m ? key_index(m) : -1;
        if (a.out.val) a.out.val[seg_row] = m ? key_value(m) : -INFINITY;
      }
    } else {
      tk = warp_max_u64(tk);
      cb.cnt = 0;
      cb.tau = 0ull;
      // (the offer loops stay rolled: one copy of offer/select in the code, so
      // the finalizer, run once per row on a cold instruction cache, is short)
#pragma unroll 1
      for (int t = 0; t < 4; ++t) cb.offer(pick(f2, t), k);
      cb.select(k);
      const uint64_t bound = umax64(tk, cb.cnt >= k ? cb.buf[k - 1] : 0ull);
      __syncwarp();
      cb.cnt = 0;
      cb.tau = bound ? bound - 1ull : 0ull;  // keys at or above the bound
      for (int e0 = 0; e0 < total; e0 += 256) {
        if (e0 > 0) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int i = e0 + lane + 32 * t;
            kv[t] = i < total ? __ldcg(kq + i) : 0ull;
          }
        }
#pragma unroll 1
        for (int t = 0; t < 8; ++t) cb.offer(pick(kv, t), k);
      }
      cb.select(k);
      if (lane < k) {
        const uint64_t m = lane < cb.cnt ? cb.buf[lane] : 0ull;
        if (a.out.tok) a.out.tok[seg_row * k + lane] = m ? key_index(m) : -1;
        if (a.out.val) a.out.val[seg_row * k + lane] = m ? key_value(m) : -INFINITY;
      }
    }
    if (a.out.lse && lane == 0) a.out.lse[seg_row] = lse;
  };

  for (int j = 0; j < nj; ++j) {
    if (row != seg_row) {  // the range crossed into the next row (at its chunk 0)
      finish_segment(a.ncpr - 1);
      seg_row = row;
      seg_c0 = c;
      best = 0ull;
      best_v = -INFINITY;
      cb.cnt = 0;
      cb.tau = 0ull;
      fresh = true;
    }
    const int st = j % S;
    // a wait that gives up leaves the data undefined (the status word reports it)
    mbar_wait(smem_u32(&sh.full[warp][st]), (j / S) & 1, abort, 2000000000ull, 1000u);
    const int nvec = min(kSwChunkBytes, a.row_bytes - c * kSwChunkBytes) / 16;
    const uint4* sp = reinterpret_cast<const uint4*>(ringp + st * kSwChunkBytes);
    const int idx_base = c * a.chunk_elems;
    const ChunkStat cs = sweep_chunk<T, K1>(sp, nvec, idx_base, k, best, best_v, cb, fresh);
    if (lane == 0) a.stats[(size_t)row * a.ncpr + c] = cs;
    __syncwarp();
    if (lane == 0 && issued < nj && !*abort) {
      fence_proxy_async_smem();  // this stage's reads come before the copy that overwrites it
      issue_next();
    }
    if (++c == a.ncpr) { c = 0; ++row; }
  }
  griddep_launch_dependents();
  if (nj > 0) finish_segment(c == 0 ? a.ncpr - 1 : c - 1);
  if (lane == 0) {
    // every copy issued lands before the CTA may exit
    for (int d = issued > S ? issued - S : 0; d < issued; ++d)
      mbar_wait_drain(smem_u32(&sh.full[warp][d % S]), (d / S) & 1, 200000000ull);
    if (*abort) atomicExch(a.status, 1);
  }
}

// ------------------------------------------------- one row per CTA (few rows)
// When every CTA of the grid is resident at once, each row (or each half of a
// long row: a cluster of two CTAs) is one CTA's work: every warp requests its
// four chunks with one bulk copy at the start, folds them with sweep_chunk,
// and the CTA merges its warps' results in shared memory (the second CTA of a
// pair hands its chunk partials and lists to the first through distributed
// shared memory).  No global tickets, no merging warp on another SM.  The
// chunks and the log-sum-exp combine order are row_sweep_kernel's, so both
// kernels give bit-identical outputs.
constexpr int kRcWarps = 8;
constexpr int kRcThreads = kRcWarps * 32;
constexpr int kRcChunksPerWarp = 4;
constexpr int kRcChunks = kRcWarps * kRcChunksPerWarp;  // 128 KB of row per CTA
constexpr int kRcMaxCluster = 2;

struct RcShared {
  uint64_t full[kRcWarps];
  uint64_t cand[kRcWarps][kSwCap];
  ChunkStat stats[kRcMaxCluster * kRcChunks];               // first CTA: the row's chunk partials
  uint64_t lists[kRcMaxCluster * kRcWarps][EAGLE_MAX_TOPK];  // first CTA: every warp's list
  int abort;
};
constexpr size_t kRcSmemBytes = (size_t)kRcChunks * kSwChunkBytes + sizeof(RcShared);

template <typename T, bool K1>
__global__ void __launch_bounds__(kRcThreads, 1) row_cta_kernel(SweepArgs a, int cl) {
  using namespace sm100;
  extern __shared__ __align__(1024) unsigned char rc_smem[];
  RcShared& sh = *reinterpret_cast<RcShared*>(rc_smem + (size_t)kRcChunks * kSwChunkBytes);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int k = K1 ? 1 : a.k;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = cl > 1 ? (int)cluster.block_rank() : 0;
  const long long row = blockIdx.x / cl;
  const int wc0 = rank * kRcChunks + warp * kRcChunksPerWarp;  // this warp's first chunk of the row
  const int nwc = max(0, min(a.ncpr, wc0 + kRcChunksPerWarp) - wc0);
  const unsigned char* wsm = rc_smem + (size_t)warp * kRcChunksPerWarp * kSwChunkBytes;
  volatile int* abort = &sh.abort;
  if (threadIdx.x == 0) sh.abort = 0;
  if (lane == 0) {
    mbar_init(smem_u32(&sh.full[warp]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();  // the logits (and the outputs) may belong to the previous kernel
  if (lane == 0 && nwc > 0) {
    const int bytes = min(nwc * kSwChunkBytes, a.row_bytes - wc0 * kSwChunkBytes);
    const uint32_t fb = smem_u32(&sh.full[warp]);
    mbar_arrive_expect_tx(fb, (uint32_t)bytes);
    bulk_load(smem_u32(wsm), a.x + (size_t)row * a.row_bytes + (size_t)wc0 * kSwChunkBytes, (uint32_t)bytes, fb);
  }
  // where the first CTA of the row collects the partials and lists
  ChunkStat* stats = sh.stats;
  uint64_t* lists = &sh.lists[0][0];
  if (rank > 0) {
    stats = cluster.map_shared_rank(stats, 0);
    lists = cluster.map_shared_rank(lists, 0);
  }
  uint64_t best = 0ull;
  float best_v = -INFINITY;
  CandBuf cb;
  cb.buf = sh.cand[warp];
  cb.cnt = 0;
  cb.tau = 0ull;
  bool fresh = true;
  if (nwc > 0) {
    // a wait that gives up leaves the data undefined (the status word reports it)
    mbar_wait(smem_u32(&sh.full[warp]), 0, abort, 2000000000ull, 1000u);
    for (int j = 0; j < nwc; ++j) {
      const int c = wc0 + j;
      const int nvec = min(kSwChunkBytes, a.row_bytes - c * kSwChunkBytes) / 16;
      const ChunkStat cs = sweep_chunk<T, K1>(reinterpret_cast<const uint4*>(wsm + (size_t)j * kSwChunkBytes), nvec,
                                              c * a.chunk_elems, k, best, best_v, cb, fresh);
      if (lane == 0) stats[c] = cs;
    }
  }
  uint64_t* my_list = lists + (size_t)(rank * kRcWarps + warp) * EAGLE_MAX_TOPK;
  if constexpr (K1) {
    if (lane == 0) my_list[0] = best;
  } else {
    if (nwc > 0) cb.select(k);
    if (lane < k) my_list[lane] = (nwc > 0 && lane < cb.cnt) ? cb.buf[lane] : 0ull;
  }
  griddep_launch_dependents();
  if (cl > 1) cluster.sync();  // the second CTA's stores land before the first reads them
  else __syncthreads();
  if (rank == 0 && warp == 0) {
    const int nl = cl * kRcWarps;
    LseAccum la;
    la.init();
    for (int c0 = 0; c0 < a.ncpr; c0 += 64) {  // lane l adds chunks l, l + 32, ... in order
      const int i0 = c0 + lane, i1 = c0 + 32 + lane;
      float e0 = -INFINITY, e1 = -INFINITY;
      double s0 = 0.0, s1 = 0.0;
      if (i0 < a.ncpr) {
        e0 = sh.stats[i0].e_ref;
        s0 = sh.stats[i0].acc;
      }
      if (i1 < a.ncpr) {
        e1 = sh.stats[i1].e_ref;
        s1 = sh.stats[i1].acc;
      }
      la.add(e0, s0);
      la.add(e1, s1);
    }
    const float e = warp_max_f(la.e);
    double sum = la.s > 0.0 ? rescale_pow2(la.s, la.e, e) : 0.0;
    sum = warp_sum_d(sum);
    const double lse = sum > 0.0 ? kLn2 * ((double)e + log2(sum)) : -INFINITY;
    if constexpr (K1) {
      const uint64_t m = warp_max_u64(lane < nl ? sh.lists[lane][0] : 0ull);
      if (lane == 0) {
        if (a.out.tok) a.out.tok[row] = m ? key_index(m) : -1;
        if (a.out.val) a.out.val[row] = m ? key_value(m) : -INFINITY;
      }
    } else {
      // the same bounds as the segment merge: the best list's k-th key and the
      // k-th largest of the lists' first two keys; then every key at or above
      uint64_t tk = warp_max_u64(lane < nl ? sh.lists[lane][k - 1] : 0ull);
      cb.cnt = 0;
      cb.tau = 0ull;
      cb.offer((lane >> 1) < nl ? sh.lists[lane >> 1][lane & 1] : 0ull, k);
      cb.select(k);
      const uint64_t bound = umax64(tk, cb.cnt >= k ? cb.buf[k - 1] : 0ull);
      __syncwarp();
      cb.cnt = 0;
      cb.tau = bound ? bound - 1ull : 0ull;
#pragma unroll 1
      for (int e0 = 0; e0 < nl * k; e0 += 32) {
        const int i = e0 + lane;
        cb.offer(i < nl * k ? sh.lists[i / k][i % k] : 0ull, k);
      }
      cb.select(k);
      if (lane < k) {
        const uint64_t m = lane < cb.cnt ? cb.buf[lane] : 0ull;
        if (a.out.tok) a.out.tok[row * k + lane] = m ? key_index(m) : -1;
        if (a.out.val) a.out.val[row * k + lane] = m ? key_value(m) : -INFINITY;
      }
    }
    if (a.out.lse && lane == 0) a.out.lse[row] = lse;
  }
  if (lane == 0) {
    if (nwc > 0 && *abort) mbar_wait_drain(smem_u32(&sh.full[warp]), 0, 200000000ull);  // the copy lands first
    if (*abort) atomicExch(a.status, 1);
  }
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

namespace {

// Chunks per row of the TMA sweep (fixed 16 KB chunks: independent of the row count).
int sweep_chunks_per_row(int V, int elem_bytes) {
  return (int)(((long long)V * elem_bytes + kSwChunkBytes - 1) / kSwChunkBytes);
}

// workspace: [chunk stats rows*nc][chunk keys rows*nc*k][row tickets rows + status word]
// with nc the larger chunk count of the two kernels, so either one fits.
struct RsLayout {
  size_t keys_off, tickets_off, status_off, bytes;
};
RsLayout rs_layout(long long rows, int V, int elem_bytes, int k, long long plan_rows) {
  const ChunkPlan p = plan_chunks(plan_rows > 0 ? plan_rows : rows, V, elem_bytes);
  const int nc_sw = sweep_chunks_per_row(V, elem_bytes);
  const size_t n = (size_t)rows * (size_t)(p.n_chunks > nc_sw ? p.n_chunks : nc_sw);
  RsLayout l;
  l.keys_off = align_up(n * sizeof(ChunkStat), 256);
  l.tickets_off = l.keys_off + align_up(n * k * sizeof(uint64_t), 256);
  l.status_off = l.tickets_off + (size_t)rows * sizeof(int);
  l.bytes = align_up(l.status_off + sizeof(int), 256);
  return l;
}

}  // namespace

size_t row_stats_ws_bytes(long long rows, int V, int elem_bytes, int k, long long plan_rows) {
  return rs_layout(rows, V, elem_bytes, k, plan_rows).bytes;
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

// One row per CTA (a pair for rows over 128 KB) when the whole grid fits on
// the GPU at once and the rows are either short (a row is one warp's work) or
// long (over 128 KB, so an SM would carry a comparable share in the persistent
// kernel anyway); returns false (launching nothing) otherwise.  In between
// (e.g. 51 rows of 32 chunks) the persistent kernel, one chunk a warp over
// every SM, measured faster in spite of its cross-SM merge.
template <typename T, bool K1>
static bool launch_rows(const SweepArgs& a, long long rows, cudaStream_t s, bool pdl, cudaError_t* err) {
  const int cl = (a.ncpr + kRcChunks - 1) / kRcChunks;
  if (cl > kRcMaxCluster || rows * cl > device_sm_count()) return false;
  if (a.ncpr > kRcChunksPerWarp && cl < 2) return false;
  cudaError_t e = ensure_smem_limit((const void*)row_cta_kernel<T, K1>, kRcSmemBytes);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * cl));
    cfg.blockDim = dim3(kRcThreads);
    cfg.dynamicSmemBytes = kRcSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, row_cta_kernel<T, K1>, a, cl);
  }
  *err = e;
  return true;
}

template <typename T, bool K1>
static cudaError_t launch_sweep(const SweepArgs& a, cudaStream_t s, bool pdl) {
  cudaError_t e0;
  if (launch_rows<T, K1>(a, a.nchunks / a.ncpr, s, pdl, &e0)) return e0;
  cudaError_t e = ensure_smem_limit((const void*)row_sweep_kernel<T, K1>, kSwSmemBytes);
  if (e != cudaSuccess) return e;
  // at most three CTAs per SM, and no more warps than chunks (one chunk a
  // warp beat two: a warp's second chunk waited on the first one's work)
  long long C = (long long)device_sm_count() * kSwCtasPerSm;
  const long long want = (a.nchunks + kSwWarps - 1) / kSwWarps;
  if (C > want) C = want;
  return launch_kernel(row_sweep_kernel<T, K1>, dim3((unsigned)C), dim3(kSwThreads), kSwSmemBytes, s, pdl, a);
}

void row_stats_tickets_span(long long rows, int V, int elem_bytes, int k, size_t* off, size_t* bytes) {
  const RsLayout l = rs_layout(rows, V, elem_bytes, k, 0);
  *off = l.tickets_off;
  *bytes = (size_t)rows * sizeof(int) + sizeof(int);  // the tickets and the status word
}

cudaError_t launch_row_stats(const void* x, int dtype, long long rows, int V, int k, bool lse, const RowOut& out,
                             void* ws, cudaStream_t s, bool zero_tickets, bool pdl, long long plan_rows) {
  const int eb = dtype_bytes(dtype);
  const RsLayout l = rs_layout(rows, V, eb, k, plan_rows);
  char* base = static_cast<char*>(ws);
  ChunkStat* stats = reinterpret_cast<ChunkStat*>(base);
  uint64_t* keys = reinterpret_cast<uint64_t*>(base + l.keys_off);
  int* tickets = reinterpret_cast<int*>(base + l.tickets_off);
  if (zero_tickets) {
    cudaError_t e = cudaMemsetAsync(tickets, 0, (size_t)rows * sizeof(int) + sizeof(int), s);
    if (e != cudaSuccess) return e;
  }
  const bool vec = ((uintptr_t)x % 16 == 0) && (((size_t)V * eb) % 16 == 0);
  // a large argmax sweep (k = 1 over many rows) goes to row_argmax_kernel
  // (one CTA per (row, chunk), plain 16-byte loads four vectors ahead): it
  // keeps more bytes in flight per SM than the warps' two-stage rings
  const bool wide_argmax = k == 1 && rows >= 4LL * device_sm_count();
  if (vec && (size_t)V * eb <= 0x7fffffffu && !wide_argmax) {
    // the chunked TMA sweep computes the log-sum-exp always (lse == false only drops the output)
    SweepArgs a;
    a.x = static_cast<const unsigned char*>(x);
    a.ncpr = sweep_chunks_per_row(V, eb);
    a.nchunks = rows * a.ncpr;
    a.V = V;
    a.k = k;
    a.chunk_elems = kSwChunkBytes / eb;
    a.row_bytes = V * eb;
    a.stats = stats;
    a.keys = keys;
    a.tickets = tickets;
    a.status = reinterpret_cast<int*>(base + l.status_off);
    a.out = out;
    if (!lse) a.out.lse = nullptr;
    if (dtype == EAGLE_F32) return k == 1 ? launch_sweep<float, true>(a, s, pdl) : launch_sweep<float, false>(a, s, pdl);
    return k == 1 ? launch_sweep<__nv_bfloat16, true>(a, s, pdl) : launch_sweep<__nv_bfloat16, false>(a, s, pdl);
  }
  const ChunkPlan p = plan_chunks(plan_rows > 0 ? plan_rows : rows, V, eb);
  if (wide_argmax && vec) {
    RowOut o = out;
    if (!lse) o.lse = nullptr;
    const dim3 grid((unsigned)rows, (unsigned)p.n_chunks);
    if (dtype == EAGLE_F32)
      return launch_kernel(row_argmax_kernel<float>, grid, dim3(kStatThreads), 0, s, pdl,
                           static_cast<const float*>(x), V, p.chunk_elems, stats, keys, tickets, o);
    return launch_kernel(row_argmax_kernel<__nv_bfloat16>, grid, dim3(kStatThreads), 0, s, pdl,
                         static_cast<const __nv_bfloat16*>(x), V, p.chunk_elems, stats, keys, tickets, o);
  }
  if (dtype == EAGLE_F32) return launch_t<float>(x, rows, V, k, lse, p, vec, stats, keys, tickets, out, s, pdl);
  return launch_t<__nv_bfloat16>(x, rows, V, k, lse, p, vec, stats, keys, tickets, out, s, pdl);
}

}  // namespace eagle
