// Acceptance walk ("EAGLE" notes, EAGLE-2 "Well-Calibrated Draft Model":
// acceptance min(1, P_target/P_draft), greedy = argmaxes agree; "Что такое
// EAGLE-3", section 4 steps 3-4: on rejection the target samples from the
// adjusted distribution and the longest accepted prefix wins).
//
// Target rows first go through the vocabulary sweep (row_stats.cu, k = 1):
// argmax and log-sum-exp per row.  Then one thread-block cluster per sequence
// walks its tree; a prologue stages every per-node value a decision reads
// (argmax, log-sum-exps, each child's target and draft logit) in shared memory.  Every CTA of the cluster evaluates the same scalar
// decisions from the same data, so they stay in step; the vocabulary-wide
// quantities a decision needs are computed cooperatively, each thread on its
// own contiguous slice of the vocabulary, and combined through distributed
// shared memory in a fixed order (so every CTA sees bit-identical totals):
//   * after a rejection at node j the current target becomes
//     max(0, p - q) / Z.  After r rejections it equals
//     max(0, p - t q) / F(t) with F(t) = sum_x max(0, p(x) - t q(x)),
//     t_0 = 0 (F = 1), t_{r+1} = t_r + F(t_r); one sweep per rejection gives
//     F at the new t;
//   * sampling without replacement also removes each rejected token from q
//     and renormalises it.  With S = the draft mass not yet rejected at j, the
//     current target is still max(0, p - t q) / F(t) (q the unchanged draft
//     row), the ratio gains a factor S and the update becomes
//     t_{r+1} = t_r + F(t_r) / S_r; with replacement S stays 1;
//   * the bonus token is the smallest x whose cumulative weight exceeds
//     u_res * total (inverse CDF), found by a prefix scan over the slices.
// A thread copies its slice of node j's target row and of its draft row into
// shared memory on the first sweep at j; later sweeps at j read only that
// copy (each thread only ever reads its own slice, so no barrier is needed).
#include <cooperative_groups.h>

#include "eagle_internal.h"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace eagle {

constexpr int kAcceptThreads = 256;
constexpr int kAcceptWarps = kAcceptThreads / 32;
constexpr int kCacheBytesPerCta = 64 * 1024;  // both row slices of one CTA
constexpr int kMaxCluster = 16;

template <typename T>
__device__ __forceinline__ float load_logit(const T* p) { return Elem<T>::load(p); }
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__host__ __device__ constexpr int slice_max() { return kCacheBytesPerCta / (2 * kAcceptThreads * (int)sizeof(T)); }

struct SweepArgs {
  Split2 lse_t, lse_d, t;
  bool use_q;  // false: weights are p itself
};

struct AcceptSmem {
  int tok[EAGLE_MAX_NODES];
  int par[EAGLE_MAX_NODES];
  int drow[EAGLE_MAX_NODES + 1];
  int amax[EAGLE_MAX_NODES + 1];       // target argmax of row j
  double lse_t[EAGLE_MAX_NODES + 1];   // target log-sum-exp of row j
  double lse_d[EAGLE_MAX_NODES + 1];   // log-sum-exp of node j's draft row
  double px[EAGLE_MAX_NODES + 1];      // child c: p(x_c) under its parent's target row
  double qx[EAGLE_MAX_NODES + 1];      // child c: q(x_c) under its parent's draft row
  float u_acc[EAGLE_MAX_NODES + 1];    // the walk's uniforms, staged once
  float u_res[EAGLE_MAX_NODES + 1];
  int first_child[EAGLE_MAX_NODES + 1];  // node j's first child in node order (n + 1: none)
  double warp_part[kAcceptWarps];
  double lane_sum[kAcceptThreads];
  double prefix[kAcceptThreads + 1];
  // rejection sweeps: every warp's partial of every CTA ([parity][rank * warps + warp]),
  // and per parity the barrier that completes when all of them have landed
  double xred[2][kMaxCluster * kAcceptWarps];
  uint64_t xbar[2];
};

// Every thread performs the same sequence of reductions, so each keeps its own
// copy of the slot parities.
struct Parity {
  int xs = 0;          // cluster_total / cluster_cta_sum calls so far
  bool stuck = false;  // a cluster_total wait gave up: later ones do not wait
};

// This thread's slice [x0, x1) of the current rows, cached in shared memory.
// Element i of thread t sits at [i * kAcceptThreads + t], so a warp reading
// its threads' i-th elements touches consecutive words (no bank conflicts).
// With fp32 logits the cache holds the probabilities p = exp(l - lse_t) and
// q = exp(l - lse_d) themselves (same size as the logits), computed once when
// a row is loaded, so every later sweep at that node costs two FMAs and a max
// per token; with bf16 logits it holds the logits (half the bytes) and each
// sweep recomputes the exponentials.
template <typename T>
struct Slice {
  static constexpr bool kProbs = sizeof(T) == 4;
  static constexpr int kVec = 16 / (int)sizeof(T);              // elements per 16-byte load
  static constexpr int kMaxLoads = slice_max<T>() / kVec;       // 16-byte loads per full slice
  T* tc;  // target row slice
  T* dc;  // draft row slice
  int x0, x1;
  int slice;    // elements per full slice (a multiple of kVec)
  bool vec_ok;  // rows 16-byte aligned: full slices load as 16-byte vectors
  int cached_t, cached_d;

  __device__ __forceinline__ T& at(T* base, int i) const { return base[(size_t)i * kAcceptThreads + threadIdx.x]; }

  __device__ __forceinline__ T stored(T v, Split2 lse) const {
    if constexpr (kProbs) return exp_minus(to_f(v), lse);
    return v;
  }
  // Copy the slices of up to two rows (src may be null), all loads in flight
  // first; with kProbs each element is stored as its probability under lse0 / lse1.
  __device__ void load2(const T* s0, T* d0, Split2 lse0, const T* s1, T* d1, Split2 lse1) const {
    const int len = x1 - x0;
    if (vec_ok && len == slice) {
      uint4 v0[kMaxLoads], v1[kMaxLoads];
#pragma unroll
      for (int q = 0; q < kMaxLoads; ++q) {
        if (q * kVec < len) {
          if (s0) v0[q] = __ldg(reinterpret_cast<const uint4*>(s0 + x0) + q);
          if (s1) v1[q] = __ldg(reinterpret_cast<const uint4*>(s1 + x0) + q);
        }
      }
#pragma unroll
      for (int q = 0; q < kMaxLoads; ++q) {
        if (q * kVec < len) {
          const T* e0 = reinterpret_cast<const T*>(&v0[q]);
          const T* e1 = reinterpret_cast<const T*>(&v1[q]);
#pragma unroll
          for (int e = 0; e < kVec; ++e) {
            if (s0) at(d0, q * kVec + e) = stored(e0[e], lse0);
            if (s1) at(d1, q * kVec + e) = stored(e1[e], lse1);
          }
        }
      }
    } else {
      for (int i = 0; i < len; ++i) {
        if (s0) at(d0, i) = stored(s0[x0 + i], lse0);
        if (s1) at(d1, i) = stored(s1[x0 + i], lse1);
      }
    }
  }
  // tkey / dkey name the rows (target row j, draft row r), lse_t / lse_d their normalisers.
  __device__ void ensure(const T* trow, int tkey, Split2 lse_t, const T* drow, int dkey, Split2 lse_d) {
    const bool lt = cached_t != tkey, ld = drow && cached_d != dkey;
    if (lt || ld) load2(lt ? trow : nullptr, tc, lse_t, ld ? drow : nullptr, dc, lse_d);
    if (lt) cached_t = tkey;
    if (ld) cached_d = dkey;
  }
  __device__ __forceinline__ float weight(const SweepArgs& a, int i) const {
    float p, q = 0.f;
    if constexpr (kProbs) {
      p = to_f(at(tc, i));
      if (a.use_q) q = to_f(at(dc, i));
    } else {
      p = exp_minus(to_f(at(tc, i)), a.lse_t);
      if (a.use_q) q = exp_minus(to_f(at(dc, i)), a.lse_d);
    }
    if (!a.use_q) return p;
    return fmaxf(0.f, fmaf(-a.t.lo, q, fmaf(-a.t.hi, q, p)));
  }
};



__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_async_f64(uint32_t cluster_addr, double v, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f64 [%0], %1, [%2];" ::"r"(cluster_addr),
               "d"(v), "r"(cluster_bar)
               : "memory");
}

// Cluster-wide total of one double per warp (the same value in all its
// lanes), bit-identical in every thread of every CTA.  Lane r of every warp
// stores the value into rank r's slot [me][warp] with st.async, which counts
// its bytes on rank r's barrier; a CTA waits until all CL * 16 values have
// landed, and each warp adds them in a fixed order (lane l: entries l, l + 32,
// ... in order, then a fixed butterfly).  No cluster barrier: a CTA sends the
// values of call c + 2 (same slots) only after finishing call c + 1, which
// needs every CTA's values of c + 1, sent only after each CTA finished reading
// call c.  A wait that gives up sets *status and the later calls stop waiting.
__device__ double cluster_total(double wv, AcceptSmem& sm, cg::cluster_group& cluster, Parity& par,
                                int* status) {
  const unsigned nb = cluster.num_blocks(), me = cluster.block_rank();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int x = par.xs & 1;
  const uint32_t phase = (uint32_t)(par.xs >> 1) & 1u;
  ++par.xs;
  const uint32_t bar = sm100::smem_u32(&sm.xbar[x]);
  if (threadIdx.x == 0) sm100::mbar_arrive_expect_tx(bar, nb * kAcceptWarps * (uint32_t)sizeof(double));
  if ((unsigned)lane < nb)
    st_async_f64(cluster_map(sm100::smem_u32(&sm.xred[x][me * kAcceptWarps + warp]), lane), wv,
                 cluster_map(bar, lane));
  if (!par.stuck && !sm100::mbar_wait_drain(bar, phase, 100000000ull)) {  // 100 ms
    par.stuck = true;
    if (status) atomicExch(status, 1);
  }
  double acc = 0.0;
  for (int i = lane; i < (int)nb * kAcceptWarps; i += 32) acc += sm.xred[x][i];
  return warp_sum_d(acc);
}

// Cluster-wide total of one double per CTA (the same value in every thread)
// and the sum of the ranks before this one, both bit-identical in every CTA:
// thread r stores the value into rank r's slot [me] with st.async; after the
// barrier every thread adds the CL values in rank order.  Same slots, barriers
// and call sequence as cluster_total.
__device__ double cluster_cta_sum(double cta_value, AcceptSmem& sm, cg::cluster_group& cluster, Parity& par,
                                  int* status, double* prefix_of_rank) {
  const unsigned nb = cluster.num_blocks(), me = cluster.block_rank();
  const int x = par.xs & 1;
  const uint32_t phase = (uint32_t)(par.xs >> 1) & 1u;
  ++par.xs;
  const uint32_t bar = sm100::smem_u32(&sm.xbar[x]);
  if (threadIdx.x == 0) sm100::mbar_arrive_expect_tx(bar, nb * (uint32_t)sizeof(double));
  if (threadIdx.x < nb)
    st_async_f64(cluster_map(sm100::smem_u32(&sm.xred[x][me]), threadIdx.x), cta_value,
                 cluster_map(bar, threadIdx.x));
  if (!par.stuck && !sm100::mbar_wait_drain(bar, phase, 100000000ull)) {  // 100 ms
    par.stuck = true;
    if (status) atomicExch(status, 1);
  }
  double acc = 0.0;
  for (unsigned r = 0; r < nb; ++r) {
    if (r == me) *prefix_of_rank = acc;
    acc += sm.xred[x][r];
  }
  return acc;
}

template <typename T>
__device__ double sweep_total(const Slice<T>& sl, const SweepArgs& a, AcceptSmem& sm, cg::cluster_group& cluster,
                              Parity& par, int* status) {
  float acc = 0.f;  // a slice is <= 32 terms: fp32 within it, fp64 across slices
  for (int i = 0; i < sl.x1 - sl.x0; ++i) acc += sl.weight(a, i);
  return cluster_total(warp_sum_d((double)acc), sm, cluster, par, status);
}

// Inverse CDF over the weights: smallest x with cumsum_x > u * total.  Writes
// the token to *out from the one thread that owns the crossing; returns the
// total weight (every thread).  Each thread sums its slice (<= 32 terms) in
// token order in fp32; the owner's rescan repeats exactly those additions, so
// the crossing lies inside the slice whose interval contains the threshold.
template <typename T>
__device__ double sweep_sample(const Slice<T>& sl, const SweepArgs& a, float u, AcceptSmem& sm,
                               cg::cluster_group& cluster, int32_t* out, Parity& par, int* status) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = sl.x1 - sl.x0;
  float mine_f = 0.f;  // fp32 within the slice; the owner's rescan repeats these additions
  for (int i = 0; i < len; ++i) mine_f += sl.weight(a, i);
  const double mine = (double)mine_f;
  // Block exclusive prefix of the per-thread sums, summed serially (lane order
  // within a warp, then warp order) so the prefixes never decrease and the
  // ownership intervals [prefix[t], prefix[t+1]) tile [0, total) exactly.
  sm.lane_sum[tid] = mine;
  __syncthreads();
  if (lane == 0) {
    double acc = 0.0;
    for (int l = 0; l < 32; ++l) { const double v = sm.lane_sum[tid + l]; sm.prefix[tid + l] = acc; acc += v; }
    sm.warp_part[warp] = acc;
  }
  __syncthreads();
  if (tid == 0) {
    double acc = 0.0;
    for (int w = 0; w < kAcceptWarps; ++w) { const double v = sm.warp_part[w]; sm.warp_part[w] = acc; acc += v; }
    sm.prefix[kAcceptThreads] = acc;
  }
  __syncthreads();
  const double excl = sm.prefix[tid];
  __syncthreads();
  sm.prefix[tid] = sm.warp_part[warp] + excl;
  __syncthreads();
  double my_off = 0.0;
  const double cta_total = sm.prefix[kAcceptThreads];
  const double total = cluster_cta_sum(cta_total, sm, cluster, par, status, &my_off);
  if (total > 0.0) {
    const double thr = (double)u * total;
    const double start = my_off + sm.prefix[tid];
    const double end = my_off + sm.prefix[tid + 1];
    if (start <= thr && thr < end) {
      float run = 0.f;
      int pick = -1, last_nz = -1;
      for (int i = 0; i < len; ++i) {
        const float w = sl.weight(a, i);
        if (w > 0.f) last_nz = sl.x0 + i;
        run += w;
        if (my_off + (sm.prefix[tid] + (double)run) > thr) { pick = sl.x0 + i; break; }
      }
      *out = pick >= 0 ? pick : last_nz;
    }
  }
  return total;
}

template <typename T, bool STOCH>
__global__ void __launch_bounds__(kAcceptThreads, 2)
accept_walk_kernel(const T* __restrict__ tgt, const T* __restrict__ dft, const double* __restrict__ dlse,
                   int R, int V, int n, int depth, const int32_t* __restrict__ row_amax,
                   const double* __restrict__ row_lse, const int32_t* __restrict__ tokens,
                   const int32_t* __restrict__ parents, const int32_t* __restrict__ draft_row,
                   const float* __restrict__ uniforms, int32_t* __restrict__ accepted_len,
                   int32_t* __restrict__ path, int32_t* __restrict__ bonus, int slice, bool vec_ok,
                   bool without_replacement, int* __restrict__ status) {
  __shared__ AcceptSmem sm;
  extern __shared__ __align__(16) unsigned char cache_raw[];
  griddep_wait();  // the target row statistics come from the previous kernel
  griddep_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int b = blockIdx.x / CL;
  const bool leader = cluster.block_rank() == 0 && threadIdx.x == 0;
  const int tid = threadIdx.x;

  Slice<T> sl;
  {
    const int gt = (int)cluster.block_rank() * kAcceptThreads + tid;
    sl.x0 = min(V, gt * slice);
    sl.x1 = min(V, sl.x0 + slice);
    sl.slice = slice;
    sl.vec_ok = vec_ok;
    T* base = reinterpret_cast<T*>(cache_raw);
    sl.tc = base;
    sl.dc = base + (size_t)kAcceptThreads * slice;
    sl.cached_t = -1;
    sl.cached_d = -1;
  }

  // ---- prologue: every value a decision reads, staged in shared memory.
  // Thread i stages node i and child c = i + 1 (n < kAcceptThreads) in three
  // rounds of dependent loads: the child's parent and token; the parent's
  // rows, log-sum-exp and the token's target logit; the token's draft logit.
  static_assert(EAGLE_MAX_NODES < kAcceptThreads, "one node and one child per thread");
  const size_t trow0 = (size_t)b * (n + 1);
  Parity par;
  for (int i = tid; i <= n; i += kAcceptThreads) sm.first_child[i] = n + 1;
  if (STOCH && tid == 0) {
    sm100::mbar_init(sm100::smem_u32(&sm.xbar[0]), 1);
    sm100::mbar_init(sm100::smem_u32(&sm.xbar[1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const int c_me = tid + 1;
  int cpar = -1, ctok = -1;
  if (c_me <= n) {
    cpar = parents[(size_t)b * n + c_me - 1];
    ctok = tokens[(size_t)b * n + c_me - 1];
  }
  int nd_r = -1, nd_amax = 0;
  double nd_lse = 0.0;
  float nd_ua = 0.f, nd_ur = 0.f;
  if (tid <= n) {
    const int r = draft_row[trow0 + tid];
    nd_r = (r >= 0 && r < R) ? r : -1;  // an out-of-range row counts as "not expanded"
    nd_amax = row_amax[trow0 + tid];
    if (STOCH) {
      nd_lse = row_lse[trow0 + tid];
      nd_ua = uniforms[(size_t)b * 2 * (n + 1) + tid];
      nd_ur = uniforms[(size_t)b * 2 * (n + 1) + (n + 1) + tid];
    }
  }
  // second load round: the parent's rows, log-sum-exp and target logit
  const bool cvalid = c_me <= n && cpar >= 0 && cpar <= n && ctok >= 0 && ctok < V;
  double p_logit = 0.0, p_lse = 0.0, nd_lse_d = 0.0;
  int p_row = -1;
  if (STOCH) {
    if (cvalid) {
      p_logit = (double)load_logit(tgt + (trow0 + cpar) * (size_t)V + ctok);
      p_lse = row_lse[trow0 + cpar];
      const int r = draft_row[trow0 + cpar];
      p_row = (r >= 0 && r < R) ? r : -1;
    }
    if (tid <= n && nd_r >= 0) nd_lse_d = dlse[(size_t)b * R + nd_r];
  }
  // third load round: the draft logit
  double q_logit = 0.0, q_lse = 0.0;
  if (STOCH && cvalid && p_row >= 0) {
    q_logit = (double)load_logit(dft + ((size_t)b * R + p_row) * (size_t)V + ctok);
    q_lse = dlse[(size_t)b * R + p_row];
  }
  if (c_me <= n) {
    sm.tok[c_me - 1] = ctok;
    sm.par[c_me - 1] = cpar;
  }
  if (tid <= n) {
    sm.drow[tid] = nd_r;
    sm.amax[tid] = nd_amax;
    if (STOCH) {
      sm.lse_t[tid] = nd_lse;
      sm.lse_d[tid] = nd_r >= 0 ? nd_lse_d : 0.0;
      sm.u_acc[tid] = nd_ua;
      // the residual draw needs u in [0, 1): a NaN or negative u reads as 0 and
      // u >= 1 as the largest float below 1, so the bonus is always written
      sm.u_res[tid] = nd_ur >= 0.f ? fminf(nd_ur, 0x1.fffffep-1f) : 0.f;
    }
  }
  if (STOCH && c_me <= n) {
    // p and q of the child's token under its parent's rows; a token outside
    // the vocabulary has p = q = 0
    sm.px[c_me] = cvalid ? exp(p_logit - p_lse) : 0.0;
    sm.qx[c_me] = (cvalid && p_row >= 0) ? exp(q_logit - q_lse) : 0.0;
  }
  __syncthreads();  // first_child's initial values and the node arrays
  // each node's first child in node order (siblings follow it, in node order)
  if (c_me <= n && cpar >= 0 && cpar <= n) atomicMin(&sm.first_child[cpar], c_me);
  // (with sampling, a cluster barrier: every CTA's sweep barriers are initialised
  // before any CTA stores into them)
  if (STOCH) cluster.sync();
  else __syncthreads();

  int j = 0, plen = 0;
  double lse_t = STOCH ? sm.lse_t[0] : 0.0;
  int amax = sm.amax[0];
  double t = 0.0, F = 1.0, S = 1.0;  // S: draft mass not yet rejected at j (1 with replacement)
  bool rejected_here = false, degenerate = false;

  while (plen < depth) {
    int moved_to = -1;
    if (!STOCH) {
      for (int c = sm.first_child[j]; c <= n; ++c)
        if (sm.par[c - 1] == j && sm.tok[c - 1] == amax) { moved_to = c; break; }
    } else {
      const int r = sm.drow[j];
      const T* trow = tgt + (trow0 + j) * (size_t)V;
      const T* drow = r >= 0 ? dft + ((size_t)b * R + r) * (size_t)V : nullptr;
      const double lse_d = sm.lse_d[j];
      // children of j in node order
      int c = sm.first_child[j];
      while (true) {
        if (c > n || r < 0) break;
        // accept iff u < S rho / (F q), i.e. u F q < S rho (q > 0); a token
        // outside the vocabulary has p = q = 0 and is never accepted
        const double px = sm.px[c], qx = sm.qx[c];
        const double rho = t == 0.0 ? px : fmax(0.0, px - t * qx);
        if (qx > 0.0 && (double)sm.u_acc[c] * (F * qx) < S * rho) { moved_to = c; break; }
        // rejected: the current target becomes max(0, p - t' q) / F(t')
        t += F / S;
        rejected_here = true;
        if (without_replacement) {
          S -= qx;
          if (!(S > 0.0)) { degenerate = true; break; }  // q has nothing left to draw from
        }
        int nc = c + 1;
        while (nc <= n && sm.par[nc - 1] != j) ++nc;
        if (nc <= n) {  // another sibling will be tested: need F(t)
          SweepArgs a;
          a.use_q = true;
          a.lse_t.set(lse_t); a.lse_d.set(lse_d); a.t.set(t);
          sl.ensure(trow, j, a.lse_t, drow, r, a.lse_d);
          F = sweep_total<T>(sl, a, sm, cluster, par, status);
          if (!(F > 0.0)) break;  // p == q left nothing: keep the walk here
        }
        c = nc;
      }
    }
    if (moved_to < 0) break;
    if (leader) path[(size_t)b * depth + plen] = moved_to;
    ++plen;
    j = moved_to;
    t = 0.0;
    F = 1.0;
    S = 1.0;
    rejected_here = false;
    amax = sm.amax[j];
    if (STOCH) lse_t = sm.lse_t[j];
  }

  if (leader) {
    accepted_len[b] = plen;
    for (int i = plen; i < depth; ++i) path[(size_t)b * depth + i] = -1;
  }
  if (!STOCH) {
    if (leader) bonus[b] = amax;
    return;
  }
  if (degenerate) {
    if (leader) bonus[b] = amax;
    cluster.sync();
    return;
  }
  const int r = sm.drow[j];
  const bool use_q = rejected_here && r >= 0;
  SweepArgs a;
  a.use_q = use_q;
  a.lse_t.set(lse_t);
  a.lse_d.set(sm.lse_d[j]);
  a.t.set(t);
  sl.ensure(tgt + (trow0 + j) * (size_t)V, j, a.lse_t, use_q ? dft + ((size_t)b * R + r) * (size_t)V : nullptr, r,
            a.lse_d);
  const double total = sweep_sample<T>(sl, a, sm.u_res[j], sm, cluster, bonus + b, par, status);
  if (!(total > 0.0) && leader) bonus[b] = amax;  // nothing left to sample from
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------------------------- host
// workspace: [row sweep workspace][row argmax rows int32][row lse rows double]
size_t accept_ws_bytes(int B, int n, int V, int dtype) {
  const long long rows = (long long)B * (n + 1);
  return row_stats_ws_bytes(rows, V, dtype_bytes(dtype), 1) + align_up((size_t)rows * sizeof(int32_t), 256) +
         align_up((size_t)rows * sizeof(double), 256);
}

int accept_max_vocab(int dtype) {
  const int sm = dtype == EAGLE_F32 ? slice_max<float>() : slice_max<__nv_bfloat16>();
  return kMaxCluster * kAcceptThreads * sm;
}

template <typename T, bool STOCH>
static cudaError_t launch_walk(const void* tgt, const void* dft, const double* dlse, int R, int V, int n,
                               int depth, const int32_t* row_amax, const double* row_lse,
                               const int32_t* tokens, const int32_t* parents, const int32_t* draft_row,
                               const float* uniforms, int B, int32_t* acc_len, int32_t* path,
                               int32_t* bonus, cudaStream_t s, bool pdl, bool without_replacement, int* status) {
  int cl = 1, slice = 0;
  size_t dyn = 0;
  const bool vec_ok = (((uintptr_t)tgt | (uintptr_t)dft) % 16 == 0) && ((size_t)V * sizeof(T)) % 16 == 0;
  if (STOCH) {
    const int per_cta = kAcceptThreads * slice_max<T>();
    cl = (V + per_cta - 1) / per_cta;
    if (cl < 1) cl = 1;
    // with few sequences, spread each walk over more CTAs (up to 16, two per
    // SM): smaller slices load and sweep faster, and the walk is latency-bound
    const int spare = 2 * device_sm_count() / (B > 0 ? B : 1);
    const int want = spare < kMaxCluster ? spare : kMaxCluster;
    if (cl < want) cl = want;
    slice = (V + cl * kAcceptThreads - 1) / (cl * kAcceptThreads);
    constexpr int kVec = 16 / (int)sizeof(T);
    slice = (slice + kVec - 1) / kVec * kVec;  // <= slice_max, itself a multiple of kVec
    dyn = (size_t)2 * kAcceptThreads * slice * sizeof(T);
    cudaError_t e = ensure_smem_limit((const void*)accept_walk_kernel<T, STOCH>, dyn + sizeof(AcceptSmem));
    if (e != cudaSuccess) return e;
    if (cl > 8) {
      static bool np_set = false;
      if (!np_set) {
        e = cudaFuncSetAttribute(accept_walk_kernel<T, STOCH>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        np_set = true;
      }
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(B * cl));
  cfg.blockDim = dim3(kAcceptThreads);
  cfg.dynamicSmemBytes = dyn;
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
  return cudaLaunchKernelEx(&cfg, accept_walk_kernel<T, STOCH>, static_cast<const T*>(tgt),
                            static_cast<const T*>(dft), dlse, R, V, n, depth, row_amax, row_lse, tokens,
                            parents, draft_row, uniforms, acc_len, path, bonus, slice, vec_ok,
                            without_replacement, status);
}

cudaError_t launch_accept(const void* tgt, int tdtype, const void* dft, int ddtype, const double* dlse,
                          int R, const int32_t* tokens, const int32_t* parents, const int32_t* draft_row,
                          const float* uniforms, int B, int n, int V, int depth, int32_t* accepted_len,
                          int32_t* path, int32_t* bonus, void* ws, cudaStream_t s, bool zero_tickets, bool pdl,
                          bool without_replacement) {
  const long long rows = (long long)B * (n + 1);
  const bool stoch = uniforms != nullptr;
  char* tail = static_cast<char*>(ws) + row_stats_ws_bytes(rows, V, dtype_bytes(tdtype), 1);
  int32_t* row_amax = reinterpret_cast<int32_t*>(tail);
  double* row_lse = reinterpret_cast<double*>(tail + align_up((size_t)rows * sizeof(int32_t), 256));
  RowOut ro;
  ro.tok = row_amax;
  ro.val = nullptr;
  ro.lse = stoch ? row_lse : nullptr;
  cudaError_t e = launch_row_stats(tgt, tdtype, rows, V, 1, stoch, ro, ws, s, zero_tickets, pdl);
  if (e != cudaSuccess) return e;
  (void)ddtype;  // the draft rows share the target's element type (checked by the caller)
  // the sweep's device status word (after its row tickets): the walk reports a
  // wait that gave up there too
  size_t t_off = 0, t_bytes = 0;
  row_stats_tickets_span(rows, V, dtype_bytes(tdtype), 1, &t_off, &t_bytes);
  int* status = reinterpret_cast<int*>(static_cast<char*>(ws) + t_off + (size_t)rows * sizeof(int));
  if (tdtype == EAGLE_F32)
    return stoch ? launch_walk<float, true>(tgt, dft, dlse, R, V, n, depth, row_amax, row_lse, tokens, parents,
                                            draft_row, uniforms, B, accepted_len, path, bonus, s, pdl,
                                            without_replacement, status)
                 : launch_walk<float, false>(tgt, dft, dlse, R, V, n, depth, row_amax, row_lse, tokens,
                                             parents, draft_row, uniforms, B, accepted_len, path, bonus, s, pdl, false,
                                             status);
  return stoch ? launch_walk<__nv_bfloat16, true>(tgt, dft, dlse, R, V, n, depth, row_amax, row_lse, tokens,
                                                  parents, draft_row, uniforms, B, accepted_len, path, bonus, s, pdl,
                                                  without_replacement, status)
               : launch_walk<__nv_bfloat16, false>(tgt, dft, dlse, R, V, n, depth, row_amax, row_lse, tokens,
                                                   parents, draft_row, uniforms, B, accepted_len, path, bonus, s,
                                                   pdl, false, status);
}

}  // namespace eagle
