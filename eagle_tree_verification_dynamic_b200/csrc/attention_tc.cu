// Tree-masked split-KV attention on the 5th-generation tensor cores
// ("Tree Attention" verification of the EAGLE notes, "3.Verify"; mask
// semantics of "Технический анализ EAGLE-4", section "Деревья проверки
// EAGLE-4 и утилита управления").
//
// One CTA = (key split, KV head g, sequence b, group of 128 query rows).  The
// 128 rows are the (node, head-in-group) pairs of head g, so every K/V tile
// staged in shared memory serves all tree queries of the GQA group at once.
//   warp 0      TMA producer: K and V tiles of 64 keys into a 2-stage ring
//               (128-byte swizzle, no multicast); also allocates TMEM
//   warp 1      one thread issues tcgen05.mma: S = Q K^T into one of two TMEM
//               buffers (the next tile's S is computed while this tile's
//               softmax runs), then O += P V into TMEM (fp32 accumulators,
//               bf16 operands)
//   warps 2-5   softmax: thread r owns TMEM lane r = query row r; reads its S
//               row, applies the prefix range / window / tree bitmask, keeps a
//               running reference max (re-based only when it grows by > 8 in
//               log2 units, then O and the row sum are rescaled in TMEM),
//               writes P = 2^(x - m) as bf16 into swizzled shared memory
// The last split column handles the n tree keys, visible per the ancestor
// bitmask.  The splits of one (sequence, KV head, row group) form one thread
// block cluster: each CTA parks its normalised partial output and log-sum-exp
// in its own shared memory, then every CTA combines a slice of the rows from
// all partials through distributed shared memory and writes bf16 output
// (out = sum_s e^{lse_s - M} O_s / sum_s e^{lse_s - M}).  No partial leaves the
// chip and no second kernel runs.
//
// Every mbarrier wait is bounded (about 2 s of wall time); a timeout sets an
// abort flag that ends all roles, records an error word in the workspace
// header and still frees the TMEM columns.  No path returns early: every CTA
// reaches both cluster barriers of the combine.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "eagle_internal.h"
#include "sm100_ptx.cuh"

namespace cg = cooperative_groups;

namespace eagle {

using namespace sm100;

constexpr int kTcThreads = 192;  // 6 warps
constexpr int kBN = 64;          // keys per tile
constexpr int kStages = 2;
constexpr int kRowsPerCta = 128;

template <int D>
struct TcLayout {
  static constexpr int kAtoms = D / 64;                 // 128-byte column atoms along D
  static constexpr int kQBytes = kAtoms * 128 * 128;    // 128 rows
  static constexpr int kPBytes = 128 * 128;             // 128 rows x 64 keys bf16
  static constexpr int kKVAtomBytes = kBN * 128;        // 64 keys x 128 B
  static constexpr int kKBytes = kAtoms * kKVAtomBytes;
  static constexpr int kStageBytes = 2 * kKBytes;       // K + V
  static constexpr int kQOff = 0;
  static constexpr int kPOff = kQOff + kQBytes;
  static constexpr int kStageOff = kPOff + kPBytes;
  static constexpr int kBarOff = kStageOff + kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 128;  // + barriers (base is 1024-aligned, checked)
  static constexpr uint32_t kTmemCols = 256;  // S double buffer (2 x 64) + O (D)
  static constexpr uint32_t kColS = 0;        // S buffer b at column 64 * b
  static constexpr uint32_t kColO = 128;
};

struct TcBars {
  uint64_t q_full;
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full;
  uint64_t pv_done;
  uint64_t mma_idle;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(TcBars) <= 128, "barrier block");

struct TcParams {
  const __nv_bfloat16* q;
  const int32_t* plen;
  const uint64_t* mask;
  const int32_t* pos;
  __nv_bfloat16* out;
  int* err;
  int Lmax, n, Hq, Hkv, window, n_splits, chunk, row_groups;
  int q_by_tma;      // 1: Q rows arrive by TMA (G divides 128), 0: gathered by the threads
  float scale_log2;  // softmax scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_vt,
               const __grid_constant__ CUtensorMap tm_q, const TcParams p) {
  using Lay = TcLayout<D>;
  extern __shared__ __align__(1024) unsigned char smem[];
  TcBars* bars = reinterpret_cast<TcBars*>(smem + Lay::kBarOff);
  const uint32_t s_base = smem_u32(smem);
  const bool aligned = (s_base & 1023u) == 0;  // the swizzled tiles need 1024-byte alignment
  cg::cluster_group cluster = cg::this_cluster();

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, g = blockIdx.y;
  const int b = blockIdx.z / p.row_groups, rg = blockIdx.z % p.row_groups;
  const int B = gridDim.z / p.row_groups;
  const int G = p.Hq / p.Hkv;
  const int rows = p.n * G;
  const int row0 = rg * kRowsPerCta;
  const int L = min(max(p.plen[b], 0), p.Lmax);
  const bool tree = (s == p.n_splits);
  int k0, k1;
  if (!tree) {
    const int lo = p.window > 0 ? max(0, L - p.window + 1) : 0;
    k0 = lo + s * p.chunk;
    k1 = min(L, k0 + p.chunk);
  } else {
    k0 = 0;
    k1 = p.n;
  }
  const int ntiles = k1 > k0 ? (k1 - k0 + kBN - 1) / kBN : 0;

  // softmax thread -> query row
  const bool is_soft = warp >= 2;
  const int quad = warp & 3;
  const int r_local = quad * 32 + lane;   // TMEM lane = row within the tile
  const int r_glob = row0 + r_local;
  const bool row_ok = is_soft && r_glob < rows;
  const int qi = row_ok ? r_glob / G : 0;
  const int qh = row_ok ? g * G + r_glob % G : 0;

  // A CTA with nothing to do (no visible key in its split, or a misaligned
  // shared-memory base) still takes part in the cluster's combine below.
  const bool work = aligned && ntiles > 0;
  if (!aligned && tid == 0) atomicExch(p.err, 2);
  float m_used = -INFINITY, l = 0.f;  // softmax threads: reference max (scaled, log2) and row sum
  bool final_ok = false;              // softmax threads: O in TMEM is complete for this row
  uint32_t tmem = 0;
  volatile int* abort = &bars->abort;

  if (work) {
  // ---- set-up: barriers, TMEM, Q tile
  if (tid == 0) {
    mbar_init(smem_u32(&bars->q_full), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    mbar_init(smem_u32(&bars->s_full[0]), 1);
    mbar_init(smem_u32(&bars->s_full[1]), 1);
    // only warps holding at least one real query row write P and arrive; a warp
    // of padding rows never arrives (it could otherwise run a tile ahead and
    // complete a phase early, since S is double-buffered)
    const int live_warps = min(4, (rows - row0 + 31) / 32);
    mbar_init(smem_u32(&bars->p_full), 32 * live_warps);
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->mma_idle), 1);
    bars->abort = 0;
    fence_mbar_init();
    if (p.q_by_tma) {
      // the 128 query rows of this tile = (node, head-in-group) pairs: a box of
      // {64 dims, G heads, 128/G nodes} of q viewed as [B*n][Hq][D]
      const uint32_t qb = smem_u32(&bars->q_full);
      mbar_arrive_expect_tx(qb, Lay::kQBytes);
      const int rows_i = kRowsPerCta / G;
      for (int a = 0; a < Lay::kAtoms; ++a)
        tma_load_3d(s_base + Lay::kQOff + a * 16384, &tm_q, a * 64, g * G, b * p.n + rg * rows_i, qb);
    }
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_kt);
    prefetch_tmap(&tm_vt);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), Lay::kTmemCols);
    tmem_relinquish();
  }
  if (!p.q_by_tma) {
    // Q rows (bf16) -> 128-byte swizzled K-major tile; all loads issued first
    constexpr int kVec = 128 * Lay::kAtoms * 8;
    constexpr int kPer = (kVec + kTcThreads - 1) / kTcThreads;
    uint4 v[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = tid + t * kTcThreads;
      v[t] = make_uint4(0, 0, 0, 0);
      if (e < kVec) {
        const int r = e / (Lay::kAtoms * 8), a = (e / 8) % Lay::kAtoms, c = e % 8;
        const int rr = row0 + r;
        if (rr < rows) {
          const int i = rr / G, h = g * G + rr % G;
          v[t] = *reinterpret_cast<const uint4*>(p.q + (((size_t)b * p.n + i) * p.Hq + h) * D + a * 64 + c * 8);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = tid + t * kTcThreads;
      if (e < kVec) {
        const int r = e / (Lay::kAtoms * 8), a = (e / 8) % Lay::kAtoms, c = e % 8;
        *reinterpret_cast<uint4*>(smem + Lay::kQOff + a * 16384 + r * 128 + ((c ^ (r & 7)) << 4)) = v[t];
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(smem_u32(&bars->empty[st]), ((j / kStages) - 1) & 1, abort)) break;
        const uint32_t fb = smem_u32(&bars->full[st]);
        mbar_arrive_expect_tx(fb, Lay::kStageBytes);
        const uint32_t kdst = s_base + Lay::kStageOff + st * Lay::kStageBytes;
        const uint32_t vdst = kdst + Lay::kKBytes;
        const int key0 = k0 + j * kBN;
        for (int a = 0; a < Lay::kAtoms; ++a) {
          if (!tree) {
            const int y = (b * p.Hkv + g) * p.Lmax + key0;
            tma_load_2d(kdst + a * Lay::kKVAtomBytes, &tm_k, a * 64, y, fb);
            tma_load_2d(vdst + a * Lay::kKVAtomBytes, &tm_v, a * 64, y, fb);
          } else {
            tma_load_3d(kdst + a * Lay::kKVAtomBytes, &tm_kt, a * 64, g, b * p.n + key0, fb);
            tma_load_3d(vdst + a * Lay::kKVAtomBytes, &tm_vt, a * 64, g, b * p.n + key0, fb);
          }
        }
        ++issued;
      }
      // drain: wait until every issued copy has landed before the CTA may exit
      if (p.q_by_tma) mbar_wait_drain(smem_u32(&bars->q_full), 0, 200000000ull);
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        mbar_wait_drain(smem_u32(&bars->full[j % kStages]), (j / kStages) & 1, 200000000ull);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, kBN, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t t_s = tmem + Lay::kColS, t_o = tmem + Lay::kColO;
      const uint32_t q_addr = s_base + Lay::kQOff;
      const uint32_t p_addr = s_base + Lay::kPOff;
      const bool q_ok = !p.q_by_tma || mbar_wait(smem_u32(&bars->q_full), 0, abort);
      // S = Q K_j^T into S buffer (j & 1)
      auto issue_qk = [&](int jj) -> bool {
        const int st = jj % kStages;
        if (!mbar_wait(smem_u32(&bars->full[st]), (jj / kStages) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t k_addr = s_base + Lay::kStageOff + st * Lay::kStageBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk % 4) * 32;
          const uint64_t da = smem_desc(q_addr + (kk / 4) * 16384 + off, 16, 1024, kSwizzle128B);
          const uint64_t db = smem_desc(k_addr + (kk / 4) * Lay::kKVAtomBytes + off, 16, 1024, kSwizzle128B);
          mma_bf16_ss(t_s + (uint32_t)((jj & 1) * kBN), da, db, id_qk, kk > 0);
        }
        mma_commit(smem_u32(&bars->s_full[jj & 1]));
        return true;
      };
      bool ok = q_ok && issue_qk(0);
      int next_qk = 1;  // S has two buffers: QK^T runs at most one tile ahead of PV
      for (int j = 0; j < ntiles && ok; ++j) {
        // issue whichever is ready first: the next tile's QK^T (its K landed) or
        // this tile's PV (its P is written)
        const uint32_t pb = smem_u32(&bars->p_full);
        uint64_t t0 = 0;
        for (uint32_t it = 0;; ++it) {
          if (next_qk < ntiles && next_qk <= j + 1 &&
              mbar_try_wait(smem_u32(&bars->full[next_qk % kStages]), (next_qk / kStages) & 1)) {
            if (!issue_qk(next_qk)) { ok = false; break; }
            ++next_qk;
          }
          if (mbar_try_wait(pb, j & 1)) break;
          if ((it & 15u) == 15u) {
            if (*abort) { ok = false; break; }
            const uint64_t now = globaltimer();
            if (t0 == 0) t0 = now;
            else if (now - t0 > 2000000000ull) { *abort = 1; ok = false; break; }
          }
        }
        if (!ok) break;
        tc_fence_after();
        const int st = j % kStages;
        const uint32_t v_addr = s_base + Lay::kStageOff + st * Lay::kStageBytes + Lay::kKBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t da = smem_desc(p_addr + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t db = smem_desc(v_addr + kk * 2048, Lay::kKVAtomBytes, 1024, kSwizzle128B);
          mma_bf16_ss(t_o, da, db, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->empty[st]));
        mma_commit(smem_u32(&bars->pv_done));
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(smem_u32(&bars->mma_idle));
      mbar_wait_drain(smem_u32(&bars->mma_idle), 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + Lay::kColS;
    const uint32_t t_o = tmem + lane_base + Lay::kColO;
    // a warp whose 32 rows are all padding only keeps the barrier protocol going
    const bool warp_live = row0 + quad * 32 < rows;
    const int qpos = (row_ok && p.window > 0) ? p.pos[(size_t)b * p.n + qi] : 0;
    const int win_lo = qpos - p.window + 1;
    uint64_t mw0 = 0, mw1 = 0;
    if (row_ok && tree) {
      mw0 = p.mask[((size_t)b * p.n + qi) * 2];
      mw1 = p.mask[((size_t)b * p.n + qi) * 2 + 1];
    }
    const float sl2 = p.scale_log2;
    bool ok = true;
    unsigned char* prow = smem + Lay::kPOff + r_local * 128;
    for (int j = 0; j < ntiles && ok; ++j) {
      if (!warp_live) break;  // padding rows: nothing to compute, nothing to signal
      if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->s_full[j & 1]), (j >> 1) & 1, abort))) { ok = false; break; }
      tc_fence_after();
      float x[kBN];
      tmem_ld32(t_s + (uint32_t)((j & 1) * kBN), x);
      tmem_ld32(t_s + (uint32_t)((j & 1) * kBN + 32), x + 32);
      tmem_wait_ld();
      const int key0 = k0 + j * kBN;
      float mx = -INFINITY;
      if (tree || p.window > 0 || key0 + kBN > k1) {  // edge tiles: per-key visibility
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          const int kidx = key0 + c;
          bool vis = row_ok && kidx < k1;
          if (vis && tree) {
            vis = ((kidx < 64 ? mw0 >> kidx : mw1 >> (kidx - 64)) & 1ull) != 0;
            if (vis && p.window > 0) vis = p.pos[(size_t)b * p.n + kidx] >= win_lo;
          } else if (vis && p.window > 0) {
            vis = kidx >= win_lo;
          }
          x[c] = vis ? x[c] : -INFINITY;
          mx = fmaxf(mx, x[c]);
        }
      } else {  // interior prefix tile: every key visible
#pragma unroll
        for (int c = 0; c < kBN; ++c) mx = fmaxf(mx, x[c]);
      }
      mx *= sl2;  // scale > 0 keeps the order
      // PV(j-1) must be complete before P is overwritten or O is rescaled
      if (j > 0) {
        if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->pv_done), (j - 1) & 1, abort))) { ok = false; break; }
        tc_fence_after();
      }
      const bool rebase = mx > m_used + 8.f;
      if (__any_sync(kFull, rebase && j > 0 && l > 0.f)) {
        const float f = (rebase && l > 0.f) ? ex2(m_used - mx) : 1.f;
        for (int c0 = 0; c0 < D; c0 += 32) {
          float o[32];
          tmem_ld32(t_o + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] *= f;
          tmem_st32(t_o + c0, o);
        }
        tmem_wait_st();
        l *= f;
      }
      if (rebase) m_used = mx;
      const float neg_m = m_used > -INFINITY ? -m_used : 0.f;  // no visible key yet: every x is -inf
      float sum = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < kBN / 8; ++c8) {
        uint32_t packed[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float a = ex2(fmaf(x[c8 * 8 + 2 * t], sl2, neg_m));
          const float bb = ex2(fmaf(x[c8 * 8 + 2 * t + 1], sl2, neg_m));
          sum += a + bb;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, bb);
          packed[t] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        *reinterpret_cast<uint4*>(prow + ((c8 ^ (r_local & 7)) << 4)) =
            make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
      l += sum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->p_full));
    }
    final_ok = ok && warp_live &&
               __all_sync(kFull, mbar_wait(smem_u32(&bars->pv_done), (ntiles - 1) & 1, abort));
  }
  }  // work

  // ---- park this split's normalised partial (O rows, log-sum-exp) in shared
  // memory: the K/V stages hold O (row r: D floats, 16-byte chunks XOR-swizzled
  // by r), the P buffer holds the 128 log-sum-exps.  All TMA copies and MMAs of
  // this CTA have drained before the barrier below.
  float* o_part = reinterpret_cast<float*>(smem + Lay::kStageOff);
  float* lse_part = reinterpret_cast<float*>(smem + Lay::kPOff);
  constexpr int kChunks = D / 4;  // 16-byte chunks per O row
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp >= 2) {
    float lse_r = -INFINITY;
    if (final_ok) {  // warp-uniform
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const uint32_t t_o = tmem + ((uint32_t)(quad * 32) << 16) + Lay::kColO;
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tmem_ld32(t_o + c0, o);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int c = (c0 >> 2) + t;
          *reinterpret_cast<float4*>(o_part + r_local * D + ((c ^ (r_local & (kChunks - 1))) << 2)) =
              make_float4(o[4 * t] * inv, o[4 * t + 1] * inv, o[4 * t + 2] * inv, o[4 * t + 3] * inv);
        }
      }
      if (row_ok && l > 0.f) lse_r = (m_used + __log2f(l)) * (float)kLn2;
    }
    lse_part[r_local] = lse_r;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (work && *abort && tid == 0) atomicExch(p.err, 1);
  if (work && warp == 0) tmem_dealloc(tmem, Lay::kTmemCols);

  // ---- combine the splits of this (sequence, KV head, row group) across the
  // cluster: rank cr reduces a slice of the rows, reading every split's
  // partial through distributed shared memory, and writes bf16 output
  //   out = sum_s e^{lse_s - M} O_s / sum_s e^{lse_s - M}
  cluster.sync();
  {
    const int CS = (int)cluster.num_blocks(), cr = (int)cluster.block_rank();
    const int valid = min(kRowsPerCta, rows - row0);
    const int per = (valid + CS - 1) / CS;
    const int r_end = min(valid, (cr + 1) * per);
    constexpr int DPL = D / 32;  // output dims per lane
    for (int r = cr * per + warp; r < r_end; r += kTcThreads / 32) {
      const float ls = lane < CS ? *cluster.map_shared_rank(lse_part + r, lane) : -INFINITY;
      const float M = warp_max_f(ls);
      const float w = (lane < CS && ls > -INFINITY) ? __expf(ls - M) : 0.f;
      const float wsum = warp_sum_f(w);
      float acc[DPL];
#pragma unroll
      for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
      const int c = (lane * DPL) >> 2;  // this lane's 16-byte chunk
      const int within = (lane * DPL) & 3;
      const int off = r * D + ((c ^ (r & (kChunks - 1))) << 2) + within;
      for (int sp = 0; sp < CS; ++sp) {
        const float ws = __shfl_sync(kFull, w, sp);
        if (ws == 0.f) continue;
        const float* src = cluster.map_shared_rank(o_part, sp) + off;
#pragma unroll
        for (int t = 0; t < DPL; ++t) acc[t] = fmaf(ws, src[t], acc[t]);
      }
      const int rg_row = row0 + r;
      const int i = rg_row / G, h = g * G + rg_row % G;
      __nv_bfloat16* dst = p.out + (((size_t)b * p.n + i) * p.Hq + h) * D + lane * DPL;
      const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
      for (int t = 0; t < DPL; t += 2)
        *reinterpret_cast<__nv_bfloat162*>(dst + t) = __floats2bfloat162_rn(acc[t] * inv, acc[t + 1] * inv);
    }
  }
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------------------------- host
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor map with a 64-element x 64-row box and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int attention_row_groups(int n, int Hq, int Hkv) {
  const int rows = n * (Hq / Hkv);
  return (rows + kRowsPerCta - 1) / kRowsPerCta;
}

template <int D>
static cudaError_t launch_tc(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                             const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                             int n, int Hq, int Hkv, int window, float scale, const AttnPlan& plan, void* out,
                             int* err, cudaStream_t s) {
  CUtensorMap mk, mv, mkt, mvt;
  const int Lrows = Lmax > 0 ? Lmax : 1;
  const void* kbase = Lmax > 0 ? kc : kt;  // any valid address when the cache is empty
  const void* vbase = Lmax > 0 ? vc : vt;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)B * Hkv * Lrows};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kBN};
    const cuuint64_t dims0[2] = {(cuuint64_t)D, (cuuint64_t)(Lmax > 0 ? (cuuint64_t)B * Hkv * Lrows : 1)};
    if (!make_map(&mk, kbase, 2, Lmax > 0 ? dims : dims0, str, box) ||
        !make_map(&mv, vbase, 2, Lmax > 0 ? dims : dims0, str, box))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)B * n};
    const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hkv * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kBN};
    if (!make_map(&mkt, kt, 3, dims, str, box) || !make_map(&mvt, vt, 3, dims, str, box))
      return cudaErrorInvalidValue;
  }
  const int G = Hq / Hkv;
  CUtensorMap mq;
  const bool q_tma = (kRowsPerCta % G) == 0;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)B * n};
    const cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)(q_tma ? G : 1), (cuuint32_t)(q_tma ? kRowsPerCta / G : 1)};
    if (!make_map(&mq, q, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  TcParams p;
  p.q_by_tma = q_tma ? 1 : 0;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.plen = plen;
  p.mask = mask;
  p.pos = pos;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = err;
  p.Lmax = Lmax;
  p.n = n;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.window = window;
  p.n_splits = plan.n_splits;
  p.chunk = plan.chunk;
  p.row_groups = attention_row_groups(n, Hq, Hkv);
  p.scale_log2 = scale * 1.4426950408889634f;
  const size_t smem = TcLayout<D>::kSmemBytes;
  cudaError_t e = ensure_smem_limit((const void*)attn_tc_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const int cs = plan.n_splits + 1;  // one cluster = every split of one (sequence, KV head, row group)
  if (cs > 8) {
    static bool np_set[2] = {false, false};
    if (!np_set[D == 128]) {
      e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      np_set[D == 128] = true;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, Hkv, B * p.row_groups);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel<D>, mk, mv, mkt, mvt, mq, p);
}

cudaError_t launch_attention_tc(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                                const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                                int n, int Hq, int Hkv, int D, int window, float scale, const AttnPlan& plan,
                                void* out, int* err, cudaStream_t s) {
  if (D == 128)
    return launch_tc<128>(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, window, scale, plan, out, err, s);
  return launch_tc<64>(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, window, scale, plan, out, err, s);
}

}  // namespace eagle
