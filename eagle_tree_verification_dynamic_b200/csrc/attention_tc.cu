// Tree-masked split-KV attention on the 5th-generation tensor cores
// ("Tree Attention" verification of the EAGLE notes, "3.Verify"; mask
// semantics of "Технический анализ EAGLE-4", section "Деревья проверки
// EAGLE-4 и утилита управления").
//
// Work decomposition.  A unit is (sequence b, KV head g, group rg of 128 query
// rows); the rows are the (node, head-in-group) pairs of head g, so every K/V
// tile staged in shared memory serves all tree queries of the GQA group.  A
// unit's keys are cut into tiles of 64: its visible prefix range first, then
// its n tree keys.  All tiles of all units form one list (unit-major) that is
// cut into C equal contiguous ranges, one per CTA, with C <= the SM count and
// one CTA per SM: every CTA streams the same amount of KV whatever the prefix
// lengths of a ragged batch.  Each CTA derives the list from prefix_len itself.
// A unit that lies inside one CTA's range is finished there (bf16 output); a
// unit cut by range boundaries leaves one normalised partial (O rows and
// log-sum-exp) per piece, merged by attn_combine_kernel.
//
// Roles inside a CTA (320 threads):
//   warp 0      producer: Q of each unit (TMA box, or a gather when G does not
//               divide 128) into one of two Q buffers; K and V tiles into a
//               ring of stages (128-byte swizzle, no multicast); TMEM owner
//   warp 1      one thread issues tcgen05.mma: S = Q K^T into one of two TMEM
//               S buffers, at most one tile ahead of PV; O += P V into TMEM,
//               each tile's keys 0..31 into O_A and keys 32..63 into O_B
//   warps 2-9   softmax, two warps per TMEM lane quarter: thread r owns query
//               row r, one warp the first 32 keys of every tile (and O_A), the
//               other the last 32 (and O_B).  Each applies the prefix range /
//               window / tree bitmask, keeps its own running reference max
//               (re-based only when it grows by > 8 in log2 units, then its O
//               and row sum are rescaled in TMEM) and writes P = 2^(x - m) as
//               bf16 into one of two swizzled P buffers.  At the end of a
//               unit's piece the pair exchanges (max, sum) through shared
//               memory, merges O_A and O_B, and writes the output or partial
//
// Every mbarrier wait is bounded (about 2 s of wall time); a timeout sets an
// abort flag that ends all roles, records a per-CTA status word and still
// frees the TMEM columns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "eagle_internal.h"
#include "sm100_ptx.cuh"

namespace eagle {

using namespace sm100;

constexpr int kTcThreads = 320;   // 10 warps: producer, MMA, 8 softmax
constexpr int kBN = kAttnKeysPerTile;
constexpr int kRowsPerCta = kAttnRowsPerUnit;
constexpr int kMaxStages = 12;
constexpr int kSmemOptIn = 232448;  // largest dynamic shared memory a block may opt into on sm_100
constexpr int kCombineThreads = 128;

// Shared memory from the (1024-byte aligned) dynamic base: a 3 KB header
// (barriers, then each row's (max, sum) exchange between the two softmax
// warps of a lane quarter), two Q buffers, the K/V ring (P lives in TMEM).
template <int D>
struct TcLayout {
  static constexpr int kAtoms = D / 64;               // 128-byte column atoms along D
  static constexpr int kQBytes = kAtoms * 128 * 128;  // 128 rows
  static constexpr int kKVAtomBytes = kBN * 128;      // 64 keys x 128 B
  static constexpr int kKBytes = kAtoms * kKVAtomBytes;
  static constexpr int kStageBytes = 2 * kKBytes;     // K + V
  static constexpr int kHdrBytes = 3072;
  static constexpr int kBarOff = 0;
  static constexpr int kXchOff = 512;                 // float2 [2 halves][128 rows]
  static constexpr int kQOff = kHdrBytes;             // two Q buffers
  static constexpr int kStageOff = kQOff + 2 * kQBytes;
  static constexpr int kStagesFit = (kSmemOptIn - kStageOff) / kStageBytes;
  static constexpr int kStages = kStagesFit > kMaxStages ? kMaxStages : kStagesFit;
  static constexpr int kSmemBytes = kStageOff + kStages * kStageBytes;
  // TMEM: three S buffers (64 columns each: QK^T may run two tiles ahead of
  // PV, so the softmax warps find the next S ready), then O over each tile's
  // keys 0..31 (O_A) and over keys 32..63 (O_B): the two softmax warps of a
  // lane quarter keep independent running maxima and are merged once per piece.
  // P (bf16, two keys per column) overwrites the S it came from: keys 0..31
  // at the buffer's columns 0..15, keys 32..63 at columns 32..47, each inside
  // the columns of S its own warp has already read.
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kSBufs = 3;
  static constexpr uint32_t kColS = 0;  // S buffer i at column 64 * i
  static constexpr uint32_t kColOA = kSBufs * 64;
  static constexpr uint32_t kColOB = kSBufs * 64 + D;
  static_assert(kStages >= 2, "at least a double-buffered K/V ring");
  static_assert(kSmemBytes <= kSmemOptIn, "shared memory");
  static_assert(kXchOff + 2 * 128 * 8 <= kHdrBytes, "header");
  static_assert(kColOB + D <= kTmemCols, "TMEM");
};

struct TcBars {
  uint64_t q_full[2];
  uint64_t q_empty[2];
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t s_full[3];
  uint64_t p_full[3][2];  // per S buffer, per half of the tile's keys (the four warps writing that half)
  uint64_t pv_done[3];
  uint64_t mma_idle;
  uint64_t pair[4];  // per lane quarter: both softmax warps wrote their (max, sum)
  uint64_t never;    // nothing arrives here: the wait probe's barrier
  uint32_t tmem_base;
  int abort;
  int bad_page;  // a key inside the sequence sat on a page id outside the pool
  // this CTA's tile range [t0, t1) of the global list, and where it starts
  int n_tiles;  // t1 - t0
  int b0, hr0, off0;
};
static_assert(sizeof(TcBars) <= 512, "barrier block");  // kXchOff

// ----------------------------------------------------------- tile schedule
struct AttnGeom {
  const int32_t* plen;
  int B, Hkv, RG, n, Lmax, window, C;
  int lo_align;  // the first prefix tile starts at a multiple of this (64 for a paged cache, else 1)
};

__device__ __forceinline__ int geom_len(const AttnGeom& a, int b) {
  return min(max(__ldg(a.plen + b), 0), a.Lmax);
}
// first visible prefix key of a sequence of length L (the window of the
// shallowest tree node, depth 1, at position L)
__device__ __forceinline__ int geom_lo(const AttnGeom& a, int L) {
  const int lo = a.window > 0 ? max(0, L - a.window + 1) : 0;
  return lo - lo % a.lo_align;  // keys below the window start are masked row by row
}
__device__ __forceinline__ int geom_ptiles(const AttnGeom& a, int L) { return (L - geom_lo(a, L) + kBN - 1) / kBN; }
__device__ __forceinline__ int geom_tiles(const AttnGeom& a, int b) {
  return geom_ptiles(a, geom_len(a, b)) + (a.n + kBN - 1) / kBN;
}

// Whole warp: total tiles of all units, and the first tile of sequence b_end.
__device__ __forceinline__ long long geom_prefix(const AttnGeom& a, int b_end, int lane) {
  const int HR = a.Hkv * a.RG;
  long long acc = 0;
  for (int b = lane; b < b_end; b += 32) acc += (long long)HR * geom_tiles(a, b);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
  return acc;
}

// Whole warp: the unit (b, hr) holding global tile t and t's offset in it.
__device__ __forceinline__ void geom_locate(const AttnGeom& a, long long t, int lane, int& b_out, int& hr_out,
                                            int& off_out) {
  const int HR = a.Hkv * a.RG;
  long long base = 0;
  for (int bc = 0; bc < a.B; bc += 32) {
    const int b = bc + lane;
    const int tb = b < a.B ? geom_tiles(a, b) : 0;
    const long long v = (long long)HR * tb;
    long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += y;
    }
    const long long exc = inc - v;
    const bool hit = b < a.B && base + exc <= t && t < base + inc;
    const unsigned m = __ballot_sync(kFull, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      int bb = 0, hr = 0, off = 0;
      if (lane == src) {
        const long long within = t - (base + exc);
        bb = b;
        hr = (int)(within / tb);
        off = (int)(within % tb);
      }
      b_out = __shfl_sync(kFull, bb, src);
      hr_out = __shfl_sync(kFull, hr, src);
      off_out = __shfl_sync(kFull, off, src);
      return;
    }
    base += __shfl_sync(kFull, inc, 31);
  }
  b_out = a.B;
  hr_out = 0;
  off_out = 0;
}

// CTA c holds tiles [c*T/C, (c+1)*T/C); this is the CTA holding tile t.
__device__ __forceinline__ int cta_of_tile(long long t, long long T, int C) {
  return (int)(((t + 1) * C - 1) / T);
}
// With fewer tiles than CTAs (a ragged batch far below Lmax) some ranges are empty.
__device__ __forceinline__ bool cta_nonempty(int c, long long T, int C) {
  return (long long)(c + 1) * T / C > (long long)c * T / C;
}

// One contiguous piece of a unit inside one CTA's range.
struct Piece {
  int b, hr;    // unit = b * HR + hr
  int tb, te;   // tiles [tb, te) of the unit
  int ptiles;   // the unit's prefix tiles (tiles >= ptiles are tree tiles)
  int L, lo;    // prefix length and first visible prefix key
  bool whole;   // the piece is the entire unit
};

struct PieceCursor {
  int b, hr, off, left;
  __device__ __forceinline__ void init(int b0, int hr0, int off0, int n_tiles) {
    b = b0;
    hr = hr0;
    off = off0;
    left = n_tiles;
  }
  __device__ __forceinline__ void init(const TcBars* s) { init(s->b0, s->hr0, s->off0, s->n_tiles); }
  __device__ __forceinline__ bool next(const AttnGeom& a, Piece& pc) {
    if (left <= 0) return false;
    const int HR = a.Hkv * a.RG;
    pc.b = b;
    pc.hr = hr;
    pc.L = geom_len(a, b);
    pc.lo = geom_lo(a, pc.L);
    pc.ptiles = geom_ptiles(a, pc.L);
    const int tiles = pc.ptiles + (a.n + kBN - 1) / kBN;
    const int nt = min(tiles - off, left);
    pc.tb = off;
    pc.te = off + nt;
    pc.whole = off == 0 && nt == tiles;
    left -= nt;
    off = 0;
    if (++hr == HR) {
      hr = 0;
      ++b;
    }
    return true;
  }
};

struct TcParams {
  const __nv_bfloat16* q;
  const uint64_t* mask;
  const int32_t* pos;
  __nv_bfloat16* out;
  float* part_o;    // [C + U][128][D] normalised partial outputs
  float* part_lse;  // [C + U][128]
  int* cta_status;  // [C]
  AttnGeom geo;
  int Hq;
  int q_by_tma;      // 1: Q rows arrive by TMA (G divides 128), 0: gathered by the producer warp
  float scale_log2;  // softmax scale * log2(e)
  // paged prefix cache (block_table != null): pools [num_pages][Hkv][page_size][D],
  // block_table [B][pages_per_seq] page ids
  const int32_t* block_table;
  int page_size, pages_per_seq, num_pages;
  // > 0: every softmax warp first waits this long (ns) on a barrier nothing
  // completes, so the CTA takes its abort path (eagle_debug_attention_wait_probe)
  unsigned long long probe_ns;
  // 1: everything but mask and pos was written before the previous kernel on
  // the stream started (the fused step, where that kernel is the expansion),
  // so Q, the prefix and tree K/V and prefix_len are read at once and only the
  // softmax warps wait for the previous kernel (for mask and pos)
  int early;
};

// Loads issued now and consumed later: the K/V stream keeps HBM saturated, so
// a demand load waits behind it for microseconds; the per-row inputs of a
// piece are therefore requested a whole piece ahead (the first piece's before
// the stream starts).
__device__ __forceinline__ uint64_t ld_early_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.global.nc.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ int ld_early_s32(const int32_t* p) {
  int v;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// What a softmax thread reads besides S for one piece.
struct RowCtx {
  uint64_t mw0, mw1;  // ancestor-or-self bitmask of this row's node (pieces with tree tiles)
  int qpos;           // this row's position (window only)
  int tpos[4];        // positions of tree keys lane, 32+lane, 64+lane, 96+lane (window and tree tiles)
};

__device__ __forceinline__ void row_issue(RowCtx& rc, const Piece& pc, const TcParams& p, int r_local, int lane,
                                          int G) {
  const AttnGeom& a = p.geo;
  const int r_glob = (pc.hr % a.RG) * kRowsPerCta + r_local;
  const bool row_ok = r_glob < a.n * G;
  const int qi = row_ok ? r_glob / G : 0;
  const size_t nb = (size_t)pc.b * a.n;
  const bool has_tree = pc.te > pc.ptiles;
  rc.mw0 = rc.mw1 = 0;
  rc.qpos = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) rc.tpos[i] = 0;
  if (row_ok && has_tree) {
    rc.mw0 = ld_early_u64(p.mask + (nb + qi) * 2);
    rc.mw1 = ld_early_u64(p.mask + (nb + qi) * 2 + 1);
  }
  if (a.window > 0) {
    if (row_ok) rc.qpos = ld_early_s32(p.pos + nb + qi);
    if (has_tree) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (32 * i + lane < a.n) rc.tpos[i] = ld_early_s32(p.pos + nb + 32 * i + lane);
    }
  }
}

// Block-table entry idx of a sequence (-1 past the table's width).
__device__ __forceinline__ int table_entry(const int32_t* bt, int idx, int width) {
  return idx < width ? ld_early_s32(bt + idx) : -1;
}

// Producer for a paged prefix cache: the K/V tiles of one piece.  A prefix
// tile's 64 keys (starting at a multiple of 64) arrive as boxes of
// min(page_size, 64) keys, each from the page the sequence's block table
// names.  The whole warp walks the tiles (lane 0 waits and issues) and reads
// the table 32 entries per coalesced load; the next 32 are requested as soon
// as the current ones are first used, so only a piece's first lookup waits on
// memory.  A page id outside the pool turns into a box past the end, which
// reads zeros; if a key inside the sequence sat there, the CTA reports it.
// Returns false when a wait gave up.
template <int D>
__device__ bool produce_paged(const TcParams& p, const AttnGeom& a, const Piece& pc, int g, uint32_t s_base,
                              TcBars* bars, volatile int* abort, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                              const CUtensorMap* tm_kt, const CUtensorMap* tm_vt, int lane, int& jg) {
  using Lay = TcLayout<D>;
  constexpr int S = Lay::kStages;
  const int ps = p.page_size;
  const int sub = ps < kBN ? ps : kBN;  // keys per box
  const int nsub = kBN / sub;           // boxes per tile: 1, 2 or 4
  const int32_t* bt = p.block_table + (size_t)pc.b * p.pages_per_seq;
  const int past_end = p.num_pages * a.Hkv * ps;  // first row past the pools (the host keeps it in int range)
  int c0 = -64, cur = -1, nxt = -1;               // table chunk [c0, c0 + 32): lane l holds entry c0 + l
  for (int t = pc.tb; t < pc.te; ++t) {
    const int st = jg % S;
    bool w = true;
    if (lane == 0 && jg >= S) w = mbar_wait(smem_u32(&bars->empty[st]), ((jg / S) - 1) & 1, abort);
    if (!__shfl_sync(kFull, w, 0)) return false;
    const uint32_t fb = smem_u32(&bars->full[st]);
    const uint32_t kdst = s_base + Lay::kStageOff + st * Lay::kStageBytes;
    const uint32_t vdst = kdst + Lay::kKBytes;
    if (t < pc.ptiles) {
      const int key0 = pc.lo + t * kBN;
      const int e0 = key0 / ps;  // the tile's first entry; its nsub entries share e0's chunk
      const int base = e0 & ~31;
      if (base != c0) {  // warp-uniform
        cur = base == c0 + 32 ? nxt : table_entry(bt, base + lane, p.pages_per_seq);
        c0 = base;
        nxt = table_entry(bt, c0 + 32 + lane, p.pages_per_seq);
      }
      int row[4];
      bool bad = false;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int page = __shfl_sync(kFull, cur, (e0 - c0 + j) & 31);  // every lane takes part
        const int kj = key0 + j * sub;
        const bool valid = page >= 0 && page < p.num_pages;
        if (j < nsub && !valid && kj < pc.L) bad = true;
        row[j] = valid ? (page * a.Hkv + g) * ps + kj % ps : past_end;
      }
      if (lane == 0) {
        if (bad) bars->bad_page = 1;
        mbar_arrive_expect_tx(fb, Lay::kStageBytes);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j < nsub) {
            for (int at = 0; at < Lay::kAtoms; ++at) {
              tma_load_2d(kdst + at * Lay::kKVAtomBytes + j * sub * 128, tm_k, at * 64, row[j], fb);
              tma_load_2d(vdst + at * Lay::kKVAtomBytes + j * sub * 128, tm_v, at * 64, row[j], fb);
            }
          }
        }
      }
    } else if (lane == 0) {
      mbar_arrive_expect_tx(fb, Lay::kStageBytes);
      const int z = pc.b * a.n + (t - pc.ptiles) * kBN;
      for (int at = 0; at < Lay::kAtoms; ++at) {
        tma_load_3d(kdst + at * Lay::kKVAtomBytes, tm_kt, at * 64, g, z, fb);
        tma_load_3d(vdst + at * Lay::kKVAtomBytes, tm_vt, at * 64, g, z, fb);
      }
    }
    ++jg;
  }
  return true;
}

// How long a waiting softmax warp or producer lane may sleep per poll (ns):
// the MMA warp shares a scheduler with two softmax warps, and a warp that
// polls in a tight loop takes issue slots from it.
constexpr uint32_t kSoftmaxSleepNs = 300u;
constexpr uint32_t kProducerSleepNs = 500u;

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_vt,
               const __grid_constant__ CUtensorMap tm_q, const TcParams p) {
  using Lay = TcLayout<D>;
  constexpr int S = Lay::kStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  const AttnGeom& a = p.geo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  // The layout fills the opt-in maximum and the swizzled tiles need a
  // 1024-byte aligned base: with any other base the CTA does nothing and
  // reports status 2 (the whole CTA leaves here, before any barrier).
  if ((smem_u32(smem) & 1023u) != 0u) {
    if (tid == 0) p.cta_status[c] = 2;
    griddep_wait();
    griddep_launch_dependents();
    return;
  }
  TcBars* bars = reinterpret_cast<TcBars*>(smem + Lay::kBarOff);
  const uint32_t s_base = smem_u32(smem);
  const int G = p.Hq / a.Hkv;
  const int rows = a.n * G;
  const int HR = a.Hkv * a.RG;
  volatile int* abort = &bars->abort;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->q_full[i]), 1);
      mbar_init(smem_u32(&bars->q_empty[i]), 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      // every softmax thread of a half (4 warps) arrives for every tile, rows
      // or not; S(j) is written only after PV(j - 3) was issued, so a phase
      // completes before the next one on the same barrier begins
      mbar_init(smem_u32(&bars->p_full[i][0]), 128);
      mbar_init(smem_u32(&bars->p_full[i][1]), 128);
      mbar_init(smem_u32(&bars->pv_done[i]), 1);
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(&bars->full[i]), 1);
      mbar_init(smem_u32(&bars->empty[i]), 1);
    }
    mbar_init(smem_u32(&bars->mma_idle), 1);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars->pair[i]), 64);
    mbar_init(smem_u32(&bars->never), 1);
    bars->abort = 0;
    bars->bad_page = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_kt);
    prefetch_tmap(&tm_vt);
    if (p.q_by_tma) prefetch_tmap(&tm_q);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), Lay::kTmemCols);
    tmem_relinquish();
  }
  // inputs may come from the previous kernel on the stream (with p.early only
  // mask and pos do, and the softmax warps wait for them after the barrier)
  if (!p.early) griddep_wait();
  // softmax warps: cursor and the first piece's row inputs, requested before
  // the K/V stream starts
  PieceCursor scur;
  Piece spc;
  RowCtx src;
  bool s_have = false;
  const int quad = warp & 3;
  const int r_local = quad * 32 + lane;  // softmax: TMEM lane = row within the unit's 128
  if (warp >= 1) {
    const long long T = geom_prefix(a, a.B, lane);
    const long long t0 = (long long)c * T / a.C, t1 = (long long)(c + 1) * T / a.C;
    int b0 = a.B, hr0 = 0, off0 = 0;
    if (t1 > t0) geom_locate(a, t0, lane, b0, hr0, off0);
    if (warp == 1 && lane == 0) {
      bars->n_tiles = (int)(t1 - t0);
      bars->b0 = b0;
      bars->hr0 = hr0;
      bars->off0 = off0;
    }
    if (warp >= 2) {
      scur.init(b0, hr0, off0, (int)(t1 - t0));
      s_have = scur.next(a, spc);
      // issued before the block barrier, so ahead of the first K/V copies,
      // and consumed only at the piece's first tile: the producer does not
      // wait for them (a load issued behind the K/V stream waits microseconds)
      if (s_have && !p.early) row_issue(src, spc, p, r_local, lane, G);
    }
  }
  // a thread lets the next kernel start only after its own griddep_wait, so
  // that kernel's early reads never see work older than this kernel's
  // predecessor unfinished
  if (!p.early) griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    PieceCursor cur;
    cur.init(bars);
    Piece pc;
    int si = 0, jg = 0;  // pieces whose Q was loaded; tiles issued
    bool ok = true;
    while (ok && cur.next(a, pc)) {
      const int qb = si & 1;
      const int g = pc.hr / a.RG, rg = pc.hr % a.RG;
      // Q buffer qb was last read by the QK^T of piece si - 2
      if (si >= 2 && !__all_sync(kFull, mbar_wait(smem_u32(&bars->q_empty[qb]), ((si >> 1) - 1) & 1, abort))) {
        ok = false;
        break;
      }
      const uint32_t qdst = s_base + Lay::kQOff + qb * Lay::kQBytes;
      const uint32_t qbar = smem_u32(&bars->q_full[qb]);
      if (p.q_by_tma) {
        // the 128 rows = (node, head-in-group) pairs: a box of {64 dims, G
        // heads, 128/G nodes} of q viewed as [B*n][Hq][D]
        if (lane == 0) {
          mbar_arrive_expect_tx(qbar, Lay::kQBytes);
          const int rows_i = kRowsPerCta / G;
          for (int at = 0; at < Lay::kAtoms; ++at)
            tma_load_3d(qdst + at * 16384, &tm_q, at * 64, g * G, pc.b * a.n + rg * rows_i, qbar);
        }
      } else {
        // gather: 16-byte pieces of the 128 rows into the swizzled K-major tile
        constexpr int kVec = 128 * Lay::kAtoms * 8;
        constexpr int kBatch = 8;
        for (int e0 = lane; e0 < kVec; e0 += 32 * kBatch) {
          uint4 v[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int e = e0 + u * 32;
            v[u] = make_uint4(0, 0, 0, 0);
            if (e < kVec) {
              const int r = e / (Lay::kAtoms * 8), at = (e / 8) % Lay::kAtoms, cc = e % 8;
              const int rr = rg * kRowsPerCta + r;
              if (rr < rows) {
                const int i = rr / G, h = g * G + rr % G;
                v[u] = *reinterpret_cast<const uint4*>(p.q + (((size_t)pc.b * a.n + i) * p.Hq + h) * D + at * 64 +
                                                       cc * 8);
              }
            }
          }
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int e = e0 + u * 32;
            if (e < kVec) {
              const int r = e / (Lay::kAtoms * 8), at = (e / 8) % Lay::kAtoms, cc = e % 8;
              *reinterpret_cast<uint4*>(smem + Lay::kQOff + qb * Lay::kQBytes + at * 16384 + r * 128 +
                                        ((cc ^ (r & 7)) << 4)) = v[u];
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(qbar);
      }
      ++si;
      if (p.block_table != nullptr) {
        ok = produce_paged<D>(p, a, pc, g, s_base, bars, abort, &tm_k, &tm_v, &tm_kt, &tm_vt, lane, jg);
      } else if (lane == 0) {
        for (int t = pc.tb; t < pc.te; ++t) {
          const int st = jg % S;
          if (jg >= S && !mbar_wait(smem_u32(&bars->empty[st]), ((jg / S) - 1) & 1, abort, 2000000000ull,
                                    kProducerSleepNs)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&bars->full[st]);
          mbar_arrive_expect_tx(fb, Lay::kStageBytes);
          const uint32_t kdst = s_base + Lay::kStageOff + st * Lay::kStageBytes;
          const uint32_t vdst = kdst + Lay::kKBytes;
          if (t < pc.ptiles) {
            const int y = (pc.b * a.Hkv + g) * a.Lmax + pc.lo + t * kBN;
            for (int at = 0; at < Lay::kAtoms; ++at) {
              tma_load_2d(kdst + at * Lay::kKVAtomBytes, &tm_k, at * 64, y, fb);
              tma_load_2d(vdst + at * Lay::kKVAtomBytes, &tm_v, at * 64, y, fb);
            }
          } else {
            const int z = pc.b * a.n + (t - pc.ptiles) * kBN;
            for (int at = 0; at < Lay::kAtoms; ++at) {
              tma_load_3d(kdst + at * Lay::kKVAtomBytes, &tm_kt, at * 64, g, z, fb);
              tma_load_3d(vdst + at * Lay::kKVAtomBytes, &tm_vt, at * 64, g, z, fb);
            }
          }
          ++jg;
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      jg = __shfl_sync(kFull, jg, 0);
    }
    if (p.early) {
      griddep_wait();
      griddep_launch_dependents();
    }
    // drain: every issued copy lands before the CTA may exit
    if (lane == 0) {
      for (int j = (jg > S ? jg - S : 0); j < jg; ++j)
        mbar_wait_drain(smem_u32(&bars->full[j % S]), (j / S) & 1, 200000000ull);
      for (int s2 = (si > 2 ? si - 2 : 0); s2 < si; ++s2)
        mbar_wait_drain(smem_u32(&bars->q_full[s2 & 1]), (s2 >> 1) & 1, 200000000ull);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (p.early) {
      griddep_wait();
      griddep_launch_dependents();
    }
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16_f32(128, kBN, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t t_oa = tmem + Lay::kColOA, t_ob = tmem + Lay::kColOB;
      const int total = bars->n_tiles;
      // one throw-away MMA while the first tiles are in flight (the first
      // MMA of a CTA was measured to take ~3 us longer than the next ones):
      // it reads the second Q buffer and the last K/V stage, whatever they
      // hold, into the third S buffer, which QK^T(2) overwrites (in order)
      if (total > 0) {
        const uint64_t da = smem_desc(s_base + Lay::kQOff + Lay::kQBytes, 16, 1024, kSwizzle128B);
        const uint64_t db = smem_desc(s_base + Lay::kStageOff + (S - 1) * Lay::kStageBytes, 16, 1024, kSwizzle128B);
        mma_bf16_ss(tmem + Lay::kColS + 2u * kBN, da, db, id_qk, 0u);
      }
      PieceCursor qc, pcur;
      qc.init(bars);
      pcur.init(bars);
      Piece qp, pp;
      int q_si = -1, q_rem = 0, jq = 0;  // QK^T cursor: piece, tiles left in it, next tile
      int p_rem = 0, p_len = 0;          // PV cursor: tiles left in its piece, piece length
      bool ok = true;
      for (int jp = 0; jp < total && ok; ++jp) {
        if (p_rem == 0) {
          pcur.next(a, pp);
          p_len = p_rem = pp.te - pp.tb;
        }
        const bool first = p_rem == p_len;  // O restarts at the first tile of a piece
        // issue whatever is ready: the next QK^T (its Q and K landed; at most
        // two tiles ahead), and this tile's PV per half of its keys (that
        // half's P is written)
        const int pbuf = jp % 3;
        const uint32_t ppar = (uint32_t)(jp / 3) & 1u;
        const int st = jp % S;
        const uint32_t p_tmem = tmem + Lay::kColS + (uint32_t)(pbuf * kBN);
        const uint32_t v_addr = s_base + Lay::kStageOff + st * Lay::kStageBytes + Lay::kKBytes;
        bool done_h[2] = {false, false};
        uint64_t tw = 0;
        for (uint32_t it = 0;; ++it) {
          if (jq < total && jq <= jp + 2) {
            if (q_rem == 0) {
              qc.next(a, qp);
              ++q_si;
              q_rem = qp.te - qp.tb;
            }
            const int qb = q_si & 1;
            if (mbar_test_wait(smem_u32(&bars->q_full[qb]), (q_si >> 1) & 1) &&
                mbar_test_wait(smem_u32(&bars->full[jq % S]), (jq / S) & 1)) {
              tc_fence_after();
              const uint32_t q_addr = s_base + Lay::kQOff + qb * Lay::kQBytes;
              const uint32_t k_addr = s_base + Lay::kStageOff + (jq % S) * Lay::kStageBytes;
              const uint32_t t_s = tmem + Lay::kColS + (uint32_t)((jq % 3) * kBN);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk % 4) * 32;
                const uint64_t da = smem_desc(q_addr + (kk / 4) * 16384 + off, 16, 1024, kSwizzle128B);
                const uint64_t db = smem_desc(k_addr + (kk / 4) * Lay::kKVAtomBytes + off, 16, 1024, kSwizzle128B);
                mma_bf16_ss(t_s, da, db, id_qk, kk > 0);
              }
              mma_commit(smem_u32(&bars->s_full[jq % 3]));
              if (--q_rem == 0) mma_commit(smem_u32(&bars->q_empty[qb]));
              ++jq;
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // the first half still missing is waited for with a short sleep
            // (the MMA warp shares its scheduler with two softmax warps, whose
            // issue slots a spinning poll would take); the other is only tested
            const uint32_t pbar = smem_u32(&bars->p_full[pbuf][h]);
            const bool waited = (h == 0 || done_h[0]) ? mbar_try_wait_hint(pbar, ppar, 200u) : mbar_test_wait(pbar, ppar);
            if (!done_h[h] && waited) {
              tc_fence_after();
              // keys 32h..32h+31 of the tile into O_A (h = 0) or O_B (h = 1); P
              // from TMEM, 16 keys = 8 columns per MMA
#pragma unroll
              for (int kk = 2 * h; kk < 2 * h + 2; ++kk) {
                const uint32_t a_col = (uint32_t)((kk >> 1) * 32 + (kk & 1) * 8);
                const uint64_t db = smem_desc(v_addr + kk * 2048, Lay::kKVAtomBytes, 1024, kSwizzle128B);
                mma_bf16_ts(h ? t_ob : t_oa, p_tmem + a_col, db, id_pv, (!first || (kk & 1)) ? 1u : 0u);
              }
              done_h[h] = true;
            }
          }
          if (done_h[0] && done_h[1]) break;
          if ((it & 15u) == 15u) {
            if (*abort) { ok = false; break; }
            const uint64_t now = globaltimer();
            if (tw == 0) tw = now;
            else if (now - tw > 2000000000ull) { *abort = 1; ok = false; break; }
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(&bars->empty[st]));
        mma_commit(smem_u32(&bars->pv_done[pbuf]));
        --p_rem;
      }
      // every MMA this thread issued has finished before TMEM is released
      mma_commit(smem_u32(&bars->mma_idle));
      mbar_wait_drain(smem_u32(&bars->mma_idle), 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------------- softmax
    // warps 2..9: quad = TMEM lane quarter (32 query rows); half = which 32
    // keys of every tile, and which O accumulator, this warp owns.  The two
    // halves keep independent running maxima and sums and are merged once
    // per piece.
    const int half = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint32_t t_s = tmem + lane_base + Lay::kColS + (uint32_t)(half * 32);
    const uint32_t t_own = tmem + lane_base + (half ? Lay::kColOB : Lay::kColOA);
    const uint32_t t_oa = tmem + lane_base + Lay::kColOA, t_ob = tmem + lane_base + Lay::kColOB;
    float2* xch = reinterpret_cast<float2*>(smem + Lay::kXchOff);  // [half][row]
    const float sl2 = p.scale_log2;
    if (p.early) {
      griddep_wait();  // mask and pos come from the previous kernel
      griddep_launch_dependents();
      if (s_have) row_issue(src, spc, p, r_local, lane, G);
    }
    Piece pc = spc;
    RowCtx rc = src;
    bool have = s_have;
    int jg = 0, n_epi = 0;
    bool ok = true;
    // the wait probe: a bounded wait that runs out, then the same abort path as
    // any wait that gives up (the other roles see the flag and drain)
    if (p.probe_ns != 0ull && !__all_sync(kFull, mbar_wait(smem_u32(&bars->never), 0, abort, p.probe_ns))) ok = false;
    while (ok && have) {
      Piece pn;
      RowCtx rn;
      const bool have_next = scur.next(a, pn);
      if (have_next) row_issue(rn, pn, p, r_local, lane, G);  // in flight during this piece
      const int g = pc.hr / a.RG, rg = pc.hr % a.RG;
      const int row0 = rg * kRowsPerCta;
      const int r_glob = row0 + r_local;
      const bool row_ok = r_glob < rows;
      const bool warp_live = row0 + quad * 32 < rows;  // a warp of padding rows only keeps the protocol
      const int qi = row_ok ? r_glob / G : 0;
      const int qh = row_ok ? g * G + r_glob % G : 0;
      const int win_lo = rc.qpos - a.window + 1;
      float m_used = -INFINITY, l = 0.f;  // reference max (scaled, log2) and row sum of this half
      for (int t = pc.tb; t < pc.te; ++t, ++jg) {
        const int sbuf = jg % 3;
        if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->s_full[sbuf]), (uint32_t)(jg / 3) & 1u, abort, 2000000000ull,
                                         kSoftmaxSleepNs))) {
          ok = false;
          break;
        }
        if (warp_live) {
          tc_fence_after();
          float x[32];
          tmem_ld32(t_s + (uint32_t)(sbuf * kBN), x);
          tmem_wait_ld();
          const bool tree = t >= pc.ptiles;
          const int key0 = (tree ? (t - pc.ptiles) * kBN : pc.lo + t * kBN) + half * 32;
          const int k1 = tree ? a.n : pc.L;
          // visibility of this half's 32 keys as one bit mask, built the same
          // way on every tile (so the code stays hot in the instruction cache):
          // keys below the piece's end, then the ancestor bits (tree keys) or
          // the window's lower bound (prefix keys)
          const int lim = k1 - key0;
          uint32_t vm = lim >= 32 ? 0xffffffffu : (lim > 0 ? (1u << lim) - 1u : 0u);
          const uint64_t mw = key0 >= 64 ? rc.mw1 : rc.mw0;
          const uint32_t tree_bits = (uint32_t)(mw >> (key0 & 63));
          const int lo_cut = win_lo - key0;  // prefix keys below it are outside the window
          const uint32_t win_bits =
              (a.window == 0 || lo_cut <= 0) ? 0xffffffffu : (lo_cut >= 32 ? 0u : ~((1u << lo_cut) - 1u));
          vm &= tree ? tree_bits : win_bits;
          if (!row_ok) vm = 0u;
          if (tree && a.window > 0) {  // the window on tree keys' positions (rare; warp-uniform)
            const int grp = key0 >> 5;
            const int tsel = grp == 0 ? rc.tpos[0] : grp == 1 ? rc.tpos[1] : grp == 2 ? rc.tpos[2] : rc.tpos[3];
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) {
              const int kpos = __shfl_sync(kFull, tsel, cc);  // every lane takes part
              if (kpos < win_lo) vm &= ~(1u << cc);
            }
          }
          if (__any_sync(kFull, vm != 0xffffffffu)) {  // most prefix tiles see every key
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) x[cc] = ((vm >> cc) & 1u) ? x[cc] : -INFINITY;
          }
          float m4[4] = {fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[8]),
                         fmax3(x[9], x[10], x[11])};
#pragma unroll
          for (int cc = 12; cc < 28; cc += 8) {
            m4[0] = fmax3(m4[0], x[cc], x[cc + 1]);
            m4[1] = fmax3(m4[1], x[cc + 2], x[cc + 3]);
            m4[2] = fmax3(m4[2], x[cc + 4], x[cc + 5]);
            m4[3] = fmax3(m4[3], x[cc + 6], x[cc + 7]);
          }
          float mx = fmax3(fmax3(m4[0], m4[1], m4[2]), fmax3(m4[3], x[28], x[29]), fmaxf(x[30], x[31]));
          mx *= sl2;  // scale > 0 keeps the order
          // (P of this tile replaces S(jg) in TMEM: PV(jg - 2), the last reader of
          // those columns, completed before QK^T(jg), whose commit s_full waited on)
          const bool rebase = mx > m_used + 8.f;
          if (__any_sync(kFull, rebase && t > pc.tb && l > 0.f)) {
            // this half's O may only be rescaled once PV(jg - 1) has finished accumulating
            if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->pv_done[(jg - 1) % 3]), (uint32_t)((jg - 1) / 3) & 1u,
                                             abort))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float f = (rebase && l > 0.f) ? ex2(m_used - mx) : 1.f;
            for (int c0 = 0; c0 < D; c0 += 16) {
              float o[16];
              tmem_ld16(t_own + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int u = 0; u < 16; ++u) o[u] *= f;
              tmem_st16(t_own + c0, o);
            }
            tmem_wait_st();
            l *= f;
          }
          if (rebase) m_used = mx;
          const float neg_m = m_used > -INFINITY ? -m_used : 0.f;  // no visible key yet: every x is -inf
          float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          uint32_t packed[16];
          const float2 sl2x2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
#pragma unroll
          for (int c2 = 0; c2 < 16; ++c2) {
            const float2 z = ffma2(make_float2(x[2 * c2], x[2 * c2 + 1]), sl2x2, nm2);
            const float2 e = make_float2(ex2(z.x), ex2(z.y));
            s2[c2 & 1] = fadd2(s2[c2 & 1], e);
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(e.x, e.y);
            packed[c2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          const float2 st2 = fadd2(s2[0], s2[1]);
          l += st2.x + st2.y;
          tmem_st16u(t_s + (uint32_t)(sbuf * kBN), packed);  // P over this half's first 16 S columns
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->p_full[sbuf][half]));
      }
      if (!ok) break;
      // ---- end of the piece: merge the two halves' (max, sum), normalise,
      // write bf16 output or the partial + log-sum-exp.  Each warp of the pair
      // writes its half of the output columns from both accumulators.
      if (warp_live) {
        const int jl = jg - 1;
        if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->pv_done[jl % 3]), (uint32_t)(jl / 3) & 1u, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        xch[half * kRowsPerCta + r_local] = make_float2(m_used, l);
        mbar_arrive(smem_u32(&bars->pair[quad]));
        if (!__all_sync(kFull, mbar_wait(smem_u32(&bars->pair[quad]), n_epi & 1, abort))) {
          ok = false;
          break;
        }
        ++n_epi;
        const float2 other = xch[(half ^ 1) * kRowsPerCta + r_local];
        const float ma = half ? other.x : m_used, la = half ? other.y : l;
        const float mb = half ? m_used : other.x, lb = half ? l : other.y;
        const float M = fmaxf(ma, mb);
        const float wa = la > 0.f ? ex2(ma - M) : 0.f;
        const float wb = lb > 0.f ? ex2(mb - M) : 0.f;
        const float Ltot = la * wa + lb * wb;
        const float inv = Ltot > 0.f ? 1.f / Ltot : 0.f;
        const float fa = wa * inv, fb = wb * inv;
        const size_t slot = (size_t)c + (size_t)pc.b * HR + pc.hr;
        for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 16) {  // 16 columns at a time
          float oa[16], ob[16];
          tmem_ld16(t_oa + c0, oa);
          tmem_ld16(t_ob + c0, ob);
          tmem_wait_ld();
          if (!row_ok) continue;
#pragma unroll
          for (int u = 0; u < 16; ++u) oa[u] = fmaf(oa[u], fa, ob[u] * fb);
          if (pc.whole) {
            __nv_bfloat16* dst = p.out + (((size_t)pc.b * a.n + qi) * p.Hq + qh) * D + c0;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              uint32_t w[4];
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(oa[u * 8 + 2 * v], oa[u * 8 + 2 * v + 1]);
                w[v] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(dst + u * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            float* dst = p.part_o + (slot * kRowsPerCta + r_local) * D + c0;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              *reinterpret_cast<float4*>(dst + 4 * u) = make_float4(oa[4 * u], oa[4 * u + 1], oa[4 * u + 2], oa[4 * u + 3]);
          }
        }
        if (row_ok && !pc.whole && half == 0)
          p.part_lse[slot * kRowsPerCta + r_local] = Ltot > 0.f ? (M + __log2f(Ltot)) * (float)kLn2 : -INFINITY;
        tc_fence_before();
      }
      pc = pn;
      rc = rn;
      have = have_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, Lay::kTmemCols);
  if (tid == 0) p.cta_status[c] = bars->abort ? 1 : (bars->bad_page ? 3 : 0);
}

// Merge the pieces of every unit cut by CTA range boundaries:
//   out = sum_s e^{lse_s - M} O_s / sum_s e^{lse_s - M}
// One warp per query row (blockIdx.x = unit, blockIdx.y = group of 4 rows);
// each lane loads its D/32 dims of every piece's partial in one round of
// independent L2 reads, up to kCombChunk pieces at a time, merged online.
// A unit finished inside one CTA is skipped.  Block (0, 0) also folds the
// per-CTA status words into the workspace header.
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombChunk = 8;

struct CombParams {
  const float* part_o;
  const float* part_lse;
  const int* cta_status;
  int* status;
  __nv_bfloat16* out;
  AttnGeom geo;
  int Hq;
};

template <int D>
__global__ void __launch_bounds__(kCombineThreads)
attn_combine_kernel(const CombParams p) {
  const AttnGeom& a = p.geo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HR = a.Hkv * a.RG;
  const int u = blockIdx.x, b = u / HR, hr = u % HR;
  const int g = hr / a.RG, rg = hr % a.RG;
  const int G = p.Hq / a.Hkv;
  __shared__ long long s_T;
  __shared__ int s_cfirst, s_clast, s_stat[kCombineWarps];
  if (warp == 0) {  // the schedule depends only on prefix_len, not on the attention kernel
    const long long T = geom_prefix(a, a.B, lane);
    const long long cum = geom_prefix(a, b, lane);
    const int tiles = geom_tiles(a, b);
    if (lane == 0) {  // (64-bit divisions: done before the wait, while the attention runs)
      const long long start = cum + (long long)hr * tiles;
      s_T = T;
      s_cfirst = cta_of_tile(start, T, a.C);
      s_clast = cta_of_tile(start + tiles - 1, T, a.C);
    }
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();  // the next kernel's prologue may overlap this one
  if (blockIdx.x == 0 && blockIdx.y == 0) {
    int st = 0;
    for (int i = tid; i < a.C; i += kCombineThreads) st = max(st, p.cta_status[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) st = max(st, __shfl_xor_sync(kFull, st, o));
    if (lane == 0) s_stat[warp] = st;
    __syncthreads();
    if (tid == 0) {
      for (int w = 0; w < kCombineWarps; ++w) st = max(st, s_stat[w]);
      *p.status = st;
    }
  }
  const long long T = s_T;
  const int c_first = s_cfirst, c_last = s_clast;
  const bool all_live = T >= a.C;  // with at least one tile per CTA no range is empty
  const int r = blockIdx.y * kCombineWarps + warp;
  const int valid = min(kRowsPerCta, a.n * G - rg * kRowsPerCta);
  if (c_first == c_last || r >= valid) return;
  const int nseg = c_last - c_first + 1;
  const size_t slot0 = (size_t)c_first + u;
  constexpr int DPL = D / 32;  // output dims per lane
  float M = -INFINITY, wsum = 0.f;
  float acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += kCombChunk) {
    float ls[kCombChunk];
    float v[kCombChunk][DPL];
#pragma unroll
    for (int j = 0; j < kCombChunk; ++j) {
      // a CTA with an empty range wrote no partial: read the first piece's
      // (always written, finite) and give it weight 0
      const int s = s0 + j;
      const bool live = s < nseg && (all_live || cta_nonempty(c_first + s, T, a.C));
      const size_t sl = live ? slot0 + s : slot0;
      ls[j] = live ? __ldcg(p.part_lse + sl * kRowsPerCta + r) : -INFINITY;
      const float* src = p.part_o + (sl * kRowsPerCta + r) * D + lane * DPL;
      if constexpr (DPL == 4) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(src));
        v[j][0] = f.x; v[j][1] = f.y; v[j][2] = f.z; v[j][3] = f.w;
      } else {
        const float2 f = __ldcg(reinterpret_cast<const float2*>(src));
        v[j][0] = f.x; v[j][1] = f.y;
      }
    }
    float mc = M;
#pragma unroll
    for (int j = 0; j < kCombChunk; ++j) mc = fmaxf(mc, ls[j]);
    if (mc == -INFINITY) continue;
    const float f = M > -INFINITY ? __expf(M - mc) : 0.f;
    wsum *= f;
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc[t] *= f;
#pragma unroll
    for (int j = 0; j < kCombChunk; ++j) {
      const float w = ls[j] > -INFINITY ? __expf(ls[j] - mc) : 0.f;
      wsum += w;
#pragma unroll
      for (int t = 0; t < DPL; ++t) acc[t] = fmaf(w, v[j][t], acc[t]);
    }
    M = mc;
  }
  const int row = rg * kRowsPerCta + r;
  const int i = row / G, h = g * G + row % G;
  __nv_bfloat16* dst = p.out + (((size_t)b * a.n + i) * p.Hq + h) * D + lane * DPL;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int t = 0; t < DPL; t += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + t) = __floats2bfloat162_rn(acc[t] * inv, acc[t + 1] * inv);
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

// bf16 tensor map with 128-byte swizzle (box given by the caller).
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

template <int D>
static cudaError_t launch_tc(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                             const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                             int n, int Hq, int Hkv, int window, float scale, void* out, void* ws, cudaStream_t s,
                             const PagedKV* pg, bool early) {
  CUtensorMap mk, mv, mkt, mvt;
  const bool paged = pg != nullptr && pg->block_table != nullptr;
  if (paged) Lmax = pg->pages_per_seq * pg->page_size;  // a sequence's capacity
  const int Lrows = Lmax > 0 ? Lmax : 1;
  const void* kbase = Lmax > 0 ? kc : kt;  // any valid address when the cache is empty
  const void* vbase = Lmax > 0 ? vc : vt;
  if (paged) {
    // pools [num_pages][Hkv][page_size][D] as rows of D; a box is min(page_size, 64) keys
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)pg->num_pages * Hkv * pg->page_size};
    const cuuint64_t str[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(pg->page_size < kBN ? pg->page_size : kBN)};
    if (!make_map(&mk, kc, 2, dims, str, box) || !make_map(&mv, vc, 2, dims, str, box)) return cudaErrorInvalidValue;
  } else {
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
  const AttnWorkspace wl = attention_ws_layout(B, n, Hq, Hkv, D, Lmax, window);
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  TcParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.mask = mask;
  p.pos = pos;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.part_o = reinterpret_cast<float*>(wsb + wl.part_o_off);
  p.part_lse = reinterpret_cast<float*>(wsb + wl.part_lse_off);
  p.cta_status = reinterpret_cast<int*>(wsb + wl.cta_status_off);
  p.geo.plen = plen;
  p.geo.B = B;
  p.geo.Hkv = Hkv;
  p.geo.RG = attention_row_groups(n, Hq, Hkv);
  p.geo.n = n;
  p.geo.Lmax = Lmax;
  p.geo.window = window;
  p.geo.C = attention_ctas(B, n, Hq, Hkv, Lmax, window);
  p.geo.lo_align = paged ? kBN : 1;
  p.Hq = Hq;
  p.block_table = paged ? pg->block_table : nullptr;
  p.page_size = paged ? pg->page_size : 0;
  p.pages_per_seq = paged ? pg->pages_per_seq : 0;
  p.num_pages = paged ? pg->num_pages : 0;
  p.q_by_tma = q_tma ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.probe_ns = attention_wait_probe_ns();
  p.early = early ? 1 : 0;
  const size_t smem = TcLayout<D>::kSmemBytes;
  cudaError_t e = ensure_smem_limit((const void*)attn_tc_kernel<D>, smem);
  if (e != cudaSuccess) return e;

  // both kernels may start while their predecessor drains (programmatic
  // dependent launch); each waits in griddep_wait before reading its inputs
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.geo.C);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<D>, mk, mv, mkt, mvt, mq, p);
  if (e != cudaSuccess) return e;

  CombParams cp;
  cp.part_o = p.part_o;
  cp.part_lse = p.part_lse;
  cp.cta_status = p.cta_status;
  cp.status = reinterpret_cast<int*>(wsb + wl.status_off);
  cp.out = p.out;
  cp.geo = p.geo;
  cp.Hq = Hq;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3((unsigned)((size_t)B * Hkv * p.geo.RG), kRowsPerCta / kCombineWarps);
  cfg2.blockDim = dim3(kCombineThreads);
  cfg2.dynamicSmemBytes = 0;
  cfg2.stream = s;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg2, attn_combine_kernel<D>, cp);
}

cudaError_t launch_tree_attention(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                                  const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                                  int n, int Hq, int Hkv, int D, int window, float scale, void* out, void* ws,
                                  cudaStream_t s, const PagedKV* pg, bool early) {
  if (D == 128)
    return launch_tc<128>(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, window, scale, out, ws, s, pg,
                          early);
  return launch_tc<64>(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, window, scale, out, ws, s, pg, early);
}

}  // namespace eagle
