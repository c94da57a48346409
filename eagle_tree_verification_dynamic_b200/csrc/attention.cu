// Tree-masked split-KV attention ("Tree Attention" verification of the EAGLE
// notes, "3.Verify"; mask semantics from "Технический анализ EAGLE-4",
// section "Деревья проверки EAGLE-4 и утилита управления").
//
// Grid: (prefix splits + 1, Hkv, B).  A CTA owns one KV head of one sequence
// and one slice of its keys, and serves ALL n*G query rows of that head, so
// each key/value tile is read from HBM once.  The last split column holds
// the n tree keys, filtered by the ancestor bitmask.  Each CTA writes
// normalised partial outputs and their log-sum-exp; the combine kernel merges
// the splits: out = sum_s exp(lse_s - lse) * O_s, lse = logsumexp_s lse_s.
//
// This file is the CUDA-core path (fp32 dot products, online softmax); it
// serves every shape the library accepts.
#include <cstdlib>

#include "eagle_internal.h"

namespace eagle {

constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kRowsPerWarp = 4;
constexpr int kTileKeys = 32;

__device__ __forceinline__ float bf16_to_f(const __nv_bfloat16* p) {
  return __uint_as_float(((uint32_t)(*reinterpret_cast<const unsigned short*>(p))) << 16);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads)
attn_simt_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                 const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ plen, int Lmax,
                 const __nv_bfloat16* __restrict__ kt, const __nv_bfloat16* __restrict__ vt,
                 const uint64_t* __restrict__ mask, const int32_t* __restrict__ pos, int n, int Hq,
                 int Hkv, int window, float scale, int n_splits, int chunk,
                 float* __restrict__ part_o, float* __restrict__ part_lse) {
  constexpr int DPL = D / 32;  // dims per lane
  extern __shared__ float attn_smem[];
  float (*sK)[D + 1] = reinterpret_cast<float (*)[D + 1]>(attn_smem);
  float (*sV)[D] = reinterpret_cast<float (*)[D]>(attn_smem + kTileKeys * (D + 1));
  float (*sQ)[kRowsPerWarp][D] =
      reinterpret_cast<float (*)[kRowsPerWarp][D]>(attn_smem + kTileKeys * (2 * D + 1));

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z, B = gridDim.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = Hq / Hkv, rows = n * G;
  const int L = min(max(plen[b], 0), Lmax);
  const bool tree = (s == n_splits);
  int k0, k1;
  if (!tree) {
    const int lo = window > 0 ? max(0, L - window + 1) : 0;
    k0 = lo + s * chunk;
    k1 = min(L, k0 + chunk);
  } else {
    k0 = 0;
    k1 = n;
  }

  const int per_round = kAttnWarps * kRowsPerWarp;
  for (int base = 0; base < rows; base += per_round) {
    const int r0 = base + warp * kRowsPerWarp;
    // stage the warp's query rows
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int row = r0 + rr;
      if (row < rows) {
        const int i = row / G, h = g * G + row % G;
        const __nv_bfloat16* qp = q + (((size_t)b * n + i) * Hq + h) * D;
        for (int d = lane; d < D; d += 32) sQ[warp][rr][d] = bf16_to_f(qp + d) * scale;
      }
    }
    float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][DPL];
    int qpos[kRowsPerWarp];
    uint64_t mw0[kRowsPerWarp], mw1[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      m[rr] = -INFINITY;
      l[rr] = 0.f;
#pragma unroll
      for (int t = 0; t < DPL; ++t) o[rr][t] = 0.f;
      const int row = r0 + rr;
      const int i = row < rows ? row / G : 0;
      qpos[rr] = (window > 0 && row < rows) ? pos[(size_t)b * n + i] : 0;
      mw0[rr] = (tree && row < rows) ? mask[((size_t)b * n + i) * 2] : 0ull;
      mw1[rr] = (tree && row < rows) ? mask[((size_t)b * n + i) * 2 + 1] : 0ull;
    }

    for (int t0 = k0; t0 < k1; t0 += kTileKeys) {
      __syncthreads();
      for (int e = tid; e < kTileKeys * D; e += kAttnThreads) {
        const int kk = e / D, d = e - kk * D;
        const int j = t0 + kk;
        float kv = 0.f, vv = 0.f;
        if (j < k1) {
          const size_t off = tree ? (((size_t)b * n + j) * Hkv + g) * D + d
                                  : (((size_t)b * Hkv + g) * Lmax + j) * D + d;
          kv = bf16_to_f((tree ? kt : kc) + off);
          vv = bf16_to_f((tree ? vt : vc) + off);
        }
        sK[kk][d] = kv;
        sV[kk][d] = vv;
      }
      __syncthreads();
      const int j = t0 + lane;
#pragma unroll
      for (int rr = 0; rr < kRowsPerWarp; ++rr) {
        const int row = r0 + rr;
        if (row >= rows) continue;  // warp-uniform
        bool vis = j < k1;
        if (vis && tree) {
          const uint64_t w = lane + t0 < 64 ? mw0[rr] : mw1[rr];
          vis = (w >> ((t0 + lane) & 63)) & 1ull;
          if (vis && window > 0) vis = pos[(size_t)b * n + j] >= qpos[rr] - window + 1;
        } else if (vis && window > 0) {
          vis = j >= qpos[rr] - window + 1;
        }
        float sc = -INFINITY;
        if (vis) {
          float acc = 0.f;
#pragma unroll 8
          for (int d = 0; d < D; ++d) acc = fmaf(sQ[warp][rr][d], sK[lane][d], acc);
          sc = acc;
        }
        const float mx = warp_max_f(sc);
        const float m_new = fmaxf(m[rr], mx);
        if (m_new == -INFINITY) continue;  // nothing visible yet (warp-uniform)
        const float p = vis ? __expf(sc - m_new) : 0.f;
        const float corr = __expf(m[rr] - m_new);
        l[rr] = l[rr] * corr + warp_sum_f(p);
#pragma unroll
        for (int t = 0; t < DPL; ++t) o[rr][t] *= corr;
        for (int jj = 0; jj < kTileKeys; ++jj) {
          const float pj = __shfl_sync(kFull, p, jj);
#pragma unroll
          for (int t = 0; t < DPL; ++t) o[rr][t] = fmaf(pj, sV[jj][lane + 32 * t], o[rr][t]);
        }
        m[rr] = m_new;
      }
    }
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int row = r0 + rr;
      if (row >= rows) continue;
      const int i = row / G, h = g * G + row % G;
      const size_t slot = (((size_t)s * B + b) * n + i) * Hq + h;
      const float inv = l[rr] > 0.f ? 1.f / l[rr] : 0.f;
#pragma unroll
      for (int t = 0; t < DPL; ++t) part_o[slot * D + lane + 32 * t] = o[rr][t] * inv;
      if (lane == 0) part_lse[slot] = l[rr] > 0.f ? m[rr] + __logf(l[rr]) : -INFINITY;
    }
  }
}

// out[b][i][h][:] = sum_s w_s O_s / sum_s w_s, w_s = exp(lse_s - max lse).
// The split loops are unrolled so their independent loads are in flight together.
template <int D>
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                    int S, int B, int n, int Hq, __nv_bfloat16* __restrict__ out) {
  const int ih = blockIdx.x, b = blockIdx.y;
  const int i = ih / Hq, h = ih - i * Hq;
  const int d = threadIdx.x;
  const size_t stride = (size_t)B * n * Hq;  // between splits
  const size_t slot0 = ((size_t)b * n + i) * Hq + h;
  float mx = -INFINITY;
#pragma unroll 8
  for (int s = 0; s < S; ++s) mx = fmaxf(mx, part_lse[s * stride + slot0]);
  float num = 0.f, den = 0.f;
  if (mx > -INFINITY) {
#pragma unroll 8
    for (int s = 0; s < S; ++s) {
      const size_t slot = s * stride + slot0;
      const float w = __expf(part_lse[slot] - mx);
      den += w;
      num = fmaf(w, part_o[slot * D + d], num);
    }
  }
  out[slot0 * D + d] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
}

AttnPlan plan_attention(int B, int n, int Hq, int Hkv, int Lmax, int window) {
  AttnPlan p;
  p.span = window > 0 ? (Lmax < window ? Lmax : window) : Lmax;
  if (p.span < 1) p.span = 1;
  // two CTAs per SM: aim for ~2 x 148 CTAs over (row groups x heads x splits)
  const int heads = B * Hkv * attention_row_groups(n, Hq, Hkv);
  int splits = (2 * kNumSMs + heads - 1) / heads;
  const int max_splits = (p.span + 63) / 64;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int chunk = (p.span + splits - 1) / splits;
  chunk = (chunk + 63) / 64 * 64;
  p.chunk = chunk;
  p.n_splits = (p.span + chunk - 1) / chunk;
  return p;
}

// workspace: [256 B header: device error word][partial O][partial lse]
size_t attention_ws_bytes(int B, int n, int Hq, int Hkv, int D, int Lmax, int window) {
  const AttnPlan p = plan_attention(B, n, Hq, Hkv, Lmax, window);
  const size_t slots = (size_t)(p.n_splits + 1) * B * n * Hq;
  return 256 + align_up(slots * D * sizeof(float), 256) + align_up(slots * sizeof(float), 256);
}

cudaError_t launch_tree_attention(const void* q, const void* kc, const void* vc, const int32_t* plen, int Lmax,
                                  const void* kt, const void* vt, const uint64_t* mask, const int32_t* pos, int B,
                                  int n, int Hq, int Hkv, int D, int window, float scale, void* out, void* ws,
                                  cudaStream_t s) {
  const AttnPlan p = plan_attention(B, n, Hq, Hkv, Lmax, window);
  const size_t slots = (size_t)(p.n_splits + 1) * B * n * Hq;
  char* base = static_cast<char*>(ws);
  int* err = reinterpret_cast<int*>(base);
  float* part_o = reinterpret_cast<float*>(base + 256);
  float* part_lse = reinterpret_cast<float*>(base + 256 + align_up(slots * D * sizeof(float), 256));
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  using bf = __nv_bfloat16;
  static const bool simt = getenv("EAGLE_DEBUG_SIMT_ATTENTION") != nullptr;
  if (simt) {
    const dim3 grid(p.n_splits + 1, Hkv, B);
    const size_t smem =
        sizeof(float) * ((size_t)kTileKeys * (2 * D + 1) + (size_t)kAttnWarps * kRowsPerWarp * D);
    e = D == 128 ? ensure_smem_limit((const void*)attn_simt_kernel<128>, smem)
                 : ensure_smem_limit((const void*)attn_simt_kernel<64>, smem);
    if (e != cudaSuccess) return e;
    if (D == 128)
      attn_simt_kernel<128><<<grid, kAttnThreads, smem, s>>>(
          static_cast<const bf*>(q), static_cast<const bf*>(kc), static_cast<const bf*>(vc), plen, Lmax,
          static_cast<const bf*>(kt), static_cast<const bf*>(vt), mask, pos, n, Hq, Hkv, window, scale,
          p.n_splits, p.chunk, part_o, part_lse);
    else
      attn_simt_kernel<64><<<grid, kAttnThreads, smem, s>>>(
          static_cast<const bf*>(q), static_cast<const bf*>(kc), static_cast<const bf*>(vc), plen, Lmax,
          static_cast<const bf*>(kt), static_cast<const bf*>(vt), mask, pos, n, Hq, Hkv, window, scale,
          p.n_splits, p.chunk, part_o, part_lse);
    e = cudaGetLastError();
  } else {
    e = launch_attention_tc(q, kc, vc, plen, Lmax, kt, vt, mask, pos, B, n, Hq, Hkv, D, window, scale, p, part_o,
                            part_lse, err, s);
  }
  if (e != cudaSuccess) return e;
  const dim3 cgrid(n * Hq, B);
  if (D == 128)
    attn_combine_kernel<128><<<cgrid, 128, 0, s>>>(part_o, part_lse, p.n_splits + 1, B, n, Hq, static_cast<bf*>(out));
  else
    attn_combine_kernel<64><<<cgrid, 64, 0, s>>>(part_o, part_lse, p.n_splits + 1, B, n, Hq, static_cast<bf*>(out));
  return cudaGetLastError();
}

}  // namespace eagle
