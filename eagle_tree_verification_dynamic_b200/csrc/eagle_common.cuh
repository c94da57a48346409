// Device-side building blocks shared by the kernels of libeagle_tree.
//
//  * order keys: a float value and a token id packed into one uint64 whose
//    unsigned order is "larger value first, then lower id first", which is the
//    tie rule for every top-k and argmax in the library;
//  * warp-wide bitonic sort / merge of such keys (one key per lane);
//  * base-2 scaled partial sums for log-sum-exp: a chunk of logits reports
//    (e_ref, acc) with acc = sum_i 2^(x_i*log2(e) - e_ref) in fp64; e_ref is an
//    integer, so rescaling between chunks is an exact power-of-two multiply.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace eagle {

constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------- programmatic dependent launch
// Every kernel of the library calls griddep_wait() before it touches global
// memory: launched with programmatic stream serialization it may start while
// its predecessor on the stream drains, and this blocks until that grid has
// completed and its memory is visible (a no-op for an ordinary launch).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the grids that depend on this one be scheduled (they still wait in
// griddep_wait before reading anything this grid writes).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// log2(e) as an unevaluated sum of two fp32 numbers (the head is log2(e)
// rounded to fp32, the tail is the remainder rounded to fp32: the double-float
// representation of a constant used in Dekker's and Cody-Waite's techniques),
// good to about 48 bits.  x*log2(e) is formed as fma(x, kLog2eHi, x*kLog2eLo)
// so that the head's fp32 rounding does not bias every exponent of a row by
// the same relative amount.
constexpr float kLog2eHi = 1.4426950216293335f;
constexpr float kLog2eLo = 1.925963033500011e-08f;
constexpr double kLn2 = 0.69314718055994530942;

// ---------------------------------------------------------------- order keys
__device__ __forceinline__ uint32_t order_bits(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;  // -0 ranks with +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_value(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}
// Larger key = better.  Key 0 means "no element" (every real key is > 0).
__device__ __forceinline__ uint64_t make_key(float v, int idx) {
  return ((uint64_t)order_bits(v) << 32) | (uint64_t)(~(uint32_t)idx);
}
__device__ __forceinline__ int key_index(uint64_t k) { return (int)(~(uint32_t)k); }
__device__ __forceinline__ float key_value(uint64_t k) { return order_value((uint32_t)(k >> 32)); }

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }
__device__ __forceinline__ uint64_t umin64(uint64_t a, uint64_t b) { return a < b ? a : b; }

// Sort one key per lane so that lane 0 holds the largest (bitonic network).
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
    const bool desc = (lane & size) == 0;
#pragma unroll
    for (int j = size >> 1; j > 0; j >>= 1) {
      const uint64_t o = __shfl_xor_sync(kFull, v, j);
      const bool lower = (lane & j) == 0;
      v = (lower == desc) ? umax64(v, o) : umin64(v, o);
    }
  }
  return v;
}

// list and batch each sorted descending across the warp -> the 32 largest of
// their union, sorted descending.
__device__ __forceinline__ uint64_t warp_merge_desc(uint64_t list, uint64_t batch) {
  const int lane = threadIdx.x & 31;
  uint64_t v = umax64(list, __shfl_sync(kFull, batch, 31 - lane));
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t o = __shfl_xor_sync(kFull, v, j);
    v = ((lane & j) == 0) ? umax64(v, o) : umin64(v, o);
  }
  return v;
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = umax64(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Ranking key of a candidate: the order-preserving bit image of its fp64
// log V with the lowest 12 mantissa bits replaced by (4095 - id), so that a
// larger key means a larger log V and, among equal values, a lower id.  Two
// values that differ only in those 12 bits (relative gap < 2^-40) rank by id.
__device__ __forceinline__ uint64_t cand_key(double lv, int gid) {
  uint64_t u = (uint64_t)__double_as_longlong(lv);
  if (u == 0x8000000000000000ull) u = 0;  // -0 ranks with +0
  u = (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
  return (u & ~0xfffull) | (uint64_t)(4095 - gid);
}
__device__ __forceinline__ int key_gid(uint64_t key) { return 4095 - (int)(key & 0xfffull); }

// ------------------------------------------------------- scaled exp partials
// Partial sum of one chunk: acc = sum 2^(x*log2e - e_ref), e_ref an integer
// (as float; -inf when the chunk held no finite term).
struct ChunkStat {
  float e_ref;
  int pad;
  double acc;
};

// 2^z by the hardware approximation (about 2 ulp; results below 2^-126 flush
// to zero).  Every sum built from it is dominated by terms near 2^0, so a
// flushed term is far below the fp64 rounding of the sum.
__device__ __forceinline__ float ex2_ftz(float z) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(z));
  return y;
}

__device__ __forceinline__ float exp2_scaled(float x, float e_ref) {
  float z = fmaf(x, kLog2eHi, -e_ref);
  z = fmaf(x, kLog2eLo, z);
  return ex2_ftz(z);
}

// acc * 2^(from - to) for integer-valued from <= to (exact; the same rounding
// as ldexp when the result is subnormal).  For d = from - to >= -1022 the
// power of two is assembled from its exponent bits (d + 1.5 * 2^23 holds the
// integer d in its low mantissa bits); below that ldexp handles it.
__device__ __forceinline__ double rescale_pow2(double acc, float from, float to) {
  const float d = from - to;
  if (d >= -1022.0f) {
    const int di = __float_as_int(d + 12582912.0f) - 0x4B400000;
    return acc * __longlong_as_double((long long)(1023 + di) << 52);
  }
  return ldexp(acc, (int)fmaxf(d, -1100.0f));
}

// Merge (e_ref, acc) pairs; returns the natural-log total (fp64).
struct LseAccum {
  float e;
  double s;
  __device__ __forceinline__ void init() { e = -INFINITY; s = 0.0; }
  __device__ __forceinline__ void add(float e2, double s2) {
    if (s2 == 0.0) return;
    if (e2 > e) { s = rescale_pow2(s, e, e2); e = e2; }
    else        { s2 = rescale_pow2(s2, e2, e); }
    s += s2;
  }
  __device__ __forceinline__ double lse() const {
    return s > 0.0 ? kLn2 * ((double)e + log2(s)) : -INFINITY;
  }
};

// Split a double into fp32 head + tail (head + tail == v to ~48 bits).
struct Split2 {
  float hi, lo;
  __device__ __forceinline__ void set(double v) {
    hi = (float)v;
    lo = (float)(v - (double)hi);
  }
};

// exp(x - lse) for one logit given lse as a head/tail pair, in fp32 with the
// subtraction and the base change carried to ~fp32 accuracy of the result.
__device__ __forceinline__ float exp_minus(float x, Split2 lse) {
  float d = (x - lse.hi) - lse.lo;
  return ex2_ftz(fmaf(d, kLog2eHi, d * kLog2eLo));
}

// ------------------------------------------------------------------ loading
template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;
  __device__ static __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static __forceinline__ float load(const float* p) { return __ldg(p); }
  // the largest element of a vector (NaN ignored, as fmaxf does)
  __device__ static __forceinline__ float vec_max(const uint4& u) {
    return fmaxf(fmaxf(__uint_as_float(u.x), __uint_as_float(u.y)), fmaxf(__uint_as_float(u.z), __uint_as_float(u.w)));
  }
  __device__ static __forceinline__ uint4 neg_inf_vec() { return make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u); }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ static __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
  }
  __device__ static __forceinline__ float load(const __nv_bfloat16* p) {
    const unsigned short s = __ldg(reinterpret_cast<const unsigned short*>(p));
    return __uint_as_float(((uint32_t)s) << 16);
  }
  // the largest element of a vector: packed bf16x2 maxima (a NaN operand
  // yields the other one), then the larger half
  __device__ static __forceinline__ float vec_max(const uint4& u) {
    uint32_t m01, m23, m;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m01) : "r"(u.x), "r"(u.y));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m23) : "r"(u.z), "r"(u.w));
    asm("max.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(m01), "r"(m23));
    return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
  }
  __device__ static __forceinline__ uint4 neg_inf_vec() { return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u); }
};

// Streaming 16-byte load that does not keep the line in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

}  // namespace eagle
