// Device helpers shared by the tree-verification kernels: the Philox4x32-10
// uniforms of the acceptance walk, order-preserving integer keys for floats,
// warp reductions and the status word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/tree_verify.h"

namespace tv {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- status

__device__ __forceinline__ void set_status(uint32_t* st, uint32_t bits) {
  if (st != nullptr && bits != 0u) atomicOr(st, bits);
}

// ---------------------------------------------------------------- Philox
// Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel Random
// Numbers: As Easy as 1, 2, 3", SC'11): each round multiplies words 0 and 2
// by two fixed odd constants into 64-bit products and mixes the halves with
// words 1, 3 and the round key; the key advances by the Weyl constants
// between rounds.

struct Philox4 { uint32_t w[4]; };

__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
  const uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  const uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += kW0; k1 += kW1; }
    const uint32_t lo0 = kM0 * c0, hi0 = __umulhi(kM0, c0);
    const uint32_t lo1 = kM1 * c2, hi1 = __umulhi(kM1, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
  }
  Philox4 o; o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
  return o;
}

// Uniform in [0, 1) for one acceptance draw: counter (node, b, tag<<28 |
// draw, step), key = the 64-bit seed; 53 bits taken from words 0 and 1.
__device__ __forceinline__ double accept_uniform(uint64_t seed, uint64_t step, int b,
                                                 int node, int draw, int tag) {
  const Philox4 r = philox4x32_10(static_cast<uint32_t>(node), static_cast<uint32_t>(b),
                                  (static_cast<uint32_t>(tag) << 28) |
                                      (static_cast<uint32_t>(draw) & 0x0FFFFFFFu),
                                  static_cast<uint32_t>(step), static_cast<uint32_t>(seed),
                                  static_cast<uint32_t>(seed >> 32));
  const uint64_t bits = ((static_cast<uint64_t>(r.w[0]) << 32) | r.w[1]) >> 11;
  return static_cast<double>(bits) * 0x1.0p-53;
}

constexpr int kTagChild = 1;
constexpr int kTagResidual = 2;
constexpr int kTagSpecExec = 3;

// ---------------------------------------------------------------- keys
// Order-preserving maps: a < b  <=>  key(a) < key(b) (for non-NaN input).
// -0.0 and +0.0 compare equal, so they get one key (that of +0.0): equal
// values must tie and fall to the index tie-break.

__device__ __forceinline__ uint32_t f32_key(float x) {
  uint32_t u = __float_as_uint(x);
  u = (u == 0x80000000u) ? 0u : u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_f32(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}
__device__ __forceinline__ uint64_t f64_key(double x) {
  uint64_t u = static_cast<uint64_t>(__double_as_longlong(x));
  u = (u == 0x8000000000000000ull) ? 0ull : u;
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_f64(uint64_t k) {
  const uint64_t u = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
  return __longlong_as_double(static_cast<long long>(u));
}

// ---------------------------------------------------------------- reductions

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_sumf(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Inclusive prefix sum over the warp's lanes.
__device__ __forceinline__ double warp_incl_scan(double v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// ---------------------------------------------------------------- loads

// Four consecutive fp32 values starting at element e of a row of n values;
// positions >= n read `fill`.  vec: the row base is 16-byte aligned.
__device__ __forceinline__ float4 load4(const float* __restrict__ row, int e, int n,
                                        bool vec, float fill) {
  if (vec && e + 3 < n) return __ldg(reinterpret_cast<const float4*>(row + e));
  float4 v;
  v.x = (e + 0 < n) ? __ldg(row + e + 0) : fill;
  v.y = (e + 1 < n) ? __ldg(row + e + 1) : fill;
  v.z = (e + 2 < n) ? __ldg(row + e + 2) : fill;
  v.w = (e + 3 < n) ? __ldg(row + e + 3) : fill;
  return v;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

}  // namespace tv
