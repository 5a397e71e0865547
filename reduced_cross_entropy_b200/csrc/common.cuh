// common.cuh -- small device helpers shared by the kernels of the RECE library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rece.h"

namespace rece {

// ---------------------------------------------------------------- element loads
// Inputs are fp32 (exact mode) or bf16; arithmetic is always fp32.  A bf16 value
// converts to fp32 exactly.
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Load 8 consecutive elements starting at p (16-byte aligned for bf16, 32 for fp32
// when the caller uses the vector path; the scalar path needs no alignment).
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// ---------------------------------------------------------------- ordering keys
// Monotone map fp32 -> uint32 (a < b  <=>  key(a) < key(b)) for finite values, with
// -0.0 folded onto +0.0 so that the two zeros compare equal.  Key 0 is below every
// finite value and marks "not a candidate".
__device__ __forceinline__ uint32_t score_key(float f) {
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t key) {
  uint32_t u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
  return __uint_as_float(u);
}

// 64-bit candidate order: larger = better = (higher score, then lower item id).
__device__ __forceinline__ uint64_t cand_key(uint32_t skey, int32_t item) {
  return (static_cast<uint64_t>(skey) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(item));
}
__device__ __forceinline__ int32_t cand_item(uint64_t ck) {
  return static_cast<int32_t>(~static_cast<uint32_t>(ck & 0xFFFFFFFFull));
}

// Chunk c of an M-long sorted array starts at ceil(c*M/n_c) (RECE, Algorithm 1).
__host__ __device__ __forceinline__ int64_t chunk_start(int64_t c, int64_t M, int64_t n_c) {
  return (c * M + n_c - 1) / n_c;
}

// ---------------------------------------------------------------- status word
__device__ __forceinline__ void raise_flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------- warp helpers
// Lanes of the warp whose value dg (in [0, 2^bits)) equals this lane's, from one ballot
// per bit (the peers agree with it on every bit); lanes with !ok match only themselves.
// All 32 lanes must call it.
__device__ __forceinline__ unsigned digit_peers(int dg, int bits, bool ok, int lane) {
  unsigned m = __ballot_sync(0xFFFFFFFFu, ok);
  for (int b = 0; b < bits; ++b) {
    const bool bit = (dg >> b) & 1;
    const unsigned v = __ballot_sync(0xFFFFFFFFu, bit);
    m &= bit ? v : ~v;
  }
  return ok ? m : (1u << lane);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

}  // namespace rece
