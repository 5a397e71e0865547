// projections.cu -- the random vectors B of steps 1-2 (RECE, section 3, Algorithm 1: the
// randn step), drawn on the device from (seed, step) by a counter-based stream, so that
// every element can be drawn by its own thread and a call is reproducible:
//
//   SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
//   OOPSLA 2014), state s, gamma G = 0x9E3779B97F4A7C15: output i = mix(s + (i + 1) G),
//   mix(z) = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
//   z ^= z >> 31.  The call's state is s = mix(mix(seed) ^ step).
//   Uniform from an output x: u = ((x >> 11) + 1) 2^-53, in (0, 1].
//   Box-Muller (Box and Muller 1958) for the pair q of elements: u1 = u(x_2q),
//   u2 = u(x_2q+1), rho = sqrt(-2 ln u1), theta = 2 pi u2 (2 pi as the double
//   6.283185307179586); element 2q = rho cos(theta), element 2q+1 = rho sin(theta), in
//   fp64, rounded to fp32 (and from there to bf16, nearest even, in bf16 mode).
//
// Elements follow B's row-major order [n_r][n_b][d]; with an odd count the last sine is
// not used.  One thread per pair.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

__device__ __forceinline__ uint64_t splitmix_mix(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

template <bool kBf16>
__global__ void __launch_bounds__(256) k_draw_projections(uint64_t s, int64_t count, void* B) {
  const int64_t pairs = (count + 1) / 2;
  for (int64_t q = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; q < pairs;
       q += int64_t(gridDim.x) * blockDim.x) {
    const uint64_t x1 = splitmix_mix(s + uint64_t(2 * q + 1) * 0x9E3779B97F4A7C15ull);
    const uint64_t x2 = splitmix_mix(s + uint64_t(2 * q + 2) * 0x9E3779B97F4A7C15ull);
    const double u1 = double((x1 >> 11) + 1) * 0x1.0p-53;
    const double u2 = double((x2 >> 11) + 1) * 0x1.0p-53;
    const double rho = sqrt(-2.0 * log(u1));
    const double theta = 6.283185307179586 * u2;
    const float z0 = float(rho * cos(theta));
    const float z1 = float(rho * sin(theta));
    const bool both = 2 * q + 1 < count;
    if constexpr (kBf16) {
      __nv_bfloat16* b = static_cast<__nv_bfloat16*>(B);
      b[2 * q] = __float2bfloat16_rn(z0);
      if (both) b[2 * q + 1] = __float2bfloat16_rn(z1);
    } else {
      float* b = static_cast<float*>(B);
      b[2 * q] = z0;
      if (both) b[2 * q + 1] = z1;
    }
  }
}

}  // namespace

cudaError_t launch_draw_projections(uint64_t seed, uint64_t step, int64_t count, bool bf16,
                                    void* B, cudaStream_t st) {
  if (count == 0) return cudaSuccess;
  // the call's state, on the host (the same function as the device's)
  auto mix = [](uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    z ^= z >> 31;
    return z;
  };
  const uint64_t s = mix(mix(seed) ^ step);
  const int64_t pairs = (count + 1) / 2;
  const int64_t want = (pairs + 255) / 256;
  const int grid = int(want < 8 * 148 ? want : 8 * 148);
  if (bf16)
    k_draw_projections<true><<<grid, 256, 0, st>>>(s, count, B);
  else
    k_draw_projections<false><<<grid, 256, 0, st>>>(s, count, B);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace rece
