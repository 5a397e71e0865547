// window.cu -- the small kernels around the all-negatives mode (Algorithm 1 of the RECE
// paper as printed, section 3: every item of a row's chunk window is a negative; the
// rounds paragraph: a pair computed in cnt of the rounds enters every round's sum as
// exp(l - ln cnt)).  The tensor-core kernels are in window_tc.cu; here:
//
//   k_window_meta     per round r and sorted position p: the chunk, in every round s, of
//                     the row (item) at p -- chunks[(r * n_r + s) * M + p] -- from which a
//                     pair's round count is a handful of integer compares; for the rows
//                     also the sorted position, in round r, of their positive
//   k_window_combine  per row: l+ = <x_i, y_{z_i}>, and lse_i from l+ and the rounds'
//                     partial (max, sum) pairs of the window terms; the row loss
//                     lse_i - l+; lse again in every round's sorted order for the backward
#include "common.cuh"
#include "plan.h"
#include "tc.h"

namespace rece {
namespace {

__global__ void __launch_bounds__(256) k_window_meta(
    const int32_t* __restrict__ perm, const int32_t* __restrict__ inv, int64_t M, int n_c,
    int n_r, int32_t* __restrict__ chunks, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ invY, int64_t C, int32_t* __restrict__ pz) {
  const int64_t total = int64_t(n_r) * M;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    const int r = int(e / M);
    const int64_t p = e - int64_t(r) * M;
    const int32_t id = perm[e];
    for (int s = 0; s < n_r; ++s)
      chunks[(int64_t(r) * n_r + s) * M + p] =
          int32_t((int64_t(inv[int64_t(s) * M + id]) * n_c) / M);
    if (pz) {
      const int32_t z = targets[id];
      pz[e] = (z >= 0 && z < C) ? invY[int64_t(r) * C + z] : -1;
    }
  }
}

// One warp per row.
template <typename T>
__global__ void __launch_bounds__(256) k_window_combine(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ invX, const float2* __restrict__ ms, int64_t N, int64_t C,
    int d, int n_r, float* __restrict__ lse, float* __restrict__ row_loss,
    float* __restrict__ lse_sorted, uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= N) return;
  const int32_t z = targets[i];
  if (z < 0 || z >= C) {
    if (lane == 0) {
      raise_flag(status, RECE_DEVICE_BAD_TARGET);
      lse[i] = NAN;
      row_loss[i] = NAN;
      for (int r = 0; r < n_r; ++r) lse_sorted[int64_t(r) * N + invX[int64_t(r) * N + i]] = NAN;
    }
    return;
  }
  float part = 0.0f;
  for (int t = lane; t < d; t += 32)
    part = fmaf(to_f32(X[i * d + t]), to_f32(Y[int64_t(z) * d + t]), part);
  const float lp = warp_sum(part);
  if (lane != 0) return;
  float m = lp;
  for (int r = 0; r < n_r; ++r) {
    const float2 v = ms[int64_t(r) * N + invX[int64_t(r) * N + i]];
    if (v.y > 0.0f) m = fmaxf(m, v.x);
  }
  float s = expf(lp - m);
  for (int r = 0; r < n_r; ++r) {
    const float2 v = ms[int64_t(r) * N + invX[int64_t(r) * N + i]];
    if (v.y > 0.0f) s += v.y * expf(v.x - m);
  }
  const float li = m + logf(s);
  lse[i] = li;
  row_loss[i] = li - lp;
  for (int r = 0; r < n_r; ++r) lse_sorted[int64_t(r) * N + invX[int64_t(r) * N + i]] = li;
}

}  // namespace

cudaError_t launch_window_meta(const int32_t* perm, const int32_t* inv, int64_t M, int n_c,
                               int n_r, int32_t* chunks, const int32_t* targets,
                               const int32_t* invY, int64_t C, int32_t* pz, cudaStream_t st) {
  const int64_t total = int64_t(n_r) * M;
  if (total == 0) return cudaSuccess;
  const int64_t want = (total + 255) / 256;
  k_window_meta<<<unsigned(want < 16 * 148 ? want : 16 * 148), 256, 0, st>>>(
      perm, inv, M, n_c, n_r, chunks, targets, invY, C, pz);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_window_combine(const rece_plan_s& p, const T* X, const T* Y,
                                  const int32_t* targets, const int32_t* invX, const float2* ms,
                                  float* lse, float* row_loss, float* lse_sorted,
                                  uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  k_window_combine<T><<<unsigned(ceil_div(c.N, 8)), 256, 0, st>>>(
      X, Y, targets, invX, ms, c.N, c.C, c.d, c.n_r, lse, row_loss, lse_sorted, status);
  count_launches(1);
  return cudaGetLastError();
}

template cudaError_t launch_window_combine<float>(
    const rece_plan_s&, const float*, const float*, const int32_t*, const int32_t*,
    const float2*, float*, float*, float*, uint32_t*, cudaStream_t);
template cudaError_t launch_window_combine<__nv_bfloat16>(
    const rece_plan_s&, const __nv_bfloat16*, const __nv_bfloat16*, const int32_t*,
    const int32_t*, const float2*, float*, float*, float*, uint32_t*, cudaStream_t);

}  // namespace rece
