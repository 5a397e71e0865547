// window_fma.cu -- the all-negatives mode (Algorithm 1 of the RECE paper as printed,
// section 3, and the rounds paragraph) on the CUDA cores: every item of a row's chunk
// windows is a negative, and a pair computed in cnt of the n_r rounds enters each round's
// sum as exp(l - ln cnt) = exp(l) / cnt, the positive left out of the window sums.
//
// These kernels serve the fp32 exact mode, the bf16 mode with RECE_FLAG_FMA_SCORES, and
// the bf16 widths the tcgen05 window kernels (window_tc.cu) do not take.  Every score is
// the fixed-order chain s = fmaf(x[t], y[t], s), t = 0..d-1 from s = 0, the same in all
// three kernels, so a pair's score in the backward is bit for bit the forward's.
//
//   k_window_lse_fma  warp per (round r, sorted row p): over the items q of the row's
//                     round-r window, (max, sum of exp(s - max) / cnt) -- the pair of the
//                     window terms that k_window_combine folds into lse with l+
//   k_window_dx_fma   warp per (round r, sorted row p): dX_i += sum_q g_iq y_q,
//                     g = exp(s - lse_i) / cnt * dloss / N, items in position order
//   k_window_dy_fma   warp per (round r, sorted catalogue position q): dY_j += sum_p g_pj
//                     x_p over the sorted rows whose round-r window holds q, in row order
// Lanes split the window (or the rows) for the scores; the sums over items (rows) are
// taken in a fixed order -- a fixed xor tree for (max, sum), item by item for the
// gradients, each lane owning dimensions t = lane, lane + 32, ... -- and the rounds add
// one launch each, after the positives' terms: deterministic.
//
// cnt of a pair (row at p, item at q, both in round r's orders) is the number of rounds
// s whose window of the row holds the item: |chunk_s(row) - chunk_s(item)| <= n_ec, the
// chunks read from the tables k_window_meta writes (rowc, itemc); the round r itself
// always counts, so cnt >= 1.
#include "common.cuh"
#include "plan.h"
#include "tc.h"

namespace rece {
namespace {

__device__ __forceinline__ int64_t chunk_of(int64_t p, int64_t M, int n_c) {
  return (p * n_c) / M;
}

// Rounds whose window of the row at sorted position p holds the item at position q (both
// positions in round r's orders).
__device__ __forceinline__ int pair_rounds(const int32_t* __restrict__ rowc,
                                           const int32_t* __restrict__ itemc, int r, int64_t p,
                                           int64_t q, int64_t N, int64_t C, int n_r, int n_ec) {
  int cnt = 0;
  for (int s = 0; s < n_r; ++s) {
    const int dc = rowc[(int64_t(r) * n_r + s) * N + p] - itemc[(int64_t(r) * n_r + s) * C + q];
    cnt += (dc >= -n_ec && dc <= n_ec) ? 1 : 0;
  }
  return cnt;
}

// The fixed-order fmaf chain of a (shared-memory, fp32) row against a row of V.
template <typename T>
__device__ __forceinline__ float chain(const float* __restrict__ a, const T* __restrict__ v,
                                       int d) {
  float s = 0.0f;
  for (int t = 0; t < d; ++t) s = fmaf(a[t], to_f32(v[t]), s);
  return s;
}

template <typename T>
__global__ void __launch_bounds__(256) k_window_lse_fma(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ px,
    const int32_t* __restrict__ py, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ itemc, const int32_t* __restrict__ rowc, int64_t N, int64_t C,
    int d, int n_c, int n_ec, int n_r, float2* __restrict__ ms) {
  extern __shared__ float sh[];
  const int warps = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xr = sh + size_t(w) * d;
  const int64_t total = int64_t(n_r) * N;
  for (int64_t e = int64_t(blockIdx.x) * warps + w; e < total; e += int64_t(gridDim.x) * warps) {
    const int r = int(e / N);
    const int64_t p = e - int64_t(r) * N;
    const int32_t i = px[e];
    const int32_t z = targets[i];
    for (int t = lane; t < d; t += 32) xr[t] = to_f32(X[int64_t(i) * d + t]);
    __syncwarp();
    const int64_t c = chunk_of(p, N, n_c);
    const int64_t w0 = chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c);
    const int64_t w1 = chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c);
    float m = -INFINITY, sum = 0.0f;
    for (int64_t q = w0 + lane; q < w1; q += 32) {
      const int32_t j = py[int64_t(r) * C + q];
      if (j == z) continue;
      const int cnt = pair_rounds(rowc, itemc, r, p, q, N, C, n_r, n_ec);
      const float s = chain(xr, Y + int64_t(j) * d, d);
      const float wgt = 1.0f / float(cnt);
      if (s > m) {
        sum = sum * expf(m - s) + wgt;
        m = s;
      } else {
        sum += wgt * expf(s - m);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
      const float s2 = __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      const float M = fmaxf(m, m2);
      sum = (m == -INFINITY ? 0.0f : sum * expf(m - M)) + (m2 == -INFINITY ? 0.0f : s2 * expf(m2 - M));
      m = M;
    }
    if (lane == 0) ms[e] = make_float2(m, sum);
    __syncwarp();  // xr is rewritten by the next row
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_window_dx_fma(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ px,
    const int32_t* __restrict__ py, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ itemc, const int32_t* __restrict__ rowc,
    const float* __restrict__ lse, const float* __restrict__ dloss, int64_t N, int64_t C, int d,
    int n_c, int n_ec, int n_r, int r, float* __restrict__ dX) {
  extern __shared__ float sh[];
  const int warps = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* xr = sh + size_t(w) * 2 * d;
  float* acc = xr + d;
  const float scale = dloss[0] / float(N);
  for (int64_t p = int64_t(blockIdx.x) * warps + w; p < N; p += int64_t(gridDim.x) * warps) {
    const int32_t i = px[int64_t(r) * N + p];
    const int32_t z = targets[i];
    const float li = lse[i];
    for (int t = lane; t < d; t += 32) {
      xr[t] = to_f32(X[int64_t(i) * d + t]);
      acc[t] = 0.0f;
    }
    __syncwarp();
    const int64_t c = chunk_of(p, N, n_c);
    const int64_t w0 = chunk_start(c - n_ec < 0 ? 0 : c - n_ec, C, n_c);
    const int64_t w1 = chunk_start(c + n_ec + 1 > n_c ? n_c : c + n_ec + 1, C, n_c);
    for (int64_t q0 = w0; q0 < w1; q0 += 32) {
      const int64_t q = q0 + lane;
      float g = 0.0f;
      int32_t j = 0;
      if (q < w1) {
        j = py[int64_t(r) * C + q];
        if (j != z) {
          const int cnt = pair_rounds(rowc, itemc, r, p, q, N, C, n_r, n_ec);
          g = expf(chain(xr, Y + int64_t(j) * d, d) - li) / float(cnt) * scale;
        }
      }
      for (int u = 0; u < 32; ++u) {
        const float gu = __shfl_sync(0xFFFFFFFFu, g, u);
        const int32_t ju = __shfl_sync(0xFFFFFFFFu, j, u);
        if (gu != 0.0f) {  // (uniform: every lane holds the same gu)
          const T* y = Y + int64_t(ju) * d;
          for (int t = lane; t < d; t += 32) acc[t] = fmaf(gu, to_f32(y[t]), acc[t]);
        }
      }
    }
    for (int t = lane; t < d; t += 32) dX[int64_t(i) * d + t] += acc[t];
    __syncwarp();
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_window_dy_fma(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ px,
    const int32_t* __restrict__ py, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ itemc, const int32_t* __restrict__ rowc,
    const float* __restrict__ lse, const float* __restrict__ dloss, int64_t N, int64_t C, int d,
    int n_c, int n_ec, int n_r, int r, float* __restrict__ dY) {
  extern __shared__ float sh[];
  const int warps = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* yr = sh + size_t(w) * 2 * d;
  float* acc = yr + d;
  const float scale = dloss[0] / float(N);
  for (int64_t q = int64_t(blockIdx.x) * warps + w; q < C; q += int64_t(gridDim.x) * warps) {
    const int32_t j = py[int64_t(r) * C + q];
    for (int t = lane; t < d; t += 32) {
      yr[t] = to_f32(Y[int64_t(j) * d + t]);
      acc[t] = 0.0f;
    }
    __syncwarp();
    // the sorted rows whose round-r window holds q: chunks within n_ec of q's chunk
    const int64_t cq = chunk_of(q, C, n_c);
    const int64_t h0 = chunk_start(cq - n_ec < 0 ? 0 : cq - n_ec, N, n_c);
    const int64_t h1 = chunk_start(cq + n_ec + 1 > n_c ? n_c : cq + n_ec + 1, N, n_c);
    for (int64_t p0 = h0; p0 < h1; p0 += 32) {
      const int64_t p = p0 + lane;
      float g = 0.0f;
      int32_t i = 0;
      if (p < h1) {
        i = px[int64_t(r) * N + p];
        if (targets[i] != j) {
          const int cnt = pair_rounds(rowc, itemc, r, p, q, N, C, n_r, n_ec);
          // fmaf(x, y, s) == fmaf(y, x, s): the forward's score exactly
          g = expf(chain(yr, X + int64_t(i) * d, d) - lse[i]) / float(cnt) * scale;
        }
      }
      for (int u = 0; u < 32; ++u) {
        const float gu = __shfl_sync(0xFFFFFFFFu, g, u);
        const int32_t iu = __shfl_sync(0xFFFFFFFFu, i, u);
        if (gu != 0.0f) {
          const T* x = X + int64_t(iu) * d;
          for (int t = lane; t < d; t += 32) acc[t] = fmaf(gu, to_f32(x[t]), acc[t]);
        }
      }
    }
    for (int t = lane; t < d; t += 32) dY[int64_t(j) * d + t] += acc[t];
    __syncwarp();
  }
}

// Warps per block so that `rows` fp32 rows of d per warp fit the shared memory given.
int warps_for(int d, int rows) {
  const size_t per = size_t(rows) * d * sizeof(float);
  int w = int((200 * 1024) / (per > 0 ? per : 1));
  return w > 8 ? 8 : (w < 1 ? 1 : w);
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
}

}  // namespace

template <typename T>
cudaError_t launch_window_lse_fma(const rece_plan_s& p, const T* X, const T* Y,
                                  const int32_t* px, const int32_t* py, const int32_t* targets,
                                  const int32_t* itemc, const int32_t* rowc, float2* ms,
                                  cudaStream_t st) {
  const auto& c = p.cfg;
  const int64_t total = int64_t(c.n_r) * c.N;
  if (total == 0) return cudaSuccess;
  const int warps = warps_for(c.d, 1);
  const size_t smem = size_t(warps) * c.d * sizeof(float);
  cudaError_t e = set_smem(k_window_lse_fma<T>, smem);
  if (e != cudaSuccess) return e;
  const int64_t want = ceil_div(total, warps);
  k_window_lse_fma<T><<<unsigned(want < 16 * 148 ? want : 16 * 148), 32 * warps, smem, st>>>(
      X, Y, px, py, targets, itemc, rowc, c.N, c.C, c.d, c.n_c, c.n_ec, c.n_r, ms);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_window_grad_fma(const rece_plan_s& p, bool dy, const T* X, const T* Y,
                                   const int32_t* px, const int32_t* py, const int32_t* targets,
                                   const int32_t* itemc, const int32_t* rowc, const float* lse,
                                   const float* dloss, float* out, cudaStream_t st) {
  const auto& c = p.cfg;
  const int64_t M = dy ? c.C : c.N;
  if (c.N == 0 || M == 0) return cudaSuccess;
  const int warps = warps_for(c.d, 2);
  const size_t smem = size_t(warps) * 2 * c.d * sizeof(float);
  cudaError_t e = dy ? set_smem(k_window_dy_fma<T>, smem) : set_smem(k_window_dx_fma<T>, smem);
  if (e != cudaSuccess) return e;
  const int64_t want = ceil_div(M, warps);
  const unsigned grid = unsigned(want < 16 * 148 ? want : 16 * 148);
  for (int r = 0; r < c.n_r; ++r) {  // the rounds add in order
    if (dy)
      k_window_dy_fma<T><<<grid, 32 * warps, smem, st>>>(X, Y, px, py, targets, itemc, rowc,
                                                         lse, dloss, c.N, c.C, c.d, c.n_c,
                                                         c.n_ec, c.n_r, r, out);
    else
      k_window_dx_fma<T><<<grid, 32 * warps, smem, st>>>(X, Y, px, py, targets, itemc, rowc,
                                                         lse, dloss, c.N, c.C, c.d, c.n_c,
                                                         c.n_ec, c.n_r, r, out);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

#define RECE_WINDOW_FMA(T)                                                                    \
  template cudaError_t launch_window_lse_fma<T>(const rece_plan_s&, const T*, const T*,       \
                                                const int32_t*, const int32_t*,               \
                                                const int32_t*, const int32_t*,               \
                                                const int32_t*, float2*, cudaStream_t);       \
  template cudaError_t launch_window_grad_fma<T>(const rece_plan_s&, bool, const T*, const T*, \
                                                 const int32_t*, const int32_t*,              \
                                                 const int32_t*, const int32_t*,              \
                                                 const int32_t*, const float*, const float*,  \
                                                 float*, cudaStream_t);
RECE_WINDOW_FMA(float)
RECE_WINDOW_FMA(__nv_bfloat16)
#undef RECE_WINDOW_FMA

}  // namespace rece
