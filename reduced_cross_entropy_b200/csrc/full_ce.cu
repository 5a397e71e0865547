// full_ce.cu -- exact full cross-entropy, fused (RECE, equations 3 and 4).
//
// The logits are formed 64 x 64 at a time in registers and never stored:
//   forward   one CTA per 64 rows streams the whole catalogue, keeping an online
//             log-sum-exp per row (and picking up the positive logit on the way);
//   backward  recomputes each logit tile, turns it into g = (softmax - onehot) * dloss/N
//             in shared memory, and multiplies it into a 64 x 64 slice of dX (CTA per
//             rows x dims) or of dY (CTA per items x dims).  Every output element has
//             one owner and a fixed summation order: deterministic, no atomics.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kT = 64;   // rows / items per tile
constexpr int kTk = 32;  // depth staged per step

struct Smem {
  float a[kT][kTk + 1];
  float b[kT][kTk + 1];
};

// acc[i][j] = <A[r0 + ty + 16 i], B[c0 + tx + 16 j]>, fp32, t ascending.
template <typename T>
__device__ __forceinline__ void tile_dot(const T* __restrict__ A, int64_t nA, int64_t r0,
                                         const T* __restrict__ B, int64_t nB, int64_t c0, int d,
                                         Smem& s, float (&acc)[4][4]) {
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int t0 = 0; t0 < d; t0 += kTk) {
    __syncthreads();
    for (int e = tid; e < kT * kTk; e += 256) {
      const int rr = e / kTk, cc = e % kTk, t = t0 + cc;
      s.a[rr][cc] = (r0 + rr < nA && t < d) ? to_f32(A[(r0 + rr) * d + t]) : 0.0f;
      s.b[rr][cc] = (c0 + rr < nB && t < d) ? to_f32(B[(c0 + rr) * d + t]) : 0.0f;
    }
    __syncthreads();
    const int tmax = min(kTk, d - t0);
    for (int t = 0; t < tmax; ++t) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = s.a[ty + 16 * i][t];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = s.b[tx + 16 * j][t];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_full_ce_fwd(const T* __restrict__ X,
                                                     const T* __restrict__ Y,
                                                     const int32_t* __restrict__ targets,
                                                     int64_t N, int64_t C, int d,
                                                     float* __restrict__ row_loss,
                                                     float* __restrict__ lse_out,
                                                     uint32_t* status) {
  __shared__ Smem s;
  __shared__ float lpos[kT];
  __shared__ int zrow[kT];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t r0 = int64_t(blockIdx.x) * kT;
  if (tid < kT) {
    lpos[tid] = NAN;
    zrow[tid] = r0 + tid < N ? targets[r0 + tid] : -1;
  }
  float m[4], sum[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    sum[i] = 0.0f;
  }
  for (int64_t c0 = 0; c0 < C; c0 += kT) {
    float acc[4][4];
    tile_dot(X, N, r0, Y, C, c0, d, s, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t col = c0 + tx + 16 * j;
        if (col >= C) continue;
        const float v = acc[i][j];
        if (col == zrow[ty + 16 * i]) lpos[ty + 16 * i] = v;
        if (v > m[i]) {
          sum[i] = sum[i] * expf(m[i] - v) + 1.0f;
          m[i] = v;
        } else {
          sum[i] += expf(v - m[i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m[i], o);
      const float s2 = __shfl_xor_sync(0xFFFFFFFFu, sum[i], o);
      const float mm = fmaxf(m[i], m2);
      sum[i] = (m[i] == -INFINITY ? 0.0f : sum[i] * expf(m[i] - mm)) +
               (m2 == -INFINITY ? 0.0f : s2 * expf(m2 - mm));
      m[i] = mm;
    }
  }
  __syncthreads();
  if (tx == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = ty + 16 * i;
      const int64_t row = r0 + rr;
      if (row >= N) continue;
      const int z = zrow[rr];
      if (z < 0 || z >= C) {
        raise_flag(status, RECE_DEVICE_BAD_TARGET);
        lse_out[row] = NAN;
        row_loss[row] = NAN;
      } else {
        const float lse = m[i] + logf(sum[i]);
        lse_out[row] = lse;
        row_loss[row] = lse - lpos[rr];
      }
    }
  }
}

// dX (mode 0: A = X rows, B = Y items, out rows) or dY (mode 1: A = Y items, B = X rows).
// The CTA owns a 64-row slice of the output and 64 of its dims; it loops over the
// other side in 64-wide tiles.
template <typename T, int kMode>
__global__ void __launch_bounds__(256) k_full_ce_bwd(const T* __restrict__ X,
                                                     const T* __restrict__ Y,
                                                     const int32_t* __restrict__ targets,
                                                     const float* __restrict__ lse,
                                                     const float* __restrict__ dloss,
                                                     int64_t N, int64_t C, int d,
                                                     float* __restrict__ out) {
  __shared__ union {
    Smem s;
    float slice[kT][kT + 1];
  } u;
  __shared__ float g[kT][kT + 1];  // g[own][other]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t own0 = int64_t(blockIdx.x) * kT;
  const int dim0 = blockIdx.y * kT;
  const int64_t n_own = kMode == 0 ? N : C, n_other = kMode == 0 ? C : N;
  const T* own = kMode == 0 ? X : Y;
  const T* other = kMode == 0 ? Y : X;
  const float scale = N > 0 ? dloss[0] / float(N) : 0.0f;
  float res[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) res[i][j] = 0.0f;

  for (int64_t o0 = 0; o0 < n_other; o0 += kT) {
    float acc[4][4];  // acc[i][j]: own ty+16i, other tx+16j
    tile_dot(own, n_own, own0, other, n_other, o0, d, u.s, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t a = own0 + ty + 16 * i, b = o0 + tx + 16 * j;
        const int64_t row = kMode == 0 ? a : b, col = kMode == 0 ? b : a;
        float v = 0.0f;
        if (a < n_own && b < n_other) {
          const float p = expf(acc[i][j] - lse[row]);
          v = (col == targets[row] ? p - 1.0f : p) * scale;
        }
        g[ty + 16 * i][tx + 16 * j] = v;
      }
    }
    __syncthreads();
    for (int e = tid; e < kT * kT; e += 256) {  // slice of the other side's vectors
      const int rr = e / kT, cc = e % kT;
      const int64_t b = o0 + rr;
      const int t = dim0 + cc;
      u.slice[rr][cc] = (b < n_other && t < d) ? to_f32(other[b * d + t]) : 0.0f;
    }
    __syncthreads();
    for (int b = 0; b < kT; ++b) {
      float gv[4], sv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) gv[i] = g[ty + 16 * i][b];
#pragma unroll
      for (int j = 0; j < 4; ++j) sv[j] = u.slice[b][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) res[i][j] = fmaf(gv[i], sv[j], res[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t a = own0 + ty + 16 * i;
      const int t = dim0 + tx + 16 * j;
      if (a < n_own && t < d) out[a * d + t] = res[i][j];
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_full_ce_fwd(int64_t N, int64_t C, int d, const T* X, const T* Y,
                               const int32_t* targets, float* row_loss, float* lse,
                               uint32_t* status, cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  k_full_ce_fwd<T><<<unsigned(ceil_div(N, kT)), 256, 0, st>>>(X, Y, targets, N, C, d, row_loss,
                                                             lse, status);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_full_ce_bwd(int64_t N, int64_t C, int d, const T* X, const T* Y,
                               const int32_t* targets, const float* lse, const float* dloss,
                               float* dX, float* dY, cudaStream_t st) {
  const unsigned dims = unsigned(ceil_div(d, kT));
  if (N > 0) {
    k_full_ce_bwd<T, 0><<<dim3(unsigned(ceil_div(N, kT)), dims), 256, 0, st>>>(
        X, Y, targets, lse, dloss, N, C, d, dX);
    count_launches(1);
  }
  k_full_ce_bwd<T, 1><<<dim3(unsigned(ceil_div(C, kT)), dims), 256, 0, st>>>(
      X, Y, targets, lse, dloss, N, C, d, dY);
  count_launches(1);
  return cudaGetLastError();
}

#define RECE_INST(T)                                                                        \
  template cudaError_t launch_full_ce_fwd<T>(int64_t, int64_t, int, const T*, const T*,    \
                                             const int32_t*, float*, float*, uint32_t*,    \
                                             cudaStream_t);                                \
  template cudaError_t launch_full_ce_bwd<T>(int64_t, int64_t, int, const T*, const T*,    \
                                             const int32_t*, const float*, const float*,   \
                                             float*, float*, cudaStream_t);
RECE_INST(float)
RECE_INST(__nv_bfloat16)
#undef RECE_INST

}  // namespace rece
