// bucketize.cu -- step 1 of the path: bucket of every row = argmax over the random
// vectors of the inner product (RECE, section 3, Algorithm 1: the randn / argmax steps).
//
// CUDA-core version: every projection is the fixed-order chain
//   s = 0; for t = 0..d-1: s = fmaf(v[t], b[t], s)
// so the bucket ids are reproducible bit for bit.  A 64-row x 64-vector tile is
// register-blocked (4 x 4 per thread, d staged through shared memory 32 columns at a
// time, the chain order untouched), and the argmax is reduced in the epilogue so the
// (rows x n_b) projection matrix never leaves the chip.
#include <climits>

#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kTile = 64;
constexpr int kTk = 32;

// (score, index) order for the argmax: larger score wins; equal scores -> lower index.
__device__ __forceinline__ bool better(float s, int b, float s2, int b2) {
  return s > s2 || (s == s2 && b < b2);
}

template <typename T>
__global__ void __launch_bounds__(256) k_bucketize_fma(const T* __restrict__ V, int64_t M,
                                                       int d, const T* __restrict__ B, int n_b,
                                                       int32_t* __restrict__ bucket) {
  __shared__ float vs[kTile][kTk + 1];
  __shared__ float bs[kTile][kTk + 1];
  __shared__ float best_s[kTile];
  __shared__ int best_b[kTile];

  const int r = blockIdx.y;
  const T* Br = B + int64_t(r) * n_b * d;
  int32_t* out = bucket + int64_t(r) * M;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t row0 = int64_t(blockIdx.x) * kTile;

  if (tid < kTile) {
    best_s[tid] = -INFINITY;
    best_b[tid] = INT_MAX;
  }
  for (int b0 = 0; b0 < n_b; b0 += kTile) {
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

    for (int t0 = 0; t0 < d; t0 += kTk) {
      __syncthreads();
      for (int e = tid; e < kTile * kTk; e += 256) {
        const int rr = e / kTk, cc = e % kTk, t = t0 + cc;
        const int64_t row = row0 + rr;
        vs[rr][cc] = (row < M && t < d) ? to_f32(V[row * d + t]) : 0.0f;
        const int b = b0 + rr;
        bs[rr][cc] = (b < n_b && t < d) ? to_f32(Br[int64_t(b) * d + t]) : 0.0f;
      }
      __syncthreads();
      const int tmax = min(kTk, d - t0);
      for (int t = 0; t < tmax; ++t) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = vs[ty + 16 * i][t];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = bs[tx + 16 * j][t];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
    }
    // epilogue: argmax over this tile's vectors, merged into the running best
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float s = -INFINITY;
      int bb = INT_MAX;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int b = b0 + tx + 16 * j;
        if (b < n_b && better(acc[i][j], b, s, bb)) {
          s = acc[i][j];
          bb = b;
        }
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const float s2 = __shfl_xor_sync(0xFFFFFFFFu, s, o);
        const int b2 = __shfl_xor_sync(0xFFFFFFFFu, bb, o);
        if (better(s2, b2, s, bb)) {
          s = s2;
          bb = b2;
        }
      }
      const int rr = ty + 16 * i;
      if (tx == 0 && better(s, bb, best_s[rr], best_b[rr])) {
        best_s[rr] = s;
        best_b[rr] = bb;
      }
    }
  }
  __syncthreads();
  if (tid < kTile && row0 + tid < M) out[row0 + tid] = best_b[tid];
}

}  // namespace

template <typename T>
cudaError_t launch_bucketize_fma(const T* V, int64_t M, int d, const T* B, int n_b, int n_r,
                                 int32_t* bucket, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  dim3 grid(unsigned(ceil_div(M, kTile)), unsigned(n_r));
  k_bucketize_fma<T><<<grid, 256, 0, st>>>(V, M, d, B, n_b, bucket);
  count_launches(1);
  return cudaGetLastError();
}

template cudaError_t launch_bucketize_fma<float>(const float*, int64_t, int, const float*, int,
                                                 int, int32_t*, cudaStream_t);
template cudaError_t launch_bucketize_fma<__nv_bfloat16>(const __nv_bfloat16*, int64_t, int,
                                                         const __nv_bfloat16*, int, int,
                                                         int32_t*, cudaStream_t);

}  // namespace rece
