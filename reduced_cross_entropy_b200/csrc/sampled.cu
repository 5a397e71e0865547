// sampled.cu -- the sampled baselines of the RECE paper, section 2 (Related Work):
//   CE-  (equation 2): loss_i = log(exp(l+) + sum_j exp(l_ij)) - l+
//   BCE+ (equation 1): loss_i = -log sigmoid(l+) - sum_j log(1 - sigmoid(l_ij))
//                             = softplus(-l+) + sum_j softplus(l_ij)
// over n given negatives of every row (ids < 0 are padding; a sample equal to the
// positive is a negative like any other, as the sums are written), l = <x_i, y_j>.
//
// Forward: one warp per row; slot 0 is the positive, slot s >= 1 the negative
// neg[i][s-1].  Each lane forms whole dot products for its slots (x_i staged in shared
// memory in fp32; an fmaf chain in dimension order, as in the reduced loss's CUDA-core
// kernels), and the lanes' partial sums meet in a fixed xor tree: deterministic.  The
// logits go out [N][n+1] for the backward, which is the reduced loss's own
// (backward.cu) run over the sampled slots.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float softplus_f(float u) {
  return fmaxf(u, 0.0f) + log1pf(expf(-fabsf(u)));
}

template <typename T>
__device__ __forceinline__ float dot_x(const float* xs, const T* __restrict__ y, int d) {
  float s = 0.0f;
  if ((d & 7) == 0) {
    for (int t = 0; t < d; t += 8) {
      float v[8];
      load8(y + t, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) s = fmaf(xs[t + u], v[u], s);
    }
  } else {
    for (int t = 0; t < d; ++t) s = fmaf(xs[t], to_f32(y[t]), s);
  }
  return s;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_sampled_fwd(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ neg, int64_t N, int64_t C, int d, int n, int kind,
    float* __restrict__ logits, float* __restrict__ lse, float* __restrict__ row_loss,
    uint32_t* status) {
  extern __shared__ __align__(16) float sh_s[];
  const int warps = blockDim.x >> 5, wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slots = n + 1;
  float* xs = sh_s + size_t(d + slots) * wid;
  float* ls = xs + d;
  const int64_t i = int64_t(blockIdx.x) * warps + wid;
  if (i >= N) return;  // the warp leaves together; no block-wide barrier follows
  for (int t = lane; t < d; t += 32) xs[t] = to_f32(X[i * d + t]);
  __syncwarp();
  const int32_t z = targets[i];
  const bool zok = z >= 0 && z < C;
  float m = -INFINITY;
  for (int s = lane; s < slots; s += 32) {
    const int32_t j = s == 0 ? z : neg[i * n + (s - 1)];
    float l = -INFINITY;  // padding: no term
    if (j >= 0 && j < C) {
      l = dot_x(xs, Y + int64_t(j) * d, d);
      m = fmaxf(m, l);
    } else if (s == 0 || j >= C) {
      raise_flag(status, RECE_DEVICE_BAD_TARGET);
    }
    ls[s] = l;
    if (logits) logits[i * slots + s] = j >= 0 && j < C ? l : 0.0f;
  }
  __syncwarp();
  float part = 0.0f;
  if (kind == 0) {
    m = warp_max(m);
    for (int s = lane; s < slots; s += 32)
      if (ls[s] != -INFINITY) part += expf(ls[s] - m);
    const float li = m + logf(warp_sum(part));
    if (lane == 0) {
      lse[i] = zok ? li : 0.0f;
      row_loss[i] = zok ? li - ls[0] : 0.0f;
    }
  } else {
    for (int s = lane; s < slots; s += 32)
      if (ls[s] != -INFINITY) part += softplus_f(s == 0 ? -ls[s] : ls[s]);
    const float tot = warp_sum(part);
    if (lane == 0) {
      if (lse) lse[i] = 0.0f;
      row_loss[i] = zok ? tot : 0.0f;
    }
  }
}

}  // namespace

size_t sampled_fwd_warp_bytes(int d, int n) { return sizeof(float) * size_t(d + n + 1); }

template <typename T>
cudaError_t launch_sampled_fwd(int kind, int64_t N, int64_t C, int d, int n, const T* X,
                               const T* Y, const int32_t* targets, const int32_t* neg,
                               float* logits, float* lse, float* row_loss, uint32_t* status,
                               cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  const size_t per_warp = sampled_fwd_warp_bytes(d, n);
  int warps = int((200 * 1024) / per_warp);
  warps = warps < 1 ? 1 : (warps > kThreads / 32 ? kThreads / 32 : warps);
  const size_t smem = per_warp * warps;
  cudaError_t e = cudaFuncSetAttribute(k_sampled_fwd<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_sampled_fwd<T><<<unsigned(ceil_div(N, warps)), warps * 32, smem, st>>>(
      X, Y, targets, neg, N, C, d, n, kind, logits, lse, row_loss, status);
  count_launches(1);
  return cudaGetLastError();
}

template cudaError_t launch_sampled_fwd<float>(int, int64_t, int64_t, int, int, const float*,
                                               const float*, const int32_t*, const int32_t*,
                                               float*, float*, float*, uint32_t*,
                                               cudaStream_t);
template cudaError_t launch_sampled_fwd<__nv_bfloat16>(int, int64_t, int64_t, int, int,
                                                       const __nv_bfloat16*,
                                                       const __nv_bfloat16*, const int32_t*,
                                                       const int32_t*, float*, float*, float*,
                                                       uint32_t*, cudaStream_t);

}  // namespace rece
