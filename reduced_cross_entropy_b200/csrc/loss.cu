// loss.cu -- steps 4 (round merge) and 5 (loss) of the path.
//
// Per row (one CTA): the n_r per-round lists are united; an item found in several
// rounds is kept once with its higher score (the RECE paper subtracts ln(count) from a
// logit seen count times, which leaves the same softmax); the k best by (score
// descending, item ascending) are the row's negatives (SCE abstract).  Then, as in
// RECE Algorithm 1's loss:
//   l+ = <x_i, y_{z_i}>,  lse_i = log(exp(l+) + sum_j exp(l_j)),  loss_i = lse_i - l+.
// Ordering uses bitonic sorts of 64-bit keys in shared memory; every reduction has a
// fixed order, so the outputs are deterministic.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kThreads = 256;

__device__ void bitonic_sort_asc(uint64_t* a, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int e = threadIdx.x; e < (P >> 1); e += blockDim.x) {
        const int lo = 2 * stride * (e / stride) + (e % stride), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if ((x > y) == up) {
          a[lo] = y;
          a[hi] = x;
        }
      }
    }
  }
  __syncthreads();
}

// Fixed-order block sum: every thread adds its strided values in index order, then a
// tree over the threads.  Result valid in all threads.
__device__ float block_sum(float v, float* red) {
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = blockDim.x >> 1; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float r = red[0];
  __syncthreads();
  return r;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) k_merge_loss(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    int64_t N, int64_t C, int d, int k, int n_r, int P, const float* __restrict__ list_score,
    const int32_t* __restrict__ list_item, int32_t* __restrict__ selected,
    float* __restrict__ lse_out, float* __restrict__ row_loss, float* __restrict__ logits,
    uint32_t* status) {
  extern __shared__ __align__(16) uint64_t sk[];  // [2][P]
  uint64_t* tmp = sk + P;
  __shared__ float red[kThreads];
  __shared__ int sh_count;
  const int64_t i = blockIdx.x;
  const int tid = threadIdx.x;
  const int E = n_r * k;

  for (int e = tid; e < P; e += kThreads) {
    uint64_t v = ~0ull;  // sentinel: sorts last
    if (e < E) {
      const int r = e / k, a = e % k;
      const int64_t off = (int64_t(r) * N + i) * k + a;
      const int32_t item = list_item[off];
      if (item >= 0) {
        const uint32_t skey = score_key(list_score[off]);
        v = n_r > 1 ? ((uint64_t(uint32_t(item)) << 32) | uint32_t(~skey))  // item asc, score desc
                    : ~cand_key(skey, item);                                 // best first
      }
    }
    sk[e] = v;
  }
  if (tid == 0) sh_count = 0;
  uint64_t* order = sk;
  if (n_r > 1) {
    bitonic_sort_asc(sk, P);
    // keep the first (highest-scored) entry of every item
    for (int e = tid; e < P; e += kThreads) {
      const uint64_t v = sk[e];
      uint64_t m = ~0ull;
      if (v != ~0ull) {
        const uint32_t item = uint32_t(v >> 32);
        const bool dup = e > 0 && uint32_t(sk[e - 1] >> 32) == item;
        if (!dup) m = ~cand_key(~uint32_t(v), int32_t(item));
      }
      tmp[e] = m;
    }
    order = tmp;
  }
  bitonic_sort_asc(order, P);
  for (int e = tid; e < P; e += kThreads)
    if (order[e] != ~0ull && (e + 1 == P || order[e + 1] == ~0ull)) sh_count = e + 1;
  __syncthreads();
  const int kk = min(k, sh_count);
  for (int a = tid; a < k; a += kThreads)
    selected[i * k + a] = a < kk ? cand_item(~order[a]) : -1;

  // positive logit (warp 0), fp32, fixed reduction order
  const int32_t z = targets[i];
  const bool z_ok = z >= 0 && z < C;
  if (tid < 32) {
    float part = 0.0f;
    if (z_ok) {
      const T* x = X + i * d;
      const T* y = Y + int64_t(z) * d;
      for (int t = tid; t < d; t += 32) part = fmaf(to_f32(x[t]), to_f32(y[t]), part);
    }
    part = warp_sum(part);
    if (tid == 0) red[0] = part;
  }
  __syncthreads();
  const float lp = red[0];
  __syncthreads();
  if (logits) {
    float* lg = logits + i * (int64_t(k) + 1);
    if (tid == 0) lg[0] = z_ok ? lp : NAN;
    for (int a = tid; a < k; a += kThreads)
      lg[1 + a] = a < kk ? key_score(uint32_t((~order[a]) >> 32)) : -INFINITY;
  }
  const float best = kk > 0 ? key_score(uint32_t((~order[0]) >> 32)) : -INFINITY;
  const float m = fmaxf(lp, best);
  float part = 0.0f;
  for (int a = tid; a < kk; a += kThreads) part += expf(key_score(uint32_t((~order[a]) >> 32)) - m);
  const float s = block_sum(part, red) + expf(lp - m);
  if (tid == 0) {
    if (!z_ok) {
      raise_flag(status, RECE_DEVICE_BAD_TARGET);
      lse_out[i] = NAN;
      if (row_loss) row_loss[i] = NAN;
    } else {
      const float lse = m + logf(s);
      lse_out[i] = lse;
      if (row_loss) row_loss[i] = lse - lp;
    }
  }
}

// One CTA: loss = (sum of row losses in a fixed order) / N.
__global__ void __launch_bounds__(1024) k_mean(const float* __restrict__ row_loss, int64_t N,
                                               float* __restrict__ loss) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < N; i += blockDim.x) s += double(row_loss[i]);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x >> 1; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) loss[0] = N > 0 ? float(red[0] / double(N)) : 0.0f;
}

}  // namespace

int merge_pow2(int n_r, int k) {
  int P = 2;
  while (P < n_r * k) P <<= 1;
  return P;
}

template <typename T>
cudaError_t launch_merge_loss(const rece_plan_s& p, const T* X, const T* Y,
                              const int32_t* targets, const float* list_score,
                              const int32_t* list_item, int32_t* selected, float* lse,
                              float* row_loss, float* logits, uint32_t* status,
                              cudaStream_t st) {
  const auto& c = p.cfg;
  if (c.N == 0) return cudaSuccess;
  const int P = merge_pow2(c.n_r, c.k);
  const size_t smem = sizeof(uint64_t) * 2 * P;
  cudaError_t e = cudaFuncSetAttribute(k_merge_loss<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  k_merge_loss<T><<<unsigned(c.N), kThreads, smem, st>>>(X, Y, targets, c.N, c.C, c.d, c.k,
                                                         c.n_r, P, list_score, list_item,
                                                         selected, lse, row_loss, logits,
                                                         status);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_mean(const float* row_loss, int64_t N, float* loss, cudaStream_t st) {
  k_mean<<<1, 1024, 0, st>>>(row_loss, N, loss);
  count_launches(1);
  return cudaGetLastError();
}

template cudaError_t launch_merge_loss<float>(const rece_plan_s&, const float*, const float*,
                                              const int32_t*, const float*, const int32_t*,
                                              int32_t*, float*, float*, float*, uint32_t*,
                                              cudaStream_t);
template cudaError_t launch_merge_loss<__nv_bfloat16>(const rece_plan_s&, const __nv_bfloat16*,
                                                      const __nv_bfloat16*, const int32_t*,
                                                      const float*, const int32_t*, int32_t*,
                                                      float*, float*, float*, uint32_t*,
                                                      cudaStream_t);

}  // namespace rece
