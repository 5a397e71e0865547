// backward.cu -- step 6 of the path: gradients of the reduced loss (RECE, equation 4,
// restricted to the positive and the kept negatives; selection held constant).
//
//   g_ij = (exp(l_ij - lse_i) - [j == z_i]) * dloss / N
//   dX_i = sum_j g_ij y_j          (one warp per row, slots in order: deterministic)
//   dY_j = sum_i g_ij x_i          (no float atomics: the (item, row) pairs are put in
//                                   item order by a stable LSD radix sort, then every
//                                   item sums its pairs in row order)
// Pair e = i*(k+1) + s holds slot s of row i (s = 0: the positive, s >= 1: selected
// negative s-1); an empty slot carries the key C, which sorts after every item.
#include "common.cuh"
#include "plan.h"

namespace rece {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float warp_dot(const T* __restrict__ a, const T* __restrict__ b,
                                          int d, int lane) {
  float s = 0.0f;
  for (int t = lane; t < d; t += 32) s = fmaf(to_f32(a[t]), to_f32(b[t]), s);
  return warp_sum(s);
}

// One warp per row: coefficients g of every slot, the pair keys, and dX_i.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_rows(
    const T* __restrict__ X, const T* __restrict__ Y, const int32_t* __restrict__ targets,
    const int32_t* __restrict__ selected, const float* __restrict__ lse,
    const float* __restrict__ dloss, int64_t N, int64_t C, int d, int k,
    int32_t* __restrict__ e_key, float* __restrict__ e_g, float* __restrict__ dX,
    uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (i >= N) return;
  const float scale = dloss[0] / float(N);
  const float li = lse[i];
  const T* x = X + i * d;
  const int slots = k + 1;
  int32_t* keys = e_key + i * slots;
  float* gs = e_g + i * slots;
  for (int s = 0; s < slots; ++s) {
    int32_t j = s == 0 ? targets[i] : selected[i * k + (s - 1)];
    float g = 0.0f;
    if (j >= 0 && j < C) {
      const float l = warp_dot(x, Y + int64_t(j) * d, d, lane);
      const float p = expf(l - li);
      g = (s == 0 ? p - 1.0f : p) * scale;
    } else {
      if (s == 0 && lane == 0) raise_flag(status, RECE_DEVICE_BAD_TARGET);
      j = int32_t(C);
    }
    if (lane == 0) {
      keys[s] = j;
      gs[s] = g;
    }
  }
  __syncwarp();
  for (int t0 = 0; t0 < d; t0 += 32 * 4) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int s = 0; s < slots; ++s) {
      const int32_t j = keys[s];
      if (j >= C) continue;
      const float g = gs[s];
      const T* y = Y + int64_t(j) * d;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * 32 + lane;
        if (t < d) acc[u] = fmaf(g, to_f32(y[t]), acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + u * 32 + lane;
      if (t < d) dX[i * d + t] = acc[u];
    }
  }
}

__device__ __forceinline__ int64_t lower_bound(const int32_t* a, int64_t n, int32_t v) {
  int64_t lo = 0, hi = n;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// One warp per item: dY_j = sum over its pairs (row order) of g * x_row.
template <typename T>
__global__ void __launch_bounds__(kThreads) k_bwd_items(
    const T* __restrict__ X, int64_t C, int d, int k, int64_t E,
    const int32_t* __restrict__ sorted_key, const int32_t* __restrict__ order,
    const float* __restrict__ e_g, float* __restrict__ dY) {
  const int lane = threadIdx.x & 31;
  const int64_t j = int64_t(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  if (j >= C) return;
  const int64_t lo = lower_bound(sorted_key, E, int32_t(j));
  const int64_t hi = lower_bound(sorted_key, E, int32_t(j + 1));
  const int slots = k + 1;
  for (int t0 = 0; t0 < d; t0 += 32 * 4) {
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int64_t p = lo; p < hi; ++p) {
      const int32_t e = order[p];
      const float g = e_g[e];
      const T* x = X + int64_t(e / slots) * d;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = t0 + u * 32 + lane;
        if (t < d) acc[u] = fmaf(g, to_f32(x[t]), acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + u * 32 + lane;
      if (t < d) dY[j * d + t] = acc[u];
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_backward(const rece_plan_s& p, const T* X, const T* Y,
                            const int32_t* targets, const int32_t* selected, const float* lse,
                            const float* dloss, char* ws, float* dX, float* dY,
                            uint32_t* status, cudaStream_t st) {
  const auto& c = p.cfg;
  const Layout& L = p.lay;
  const int64_t E = p.entries;
  int32_t* e_key = reinterpret_cast<int32_t*>(ws + L.e_key);
  float* e_g = reinterpret_cast<float*>(ws + L.e_g);
  int32_t* perm_a = reinterpret_cast<int32_t*>(ws + L.e_perm_a);
  int32_t* perm_b = reinterpret_cast<int32_t*>(ws + L.e_perm_b);
  int32_t* sorted_key = reinterpret_cast<int32_t*>(ws + L.e_sorted_key);
  void* scratch = ws + L.e_scratch;
  const int warps = kThreads / 32;
  stage_mark(p, RECE_STAGE_BWD_ROWS, 0, st);
  if (c.N > 0) {
    k_bwd_rows<T><<<unsigned(ceil_div(c.N, warps)), kThreads, 0, st>>>(
        X, Y, targets, selected, lse, dloss, c.N, c.C, c.d, c.k, e_key, e_g, dX, status);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  stage_mark(p, RECE_STAGE_BWD_ROWS, 1, st);
  stage_mark(p, RECE_STAGE_BWD_SORT, 0, st);
  // LSD radix sort of the pairs by item key (values 0..C), 8 bits per pass
  const int32_t* in = nullptr;
  int32_t* out = perm_a;
  for (int shift = 0; shift < p.item_bits; shift += 8) {
    const int bits = min(8, p.item_bits - shift);
    const bool last = shift + 8 >= p.item_bits;
    cudaError_t e = launch_sort_pass(e_key, in, E, shift, bits, scratch, out,
                                     last ? sorted_key : nullptr, nullptr, st);
    if (e != cudaSuccess) return e;
    in = out;
    out = (out == perm_a) ? perm_b : perm_a;
  }
  stage_mark(p, RECE_STAGE_BWD_SORT, 1, st);
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 0, st);
  k_bwd_items<T><<<unsigned(ceil_div(c.C, warps)), kThreads, 0, st>>>(X, c.C, c.d, c.k, E,
                                                                      sorted_key, in, e_g, dY);
  count_launches(1);
  stage_mark(p, RECE_STAGE_BWD_ITEMS, 1, st);
  return cudaGetLastError();
}

template cudaError_t launch_backward<float>(const rece_plan_s&, const float*, const float*,
                                            const int32_t*, const int32_t*, const float*,
                                            const float*, char*, float*, float*, uint32_t*,
                                            cudaStream_t);
template cudaError_t launch_backward<__nv_bfloat16>(const rece_plan_s&, const __nv_bfloat16*,
                                                    const __nv_bfloat16*, const int32_t*,
                                                    const int32_t*, const float*, const float*,
                                                    char*, float*, float*, uint32_t*,
                                                    cudaStream_t);

}  // namespace rece
